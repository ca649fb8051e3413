// gemm_swap.cuh -- the grouped GEMMs for small per-expert batches, with the
// operands swapped (all five formats).
//
// When an expert receives only a few routed rows (decode, or many experts
// per token), a 128-row tile of routed rows is mostly padding and the tensor
// core time per K block, not the weight stream, sets the pace.  Here the
// weights are the MMA's M side and the routed rows its N side: a tile is
// (active expert, 256 weight rows = the same prepared block as the large-M
// GEMM, kNT = 32 routed rows), issued as two M128 x N32 MMAs per K step
// (weight rows 0-127 and 128-255), so the tensor work follows the rows that
// exist.  The accumulators are 128 TMEM lanes (weight rows) x 32 columns
// (routed rows); per-K-block FP8 partials take 64 columns, so eight of them
// are in flight.
//
// Block-scaled formats (NVFP4, MXFP8): the weights' scale tiles come with the
// prepared block and are the MMA's A-side scale factors; the routed rows'
// scales are its B-side (N = 32) scale factors.  Those are assembled per
// stage in 512-byte tiles of the same layout as the weights' (row r of a
// 128-row tile at byte 16 r + 4 ((r mod 128) / 32)), of which 32 rows use
// only the first 4-byte group: one tile per 64 K elements for NVFP4 (four
// E4M3 scales per row), one per stage for MXFP8 (four UE8M0 scales per row,
// one per 32-element MMA).  A copier warp moves every stage's tiles into the
// stage's TMEM scale buffer (tcgen05.cp), as in the large-M GEMM.
//
// Roles as in the large-M GEMM: warp 0 loads the stage -- lane 0 one bulk
// copy of the prepared weight block and, for down, the 32 routed rows of the
// intermediate by TMA; for gate_up the whole warp copies the routed rows
// straight from x by token id (eight 16-byte cp.async per lane into the
// swizzled rows, so no gather is needed); with block scales every lane also
// copies its routed row's scale words (4-byte cp.async, from x's scales or
// from the intermediate's scale tiles) -- warp 1 lane 0 issues the MMAs,
// (NVFP4, MXFP8) warp 2 lane 0 copies the scale factors, and the last eight
// warps are the epilogue: warp (q, half) reads lanes 32q..32q+31 of the
// accumulator of weight rows 128*half.., one weight row per thread and 32
// routed rows in its registers.
//
// Gate_up epilogue: every thread stages its FP32 row (promoted, or scaled by
// the per-expert / per-tensor factors) in shared memory; after a barrier of
// the eight warps each warp takes four routed rows, one lane per four
// intermediate columns, forms the activation from the staged gate and up
// rows, re-quantises (BF16; FP8 with one scale per routed row and 128
// columns; FP8 per-tensor against the expert's static scale; MXFP8 per 32
// columns across 8 lanes; NVFP4 per 16 columns across 4 lanes) and writes
// the row segment whole, and the block scales into the intermediate's scale
// tiles.
// Down epilogue: a thread holds one output column for 32 routed rows and adds
// them, router-weighted, into the FP32 accumulator rows of their tokens
// (a warp's 32 lanes cover 128 contiguous bytes of one row), or stores them
// in staged mode.
#pragma once

#include "gemm.cuh"

namespace moe {

constexpr int kNT = 32;                 // routed rows per tile (the MMA's N)
constexpr int kTStage = kNT * kBK;      // 4 KB of routed rows per stage

template <int FMT, int EPI>
struct SwapCfg {
  static constexpr int kBBytes = b_block_bytes(FMT);
  // the routed rows' scale tiles of one stage (NVFP4: one per 64 K elements)
  static constexpr int kRowSFBytes = (FMT == FMT_NVFP4) ? 4 * kSFTile : (FMT == FMT_MXFP8) ? kSFTile : 0;
  static constexpr int kStageLoadBytes = kTStage + kBBytes + kRowSFBytes;
  // every stage's rows start on a 1024-byte boundary (the swizzle's period)
  static constexpr int kStageBytes = (kStageLoadBytes + 1023) / 1024 * 1024;   // 36 KB (BF16, FP8)
  static constexpr int kAccCols = 2 * kNT;                  // weight-row halves 0 | 1
  static constexpr int kAccBufs = (FMT == FMT_FP8) ? 8 : 4;
  // TMEM scale buffer of each stage, after the accumulators: NVFP4 weight
  // tiles [kc][row block] in columns 8 kc + 4 rb, row tiles in 32 + 4 kc;
  // MXFP8 weight tiles in 0 and 4, the row tile in 8
  static constexpr int kSFCol0 = kAccBufs * kAccCols;
  static constexpr int kSFCols = (FMT == FMT_NVFP4) ? 48 : (FMT == FMT_MXFP8) ? 16 : 0;
  static constexpr int kFirstEpiWarp = hw_scaled(FMT) ? 3 : 2;
  static constexpr int kThreads = (kFirstEpiWarp + kEpiWarps) * 32;
  static constexpr int kBarrierBytes = 4096;
  static constexpr int kSStride = kNT + 1;                   // floats per staged weight row
  static constexpr int kSBytes = (EPI == EPI_L1) ? kBN * kSStride * 4 : 0;
  static constexpr int kHeaderBytes = 1024;
  // as many stages as fit in 227 KB, up to 5 (gate_up) / 6 (down)
  static constexpr int kFixedBytes = 1024 /*align*/ + kHeaderBytes + kBarrierBytes + kSBytes;
  static constexpr int kFitStages = (227 * 1024 - kFixedBytes) / kStageBytes;
  static constexpr int kWantStages = (EPI == EPI_L1) ? 5 : 6;
  static constexpr int kStages = kFitStages < kWantStages ? kFitStages : kWantStages;
  static_assert(kStages >= 3, "pipeline depth");
  static_assert(kSFCol0 + kStages * kSFCols <= kTmemCols, "TMEM");
  static constexpr int kPhaseBytes = kStages * kStageBytes + kBarrierBytes + kSBytes;
  static constexpr int kSmemBytes = 1024 /*align*/ + kHeaderBytes + kPhaseBytes;
};

template <int FMT, int EPI>
__device__ __forceinline__ void gemm_phase_swap(const GemmArgs& p, const CUtensorMap* tmA, uint8_t* smem,
                                                uint32_t tmem, volatile int* abort_flag, int cta, int ncta) {
  using Cfg = SwapCfg<FMT, EPI>;
  constexpr int S = Cfg::kStages;
  constexpr int NACC = Cfg::kAccBufs;
  constexpr int SB = Cfg::kStageBytes;
  constexpr int BB = b_block_bytes(FMT);
  constexpr bool kRowSF = hw_scaled(FMT);   // routed rows carry block scales

  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * SB);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* final_bar = acc_empty + NACC;
  uint64_t* sbar = final_bar + 1;    // L1: [0] rows staged, [1] staged rows consumed
  uint64_t* sf_full = sbar + 2;      // NVFP4 / MXFP8: scale buffer s holds stage s's scales
  uint64_t* sf_final = sf_full + S;  // NVFP4 / MXFP8: the copier's last copies completed
  float* stage_rows = reinterpret_cast<float*>(smem + S * SB + Cfg::kBarrierBytes);  // L1: [256][kSStride]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // gate_up reading the routed rows straight from x (no gather); with block
  // scales the rows' scale words too (both legs): the whole producer warp
  // copies them, 32 arrivals more per stage
  const bool direct = EPI == EPI_L1 && p.x_rows != nullptr;
  const bool warp_copies = direct || kRowSF;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], warp_copies ? 1 + 32 : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(final_bar, 1);
    mbar_init(&sbar[0], kEpiWarps * 32);
    mbar_init(&sbar[1], kEpiWarps * 32);
    mbar_init(sf_final, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(tmA);
  __syncthreads();

  const int na = *p.num_active;
  const int total = (na > 0) ? __ldg(p.tile_offsets + na) * p.n_tiles : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (warp_copies || lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int T = cta; T < total; T += ncta) {
        TileInfo t;
        decode_tile(p, na, T, t);
        const uint8_t* wb =
            p.wB + (static_cast<size_t>(t.e) * p.n_tiles + t.n_tile) * p.k_stages * BB;
        // direct: lane l brings routed row l of the tile (row 0's token for
        // the rows past the tile's end, whose results are never used)
        const uint8_t* xrow = nullptr;
        // block scales of routed row `lane`: the first word of the stage and
        // the strides from one stage / one 64-element K step to the next
        const uint8_t* sf_src = nullptr;
        int sf_ks = 0;
        if (direct) {
          const int r = t.row0 + (lane < t.rows ? lane : 0);
          const int tok = __ldg(p.src_info + r) / p.topk;
          xrow = p.x_rows + static_cast<size_t>(tok) * p.x_row_bytes;
          if (kRowSF) {
            // x's scales [M][x_sf_ld]: 16 (NVFP4) or 4 (MXFP8) bytes per stage
            sf_src = p.x_sf_rows + static_cast<size_t>(tok) * p.x_sf_ld;
            sf_ks = (FMT == FMT_NVFP4) ? 16 : 4;
          }
        } else if (kRowSF) {
          // the intermediate's scale tiles [P/128][K/64 | K/128], padded row
          // srow0 + lane (inside the expert's 128-padded block, so in bounds
          // for the rows past the tile's end too)
          const int pr = t.srow0 + lane;
          sf_src = p.sfa + static_cast<size_t>(pr >> 7) * p.sfa_kc * kSFTile + (pr & 31) * 16 + ((pr >> 5) & 3) * 4;
          sf_ks = (FMT == FMT_NVFP4) ? 4 * kSFTile : kSFTile;
        }
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, 21)) goto producer_done;
          uint8_t* st = smem + stage * SB;
          if (warp_copies) {
            if (direct) {
              // row `lane` of the 128-byte-swizzled tile: 16-byte chunk c at c ^ (lane mod 8)
              const uint8_t* src = xrow + ks * kBK;
              uint8_t* dst = st + lane * kBK;
#pragma unroll
              for (int c = 0; c < 8; ++c) cp_async16(dst + ((c ^ (lane & 7)) << 4), src + (c << 4));
            }
            if constexpr (kRowSF) {
              uint8_t* dst = st + kTStage + BB + lane * 16;
              const uint8_t* src = sf_src + static_cast<size_t>(ks) * sf_ks;
              if (FMT == FMT_NVFP4) {
                // tile kc: the row's four scales of K elements 64 kc .. 64 kc + 63
                const int kc_step = direct ? 4 : kSFTile;
#pragma unroll
                for (int kc = 0; kc < 4; ++kc) cp_async4(dst + kc * kSFTile, src + kc * kc_step);
              } else {
                cp_async4(dst, src);
              }
            }
            cp_async_arrive(&full[stage]);
            if (lane == 0) {
              if (direct) {
                mbar_arrive_expect_tx(&full[stage], BB);
              } else {
                mbar_arrive_expect_tx(&full[stage], kTStage + BB);
                tma_load_2d(st, tmA, &full[stage], ks * kBK, t.row0);
              }
              bulk_load(st + kTStage, wb + static_cast<size_t>(ks) * BB, BB, &full[stage]);
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], kTStage + BB);
            tma_load_2d(st, tmA, &full[stage], ks * kBK, t.row0);
            bulk_load(st + kTStage, wb + static_cast<size_t>(ks) * BB, BB, &full[stage]);
          }
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (warp_copies) asm volatile("cp.async.wait_all;" ::: "memory");
      if (*abort_flag && lane == 0) {
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < S && i < issued; ++i) {
          if (--st < 0) {
            st = S - 1;
            ph ^= 1u;
          }
          mbar_drain(&full[st], ph);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = (FMT == FMT_BF16)    ? idesc_dense(1, 1, kNT)
                                  : (FMT == FMT_NVFP4) ? idesc_nvf4(kNT)
                                  : (FMT == FMT_MXFP8) ? idesc_mxf8(kNT, 0)
                                                       : idesc_dense(0, 0, kNT);
      int stage = 0;
      uint32_t phase = 0;
      int ab = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int T = cta; T < total && ok; T += ncta) {
        if (FMT != FMT_FP8) {
          if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, abort_flag, p.status, 22)) break;
          tc_fence_after();
        }
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, 23)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // rows written by cp.async (generic proxy) are read by the MMA (async proxy)
          if (direct) fence_async_smem();
          if (kRowSF) {
            if (!mbar_wait(&sf_full[stage], phase, abort_flag, p.status, 29)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (FMT == FMT_FP8) {
            if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, abort_flag, p.status, 24)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d0 = tmem + ab * Cfg::kAccCols;
          const uint32_t sf = tmem + Cfg::kSFCol0 + Cfg::kSFCols * stage;
          uint8_t* st = smem + stage * SB;
          const uint64_t bdesc = sdesc_sw128(smem_u32(st));                       // routed rows
          const uint64_t a0 = sdesc_sw128(smem_u32(st + kTStage));                // weight rows 0..127
          const uint64_t a1 = sdesc_sw128(smem_u32(st + kTStage + kBStage / 2));  // weight rows 128..255
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            const uint32_t acc = (FMT == FMT_FP8) ? (kc > 0) : ((ks | kc) != 0);
            const uint64_t b = bdesc + static_cast<uint64_t>(2 * kc);
            const uint64_t w0 = a0 + static_cast<uint64_t>(2 * kc);
            const uint64_t w1 = a1 + static_cast<uint64_t>(2 * kc);
            if (FMT == FMT_BF16) {
              mma_f16(d0, w0, b, kIdesc, acc);
              mma_f16(d0 + kNT, w1, b, kIdesc, acc);
            } else if (FMT == FMT_NVFP4) {
              mma_nvf4(d0, w0, b, kIdesc, sf + 8 * kc, sf + 32 + 4 * kc, acc);
              mma_nvf4(d0 + kNT, w1, b, kIdesc, sf + 8 * kc + 4, sf + 32 + 4 * kc, acc);
            } else if (FMT == FMT_MXFP8) {
              // one UE8M0 scale per 32-wide K step: byte kc of the stage's scale words
              mma_mxf8(d0, w0, b, idesc_mxf8(kNT, kc), sf, sf + 8, acc);
              mma_mxf8(d0 + kNT, w1, b, idesc_mxf8(kNT, kc), sf + 4, sf + 8, acc);
            } else {
              mma_f8(d0, w0, b, kIdesc, acc);
              mma_f8(d0 + kNT, w1, b, kIdesc, acc);
            }
          }
          mma_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
          if (FMT == FMT_FP8) {
            mma_commit(&acc_full[ab]);
            if (++ab == NACC) {
              ab = 0;
              aphase ^= 1u;
            }
          }
        }
        if (FMT != FMT_FP8 && ok) {
          mma_commit(&acc_full[ab]);
          if (++ab == NACC) {
            ab = 0;
            aphase ^= 1u;
          }
        }
      }
      mma_commit(final_bar);
      mbar_drain(final_bar, 0);
    }
  } else if (kRowSF && warp == 2) {
    // ------------------------------------------------------------ scale copier
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int T = cta; T < total; T += ncta) {
        bool ok = true;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          // The stage has landed, so the MMAs that last read its scale buffer
          // (the stage's previous use) have completed.
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, 30)) {
            ok = false;
            break;
          }
          tc_fence_after();
          fence_async_smem();   // the row tiles were written by cp.async
          const uint32_t wsf = smem_u32(smem + stage * SB + kTStage + kBStage);   // weight tiles
          const uint32_t rsf = smem_u32(smem + stage * SB + kTStage + BB);        // routed-row tiles
          const uint32_t dst = tmem + Cfg::kSFCol0 + Cfg::kSFCols * stage;
          if (FMT == FMT_NVFP4) {
            // prepared weight tiles: [row block][kc]
#pragma unroll
            for (int kc = 0; kc < 4; ++kc) {
              tmem_copy_sf(dst + 8 * kc, sdesc_sf_tile(wsf + kc * kSFTile));
              tmem_copy_sf(dst + 8 * kc + 4, sdesc_sf_tile(wsf + (4 + kc) * kSFTile));
              tmem_copy_sf(dst + 32 + 4 * kc, sdesc_sf_tile(rsf + kc * kSFTile));
            }
          } else {
            tmem_copy_sf(dst, sdesc_sf_tile(wsf));
            tmem_copy_sf(dst + 4, sdesc_sf_tile(wsf + kSFTile));
            tmem_copy_sf(dst + 8, sdesc_sf_tile(rsf));
          }
          mma_commit(&sf_full[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      mma_commit(sf_final);
      mbar_drain(sf_final, 0);
    }
  } else if (warp >= Cfg::kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - Cfg::kFirstEpiWarp;
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    const int half = ew >> 2;                      // weight rows 128*half ..
    const int wr = half * 128 + q * 32 + lane;     // this thread's weight row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int ab = 0;
    uint32_t aphase = 0;
    uint32_t spar = 0;
    for (int T = cta; T < total; T += ncta) {
      TileInfo t;
      decode_tile_warp(p, na, T, t, lane);
      const bool lane_row = lane < t.rows;         // routed row `lane` of the tile exists
      // down leg: this lane's routed row -> token and router weight; NVFP4
      // gate_up with per-token rowwise scales: its token's scale
      const bool gather_wgt = EPI == EPI_L2_ACC && lane_row;
      const bool row_scaled = EPI == EPI_L1 && FMT == FMT_NVFP4 && p.x_row_scale != nullptr;
      const int s_flat = (gather_wgt || (row_scaled && lane_row)) ? __ldg(p.src_info + t.row0 + lane) : 0;
      float wgt = 1.0f;

      float acc[kNT];
      if constexpr (FMT == FMT_FP8) {
#pragma unroll
        for (int i = 0; i < kNT; ++i) acc[i] = 0.0f;
        // the weight block of this warp's rows (warp-uniform)
        const int wrow = (EPI == EPI_L1) ? l1_tile_row(t.n_tile, wr, p.I, l1_group(FMT)) : (t.n_tile * kBN + wr);
        const float* sbe = p.sb + (static_cast<size_t>(t.e) * p.sb_nb + (wrow >> 7)) * p.sb_kb;
        // lane i holds routed row i's activation scale of the next K block:
        // from x's scales by token (direct), or the gathered transposed copy
        const float* sa_col;
        size_t sa_step;
        if (direct) {
          const int r = t.row0 + (lane_row ? lane : 0);
          sa_col = p.x_sc + static_cast<size_t>(__ldg(p.src_info + r) / p.topk) * p.x_sc_ld;
          sa_step = 1;
        } else {
          sa_col = p.sa_t + t.srow0 + lane;
          sa_step = static_cast<size_t>(p.sa_ld);
        }
        float nx_sa = sa_col[0];
        bool ok = true;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          const float sa = nx_sa;
          if (ks + 1 < p.k_stages) nx_sa = sa_col[static_cast<size_t>(ks + 1) * sa_step];
          if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 25)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float sbk = __ldg(sbe + ks);
          float v[kNT];
          __syncwarp();
          tmem_ld32(tmem + ab * Cfg::kAccCols + half * kNT + lane_off, v);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          if (++ab == NACC) {
            ab = 0;
            aphase ^= 1u;
          }
          if (ks == 0 && gather_wgt) wgt = __ldg(p.topk_weights + s_flat);
#pragma unroll
          for (int i = 0; i < kNT; ++i) acc[i] = fmaf(v[i], __shfl_sync(0xFFFFFFFFu, sa, i) * sbk, acc[i]);
        }
        if (!ok) break;
      } else {
        // the factor of routed row `lane` (NVFP4 rowwise) is loaded before the wait
        const float row_s = (row_scaled && lane_row)
                                ? __uint_as_float(static_cast<uint32_t>(__ldg(p.x_row_scale + s_flat / p.topk)) << 16)
                                : 1.0f;
        if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 26)) break;
        tc_fence_after();
        __syncwarp();
        tmem_ld32(tmem + ab * Cfg::kAccCols + half * kNT + lane_off, acc);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (++ab == NACC) {
          ab = 0;
          aphase ^= 1u;
        }
        if (gather_wgt) wgt = __ldg(p.topk_weights + s_flat);
        if (FMT == FMT_FP8T) {
          // (activation scale x weight scale) or (re-quant scale x weight scale)
          float alpha = __ldg(p.alpha + t.e);
          if (p.alpha_scalar) alpha = __fmul_rn(__ldg(p.alpha_scalar), alpha);
          if (p.alpha_e2) alpha = __fmul_rn(__ldg(p.alpha_e2 + t.e), alpha);
#pragma unroll
          for (int i = 0; i < kNT; ++i) acc[i] = __fmul_rn(acc[i], alpha);
        }
        if (FMT == FMT_NVFP4) {
          const float alpha = __ldg(p.alpha + t.e);
          if (row_scaled) {
#pragma unroll
            for (int i = 0; i < kNT; ++i)
              acc[i] = __fmul_rn(acc[i], __fmul_rn(alpha, __shfl_sync(0xFFFFFFFFu, row_s, i)));
          } else {
#pragma unroll
            for (int i = 0; i < kNT; ++i) acc[i] = __fmul_rn(acc[i], alpha);
          }
        }
      }

      if constexpr (EPI == EPI_L1) {
        // stage this weight row's 32 values, then each warp finishes 4 routed rows
#pragma unroll
        for (int i = 0; i < kNT; ++i) stage_rows[wr * Cfg::kSStride + i] = acc[i];
        mbar_arrive(&sbar[0]);
        if (!mbar_wait(&sbar[0], spar, abort_flag, p.status, 27)) break;
        constexpr int G = l1_group(FMT);
        const int c0 = 4 * lane;                        // intermediate columns c0..c0+3 of the tile
        const int gate_row0 = l1_gate_row(c0, G);       // weight rows of gate (c) and up (c + G)
        const int hc0 = t.n_tile * 128 + c0;            // ... as columns of the intermediate row
        for (int j = 0; j < 4; ++j) {
          const int tr = ew * 4 + j;                    // routed row of the tile (warp-uniform)
          float h[4];
          float gv[4], uv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            gv[i] = stage_rows[(gate_row0 + i) * Cfg::kSStride + tr];
            uv[i] = stage_rows[(gate_row0 + G + i) * Cfg::kSStride + tr];
          }
          if (p.fast_math) {
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = l1_act<true>(gv[i], uv[i], p.clamp, p.act_a, p.act_b);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = l1_act<false>(gv[i], uv[i], p.clamp, p.act_a, p.act_b);
          }
          const bool row_ok = tr < t.rows;
          uint8_t* hrow = p.h_out + static_cast<size_t>(t.row0 + tr) * p.h_row_bytes;
          if constexpr (FMT == FMT_FP8) {
            float amax = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fabsf(h[2]), fabsf(h[3])));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
            const float s = __fdiv_rn(amax, 448.0f);
            const float inv = (s != 0.0f) ? __frcp_rn(s) : 0.0f;
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[0], inv), __fmul_rn(h[1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(h[2], inv), __fmul_rn(h[3], inv));
            if (row_ok) {
              *reinterpret_cast<uint32_t*>(hrow + hc0) = (s != 0.0f) ? (lo | (hi << 16)) : 0u;
              if (lane == 0) p.h_scale_t[static_cast<size_t>(t.n_tile) * p.h_scale_ld + t.srow0 + tr] = s;
            }
          } else if constexpr (FMT == FMT_FP8T) {
            // one static scale per expert: codes e4m3(h * (1 / G)), saturating
            const float inv = __frcp_rn(__ldg(p.c_in + t.e));
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[0], inv), __fmul_rn(h[1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(h[2], inv), __fmul_rn(h[3], inv));
            if (row_ok) *reinterpret_cast<uint32_t*>(hrow + hc0) = lo | (hi << 16);
          } else if constexpr (FMT == FMT_MXFP8) {
            // 32-column block over 8 lanes: scale 2^X, X = floor(log2 amax) - 8
            // clamped to [-127, 127], read off amax's exponent field (a zero
            // or subnormal amax gives -127); codes e4m3(h * 2^-X), saturating
            float amax = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fabsf(h[2]), fabsf(h[3])));
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
            const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
            const int X = ex == 0 ? -127 : max(ex - 135, -127);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);   // 2^-X
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[0], inv), __fmul_rn(h[1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(h[2], inv), __fmul_rn(h[3], inv));
            if (row_ok) {
              *reinterpret_cast<uint32_t*>(hrow + hc0) = lo | (hi << 16);
              if ((lane & 7) == 0)
                p.h_sf[sf_tile_offset(t.srow0 + tr, hc0 >> 5, p.h_sf_kc)] = static_cast<uint8_t>(X + 127);
            }
          } else if constexpr (FMT == FMT_NVFP4) {
            // 16-column block over 4 lanes: E4M3 scale of amax / (6 G), codes
            // e2m1(h / (scale G)), against the expert's c_input_scales G
            float amax = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fabsf(h[2]), fabsf(h[3])));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
            const float Gs = __ldg(p.c_in + t.e);
            const uint32_t sf_code = cvt_e4m3x2(__fdiv_rn(amax, __fmul_rn(6.0f, Gs)), 0.0f) & 0xFFu;
            const float sfv = e4m3_to_f32(sf_code);
            uint32_t w = 0;
            if (sfv != 0.0f) {
              const float inv = __frcp_rn(__fmul_rn(sfv, Gs));
              w = cvt_e2m1x2(__fmul_rn(h[0], inv), __fmul_rn(h[1], inv)) |
                  (cvt_e2m1x2(__fmul_rn(h[2], inv), __fmul_rn(h[3], inv)) << 8);
            }
            if (row_ok) {
              *reinterpret_cast<uint16_t*>(hrow + hc0 / 2) = static_cast<uint16_t>(w);
              if ((lane & 3) == 0)
                p.h_sf[sf_tile_offset(t.srow0 + tr, hc0 >> 4, p.h_sf_kc)] = static_cast<uint8_t>(sf_code);
            }
          } else {
            if (row_ok)
              *reinterpret_cast<uint2*>(hrow + hc0 * 2) =
                  make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
          }
        }
        // the staging rows may be overwritten once all eight warps are done
        mbar_arrive(&sbar[1]);
        if (!mbar_wait(&sbar[1], spar, abort_flag, p.status, 28)) break;
        spar ^= 1u;
      } else {
        // down leg: output column n of the tile for each routed row
        const int n = t.n_tile * kBN + wr;
        const int tok_l = gather_wgt ? s_flat / p.topk : 0;
#pragma unroll
        for (int i = 0; i < kNT; ++i) {
          if (i >= t.rows) break;   // warp-uniform
          if (EPI == EPI_L2_ACC) {
            const int tok = __shfl_sync(0xFFFFFFFFu, tok_l, i);
            const float w = __shfl_sync(0xFFFFFFFFu, wgt, i);
            atomicAdd(p.out + static_cast<size_t>(tok) * p.H + n, acc[i] * w);
          } else {
            p.out[static_cast<size_t>(t.row0 + i) * p.H + n] = acc[i];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

template <int FMT, int EPI>
__global__ void __launch_bounds__(SwapCfg<FMT, EPI>::kThreads, 1)
    moe_gemm_swap_kernel(const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmA) {
  uint8_t* base = smem_base_1024();
  SmemHeader* hdr = reinterpret_cast<SmemHeader*>(base);
  if (threadIdx.x == 0) hdr->abort = 0;
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&hdr->tmem, kTmemCols);
  pdl_trigger();
  pdl_wait();   // the layout, tile table, activations, accumulator and header come from earlier kernels
  if (threadIdx.x == 0) hdr->wait_us = wait_limit_us(p.status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hdr->tmem;
  gemm_phase_swap<FMT, EPI>(p, &tmA, base + SwapCfg<FMT, EPI>::kHeaderBytes, tmem, &hdr->abort, blockIdx.x,
                            gridDim.x);
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace moe

// gemm.cuh -- the grouped expert GEMMs of the routed MoE FFN on sm_100a.
//
// One persistent, warp-specialised kernel template serves both legs of the
// expert FFN (Struct_mega_ffn_ep_combine_send: "L1" gate_up and "L2" down,
// walking one shared active-expert list) in three element formats:
//
//   BF16   tcgen05.mma kind::f16, FP32 accumulation over all of K in TMEM
//   NVFP4  tcgen05.mma kind::mxf4nvf4 block_scale scale_vec::4X: e2m1
//          operands, E4M3 scale per 16 elements, copied to TMEM with
//          tcgen05.cp; FP32 accumulation over all of K in TMEM
//   FP8    tcgen05.mma kind::f8f6f4 (E4M3 x E4M3): the tensor cores sum one
//          128-wide K block into a TMEM partial; the epilogue warps promote
//          it, partial * (a_scale[row, kb] * b_scale[n_blk, kb]), into FP32
//          registers (the per-128 FP32 block scales have no hardware form)
//
// Roles: warp 0 lane 0 issues TMA loads of 128 x 128-byte A rows and
// 256 x 128-byte B rows per stage (+ the NVFP4 scale tiles as bulk copies)
// into a STAGES-deep ring guarded by mbarriers; warp 1 lane 0 issues the
// MMAs (M = 128, N = 256, four K steps of 32 bytes per stage) and commits
// them to the ring and to the accumulator barriers; the remaining warps are
// the epilogue, one TMEM lane (= one output row) per thread.
//
// Tiles are (active expert, n tile, 128-row m tile), expert-major, m
// fastest, handed out round-robin over a grid of at most one CTA per SM.
//
// L1 epilogue: g and u of the same intermediate column j sit in one tile
// (gate rows of W13 first, up rows I further down); h = min(g,c) *
// sigmoid(min(g,c)) * clamp(u,-c,c) is re-quantised in registers (BF16 by
// rounding; FP8 per 128 columns with scale amax/448; NVFP4 per 16 columns
// with an E4M3 scale against the per-expert c_input_scales) and stored in
// expert order for L2.
// L2 epilogue: every finished row is multiplied by its router weight and
// red-added (float4 atomics) into the token-ordered FP32 accumulator -- no
// (M*k, H) staging buffer -- or, in staged mode, stored per row.
//
// Every wait is bounded; a wait that runs out records MOE_ERR_TIMEOUT in the
// workspace status word, raises a CTA-wide abort flag, drains the copies and
// MMAs already in flight, frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace moe {

enum { FMT_BF16 = 0, FMT_FP8 = 1, FMT_NVFP4 = 2 };
enum { EPI_L1 = 0, EPI_L2_ACC = 1, EPI_L2_STAGED = 2 };

constexpr int kBM = 128;          // MMA M: rows of A (routed rows) per tile
constexpr int kBN = 256;          // MMA N: rows of B (weight rows) per tile
constexpr int kBK = 128;          // bytes of K per row per stage (one swizzle span)
constexpr int kAStage = kBM * kBK;            // 16 KB
constexpr int kBStage = kBN * kBK;            // 32 KB
constexpr int kSFTile = 512;                  // 128 rows x 4 scale bytes
constexpr int kSFAStage = 4 * kSFTile;        // 4 K-steps of 64 e2m1
constexpr int kSFBStage = 2 * 4 * kSFTile;    // 2 row blocks x 4 K-steps
constexpr int kTmemCols = 512;
constexpr int kSFACol = 256;                  // NVFP4: TMEM columns of the A scales
constexpr int kSFBCol = 256 + 16;             // NVFP4: TMEM columns of the B scales

template <int FMT>
struct GemmCfg {
  static constexpr int kStages = 4;
  static constexpr int kEpiWarps = (FMT == FMT_FP8) ? 8 : 4;
  // accumulator (BF16/NVFP4) or partial (FP8) buffers of 256 TMEM columns
  static constexpr int kAccBufs = (FMT == FMT_NVFP4) ? 1 : 2;
  static constexpr int kStageBytes =
      kAStage + kBStage + ((FMT == FMT_NVFP4) ? (kSFAStage + kSFBStage) : 0);
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
  static constexpr int kBarrierBytes = 4096;
  static constexpr int kSmemBytes = 1024 /*align*/ + kStages * kStageBytes + kBarrierBytes;
};

struct GemmArgs {
  int k_stages;       // K bytes / 128
  int w_rows;         // rows of B per expert: 2I (L1) or H (L2)
  int n_tiles;        // tiles along N: I/128 (L1, 128 h columns per tile) or H/256 (L2)
  int I, H, topk;
  float clamp;
  int fast_math;
  // layout (device, from the permute step)
  const int* expert_ids;
  const int* num_active;
  const int* starts;            // expert_start_indices
  const int* a_scale_offsets;
  const int* tile_offsets;
  const int* src_info;
  const float* topk_weights;
  // NVFP4 scales: 512-byte tiles [row block][K/64]
  const uint8_t* sfa;
  int sfa_kc;
  const uint8_t* sfb;
  int sfb_kc;
  // FP8 scales: A transposed [K/128][sa_ld] (padded rows), B [E][N/128][K/128]
  const float* sa_t;
  int sa_ld;
  const float* sb;
  int sb_nb, sb_kb;
  // NVFP4 per-expert scalars
  const float* alpha;   // gate_up_expert_scales (L1) or down_expert_scales (L2)
  const float* c_in;    // c_input_scales (L1 re-quant)
  // L1 output: the re-quantised intermediate, expert order
  uint8_t* h_out;
  int h_row_bytes;
  uint8_t* h_sf;        // NVFP4 scale tiles [P/128][I/64]
  int h_sf_kc;
  float* h_scale_t;     // FP8 scales transposed [I/128][h_scale_ld]
  int h_scale_ld;
  // L2 output
  float* out;           // accumulate: [M][H]; staged: [R][H]
  int* status;
};

struct TileInfo {
  int e;       // expert
  int row0;    // first routed row (expert order)
  int rows;    // valid rows in this tile (1..128)
  int srow0;   // first padded scale row
  int n_tile;
};

__device__ __forceinline__ void decode_tile(const GemmArgs& p, int na, int T, TileInfo& t) {
  const int nt = p.n_tiles;
  int lo = 0, hi = na;  // tile_offsets[lo]*nt <= T < tile_offsets[hi]*nt
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.tile_offsets + mid) * nt <= T) lo = mid; else hi = mid;
  }
  const int mt0 = __ldg(p.tile_offsets + lo);
  const int nm = __ldg(p.tile_offsets + lo + 1) - mt0;
  const int local = T - mt0 * nt;
  t.n_tile = local / nm;
  const int mt = local - t.n_tile * nm;
  t.e = __ldg(p.expert_ids + lo);
  const int start = __ldg(p.starts + t.e);
  const int cnt = __ldg(p.starts + t.e + 1) - start;
  t.row0 = start + mt * kBM;
  t.rows = min(kBM, cnt - mt * kBM);
  t.srow0 = __ldg(p.a_scale_offsets + t.e) + mt * kBM;
}

// A wait used while tearing down after an abort: ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

__device__ __forceinline__ float clamped_swiglu(float g, float u, float c, int fast) {
  const float gc = fminf(g, c);
  const float uc = fminf(fmaxf(u, -c), c);
  const float ex = fast ? __expf(-gc) : expf(-gc);
  return __fmul_rn(__fdiv_rn(gc, 1.0f + ex), uc);
}

// Byte offset of (padded row pr, scale column j) inside the 512-byte scale
// tiles [pr/128][j/4]: 32 rows x 16 bytes, row pr%32, 4-byte group
// (pr%128)/32, byte j%4.
__device__ __forceinline__ size_t sf_tile_offset(int pr, int j, int kc) {
  return (static_cast<size_t>(pr >> 7) * kc + (j >> 2)) * kSFTile + (pr & 31) * 16 +
         ((pr >> 5) & 3) * 4 + (j & 3);
}

template <int FMT, int EPI>
__global__ void __launch_bounds__(GemmCfg<FMT>::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB) {
  using Cfg = GemmCfg<FMT>;
  constexpr int S = Cfg::kStages;
  constexpr int NACC = Cfg::kAccBufs;
  constexpr int NEPI = Cfg::kEpiWarps;
  constexpr int SB = Cfg::kStageBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * SB);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* final_bar = acc_empty + NACC;
  uint64_t* xbar = final_bar + 1;  // FP8 L1: one per TMEM lane quarter
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S * SB + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xbuf = reinterpret_cast<float*>(smem + S * SB + 1024);  // FP8 L1: [2][2][128] amax

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], NEPI);
    }
    mbar_init(final_bar, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 64);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int na = *p.num_active;
  const int total = (na > 0) ? __ldg(p.tile_offsets + na) * p.n_tiles : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int T = blockIdx.x; T < total; T += gridDim.x) {
        TileInfo t;
        decode_tile(p, na, T, t);
        const int wrow = t.e * p.w_rows;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, 1)) goto producer_done;
          uint8_t* sa = smem + stage * SB;
          uint8_t* sbp = sa + kAStage;
          mbar_arrive_expect_tx(&full[stage], SB);
          const int kx = ks * kBK;
          tma_load_2d(sa, &tmA, &full[stage], kx, t.row0);
          if (EPI == EPI_L1) {
            const int j0 = t.n_tile * 128;
            if (FMT == FMT_FP8) {
              // [gate j0..+63 | up j0..+63 | gate j0+64..+127 | up j0+64..+127]
              tma_load_2d(sbp, &tmB, &full[stage], kx, wrow + j0);
              tma_load_2d(sbp + 64 * kBK, &tmB, &full[stage], kx, wrow + p.I + j0);
              tma_load_2d(sbp + 128 * kBK, &tmB, &full[stage], kx, wrow + j0 + 64);
              tma_load_2d(sbp + 192 * kBK, &tmB, &full[stage], kx, wrow + p.I + j0 + 64);
            } else {
              // [gate j0..+127 | up j0..+127]
              tma_load_2d(sbp, &tmB, &full[stage], kx, wrow + j0);
              tma_load_2d(sbp + 128 * kBK, &tmB, &full[stage], kx, wrow + p.I + j0);
            }
          } else {
            tma_load_2d(sbp, &tmB, &full[stage], kx, wrow + t.n_tile * kBN);
          }
          if (FMT == FMT_NVFP4) {
            uint8_t* sfa_s = sbp + kBStage;
            uint8_t* sfb_s = sfa_s + kSFAStage;
            bulk_load(sfa_s,
                      p.sfa + (static_cast<size_t>(t.srow0 >> 7) * p.sfa_kc + ks * 4) * kSFTile,
                      kSFAStage, &full[stage]);
            int rb0, rb1;
            if (EPI == EPI_L1) {
              rb0 = (wrow + t.n_tile * 128) >> 7;
              rb1 = (wrow + p.I + t.n_tile * 128) >> 7;
            } else {
              rb0 = (wrow + t.n_tile * kBN) >> 7;
              rb1 = rb0 + 1;
            }
            bulk_load(sfb_s, p.sfb + (static_cast<size_t>(rb0) * p.sfb_kc + ks * 4) * kSFTile,
                      4 * kSFTile, &full[stage]);
            bulk_load(sfb_s + 4 * kSFTile,
                      p.sfb + (static_cast<size_t>(rb1) * p.sfb_kc + ks * 4) * kSFTile,
                      4 * kSFTile, &full[stage]);
          }
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (*abort_flag) {
        // Let every copy already issued land before the CTA's memory goes away.
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
      constexpr uint32_t kIdesc = (FMT == FMT_BF16)  ? idesc_dense(1, 1, kBN)
                                  : (FMT == FMT_FP8) ? idesc_dense(0, 0, kBN)
                                                     : idesc_nvf4(kBN);
      int stage = 0;
      uint32_t phase = 0;
      int ab = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int T = blockIdx.x; T < total && ok; T += gridDim.x) {
        if (FMT != FMT_FP8) {
          if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, abort_flag, p.status, 2)) break;
          tc_fence_after();
        }
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (FMT == FMT_FP8) {
            if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, abort_flag, p.status, 4)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d = tmem + ab * kBN;
          uint8_t* sa = smem + stage * SB;
          uint8_t* sbp = sa + kAStage;
          const uint64_t adesc = sdesc_sw128(smem_u32(sa));
          const uint64_t bdesc = sdesc_sw128(smem_u32(sbp));
          if (FMT == FMT_NVFP4) {
            const uint32_t sfa_s = smem_u32(sbp + kBStage);
            const uint32_t sfb_s = sfa_s + kSFAStage;
#pragma unroll
            for (int kc = 0; kc < 4; ++kc) {
              tmem_copy_sf(tmem + kSFACol + 4 * kc, sdesc_sf_tile(sfa_s + kc * kSFTile));
              tmem_copy_sf(tmem + kSFBCol + 8 * kc, sdesc_sf_tile(sfb_s + kc * kSFTile));
              tmem_copy_sf(tmem + kSFBCol + 8 * kc + 4,
                           sdesc_sf_tile(sfb_s + 4 * kSFTile + kc * kSFTile));
            }
          }
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            const uint32_t acc = (FMT == FMT_FP8) ? (kc > 0) : ((ks | kc) != 0);
            const uint64_t a = adesc + static_cast<uint64_t>(2 * kc);
            const uint64_t b = bdesc + static_cast<uint64_t>(2 * kc);
            if (FMT == FMT_BF16) mma_f16(d, a, b, kIdesc, acc);
            else if (FMT == FMT_FP8) mma_f8(d, a, b, kIdesc, acc);
            else mma_nvf4(d, a, b, kIdesc, tmem + kSFACol + 4 * kc, tmem + kSFBCol + 8 * kc, acc);
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
      // Nothing may still write TMEM when it is released.
      mma_commit(final_bar);
      mbar_drain(final_bar, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int half = (NEPI == 8) ? (ew >> 2) : 0;
    const int row_local = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int ab = 0;
    uint32_t aphase = 0;
    int xpar = 0;          // FP8 L1: amax exchange buffer / barrier phase
    for (int T = blockIdx.x; T < total; T += gridDim.x) {
      TileInfo t;
      decode_tile(p, na, T, t);
      const bool valid = row_local < t.rows;
      const int r = t.row0 + row_local;
      const int pr = t.srow0 + row_local;

      if constexpr (FMT == FMT_FP8) {
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
        const float* sbe = p.sb + static_cast<size_t>(t.e) * p.sb_nb * p.sb_kb;
        int nb_lo, nb_hi;  // weight blocks of acc[0..63] and acc[64..127]
        if (EPI == EPI_L1) {
          nb_lo = (t.n_tile * 128) >> 7;
          nb_hi = (p.I + t.n_tile * 128) >> 7;
        } else {
          nb_lo = nb_hi = (t.n_tile * kBN + half * 128) >> 7;
        }
        bool ok = true;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 5)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float sa = p.sa_t[static_cast<size_t>(ks) * p.sa_ld + pr];
          const float s_lo = sa * __ldg(sbe + nb_lo * p.sb_kb + ks);
          const float s_hi = sa * __ldg(sbe + nb_hi * p.sb_kb + ks);
          const uint32_t base = tmem + ab * kBN + half * 128 + lane_off;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            __syncwarp();
            tmem_ld32(base + 32 * c, v);
            const float s = (c < 2) ? s_lo : s_hi;
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[32 * c + i] = fmaf(v[i], s, acc[32 * c + i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          if (++ab == NACC) {
            ab = 0;
            aphase ^= 1u;
          }
        }
        if (!ok) break;
        if (EPI == EPI_L1) {
          // h for intermediate columns j0 + 64*half + i, i < 64
          float h[64];
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            h[i] = clamped_swiglu(acc[i], acc[64 + i], p.clamp, p.fast_math);
            amax = fmaxf(amax, fabsf(h[i]));
          }
          // One FP8 scale covers the tile's 128 columns: combine the two
          // halves held by warps (q, 0) and (q, 1).  The buffer alternates
          // between tiles, so one barrier phase per tile suffices.
          float* xb = xbuf + xpar * 256;
          xb[half * 128 + row_local] = amax;
          mbar_arrive(&xbar[q]);
          if (!mbar_wait(&xbar[q], static_cast<uint32_t>(xpar), abort_flag, p.status, 7)) break;
          amax = fmaxf(xb[row_local], xb[128 + row_local]);
          xpar ^= 1;
          const float s = __fdiv_rn(amax, 448.0f);
          const float inv = (s != 0.0f) ? __frcp_rn(s) : 0.0f;
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[4 * i], inv), __fmul_rn(h[4 * i + 1], inv));
              const uint32_t hi =
                  cvt_e4m3x2(__fmul_rn(h[4 * i + 2], inv), __fmul_rn(h[4 * i + 3], inv));
              w[i] = (s != 0.0f) ? (lo | (hi << 16)) : 0u;
            }
            uint4* dst = reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(r) * p.h_row_bytes +
                                                  t.n_tile * 128 + half * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            if (half == 0) p.h_scale_t[static_cast<size_t>(t.n_tile) * p.h_scale_ld + pr] = s;
          }
        } else if (valid) {
          const int n0 = t.n_tile * kBN + half * 128;
          if (EPI == EPI_L2_ACC) {
            const int s_flat = __ldg(p.src_info + r);
            const int tok = s_flat / p.topk;
            const float wgt = __ldg(p.topk_weights + s_flat);
            float* dst = p.out + static_cast<size_t>(tok) * p.H + n0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              atomicAdd(reinterpret_cast<float4*>(dst) + i,
                        make_float4(acc[4 * i] * wgt, acc[4 * i + 1] * wgt, acc[4 * i + 2] * wgt,
                                    acc[4 * i + 3] * wgt));
          } else {
            float4* dst = reinterpret_cast<float4*>(p.out + static_cast<size_t>(r) * p.H + n0);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
          }
        }
      } else {
        // BF16 / NVFP4: the whole K sum is in TMEM.
        if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 6)) break;
        tc_fence_after();
        const uint32_t base = tmem + ab * kBN + lane_off;
        const float alpha = (FMT == FMT_NVFP4) ? __ldg(p.alpha + t.e) : 1.0f;
        if (EPI == EPI_L1) {
          const int j0 = t.n_tile * 128;
          const float G = (FMT == FMT_NVFP4) ? __ldg(p.c_in + t.e) : 1.0f;
          const float denom6 = __fmul_rn(6.0f, G);
#pragma unroll 1
          for (int i = 0; i < 8; ++i) {
            float g[16], u[16];
            __syncwarp();
            tmem_ld16(base + 16 * i, g);
            tmem_ld16(base + 128 + 16 * i, u);
            float h[16];
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float gg = g[j], uu = u[j];
              if (FMT == FMT_NVFP4) {
                gg = __fmul_rn(gg, alpha);
                uu = __fmul_rn(uu, alpha);
              }
              h[j] = clamped_swiglu(gg, uu, p.clamp, p.fast_math);
              amax = fmaxf(amax, fabsf(h[j]));
            }
            if (!valid) continue;
            if (FMT == FMT_BF16) {
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(h[2 * j], h[2 * j + 1]);
              uint4* dst = reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(r) * p.h_row_bytes +
                                                    (j0 + 16 * i) * 2);
              dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
              dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
              const uint32_t sf_code = cvt_e4m3x2(__fdiv_rn(amax, denom6), 0.0f) & 0xFFu;
              const float sf = e4m3_to_f32(sf_code);
              uint32_t w0 = 0, w1 = 0;
              if (sf != 0.0f) {
                const float inv = __frcp_rn(__fmul_rn(sf, G));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  w0 |= cvt_e2m1x2(__fmul_rn(h[2 * j], inv), __fmul_rn(h[2 * j + 1], inv)) << (8 * j);
                  w1 |= cvt_e2m1x2(__fmul_rn(h[8 + 2 * j], inv), __fmul_rn(h[9 + 2 * j], inv)) << (8 * j);
                }
              }
              *reinterpret_cast<uint2*>(p.h_out + static_cast<size_t>(r) * p.h_row_bytes +
                                        (j0 + 16 * i) / 2) = make_uint2(w0, w1);
              p.h_sf[sf_tile_offset(pr, (j0 >> 4) + i, p.h_sf_kc)] = static_cast<uint8_t>(sf_code);
            }
          }
        } else {
          int tok = 0;
          float wgt = alpha;
          if (valid && EPI == EPI_L2_ACC) {
            const int s_flat = __ldg(p.src_info + r);
            tok = s_flat / p.topk;
            wgt = alpha * __ldg(p.topk_weights + s_flat);
          }
          const int n0 = t.n_tile * kBN;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            float v[32];
            __syncwarp();
            tmem_ld32(base + 32 * c, v);
            if (!valid) continue;
            if (EPI == EPI_L2_ACC) {
              float* dst = p.out + static_cast<size_t>(tok) * p.H + n0 + 32 * c;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                atomicAdd(reinterpret_cast<float4*>(dst) + i,
                          make_float4(v[4 * i] * wgt, v[4 * i + 1] * wgt, v[4 * i + 2] * wgt,
                                      v[4 * i + 3] * wgt));
            } else {
              float4* dst = reinterpret_cast<float4*>(p.out + static_cast<size_t>(r) * p.H + n0 + 32 * c);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(v[4 * i] * wgt, v[4 * i + 1] * wgt, v[4 * i + 2] * wgt,
                                     v[4 * i + 3] * wgt);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (++ab == NACC) {
          ab = 0;
          aphase ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace moe

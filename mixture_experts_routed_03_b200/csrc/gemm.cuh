// gemm.cuh -- the grouped expert GEMMs of the routed MoE FFN on sm_100a.
//
// One persistent, warp-specialised kernel template serves both legs of the
// expert FFN (Struct_mega_ffn_ep_combine_send: "L1" gate_up and "L2" down,
// walking one shared active-expert list) in five element formats:
//
//   BF16   tcgen05.mma kind::f16, FP32 accumulation over all of K in TMEM
//   NVFP4  tcgen05.mma kind::mxf4nvf4 block_scale scale_vec::4X: e2m1
//          operands, E4M3 scale per 16 elements, copied to TMEM with
//          tcgen05.cp; FP32 accumulation over all of K in TMEM
//   FP8    tcgen05.mma kind::f8f6f4 (E4M3 x E4M3): the tensor cores sum one
//          128-wide K block into a TMEM partial; the epilogue warps promote
//          it, partial * (a_scale[row, kb] * b_scale[n_blk, kb]), into FP32
//          registers (the per-128 FP32 block scales have no hardware form)
//   FP8T   (per-tensor scales) tcgen05.mma kind::f8f6f4, FP32 accumulation
//          over all of K in TMEM; the epilogue applies the per-tensor and
//          per-expert scales to the sum
//   MXFP8  tcgen05.mma kind::mxf8f6f4 block_scale scale_vec::1X: E4M3
//          operands, UE8M0 scale per 32 elements (one per MMA instruction,
//          picked by the descriptor's scale-factor id), copied to TMEM with
//          tcgen05.cp; FP32 accumulation over all of K in TMEM
//
// Operands.  A (routed rows in expert order) comes by TMA, 128 rows x 128
// bytes per stage, 128-byte swizzle.  B (expert weights) is PREPARED once
// (moe_prepare_weights, the "pre-permuted" weights of mega_ffn_ep_combine_
// send): every (expert, n tile, K stage) block of 256 rows x 128 bytes is
// stored contiguously, already in the 128-byte-swizzled order the MMA reads
// (16-byte chunk c of row r at chunk c ^ (r mod 8)), followed for NVFP4 by its
// 4 KB (MXFP8: 1 KB) of scale tiles, so one bulk copy per stage streams it sequentially
// from HBM.  L1 B tiles interleave gate and up rows as [gate j0..j0+63 |
// up j0..j0+63 | gate j0+64..j0+127 | up j0+64..j0+127], so each 128-column
// half of the accumulator holds matching gate and up columns.
//
// Roles: warp 0 lane 0 issues the copies into a 4-stage ring guarded by
// mbarriers; warp 1 lane 0 issues the MMAs (M = 128, N = 256, four 32-byte K
// steps per stage) and commits them; for NVFP4 and MXFP8, warp 2 lane 0 moves each
// stage's scale factors from shared memory into the stage's own TMEM scale
// buffer (tcgen05.cp), so their issue cost overlaps the MMAs; the last 8
// warps are the epilogue, two per 32-lane TMEM quarter, one per 128-column
// half, one row per thread.
//
// Tiles are (active expert, n tile, 128-row m tile), handed out round-robin
// over at most one CTA per SM, in groups of n tiles (see decode_tile):
// expert-major with m fastest for gate_up; for down, one output n tile at a
// time while the intermediate fits in L2, else expert-major.  (Small
// per-expert batches use the swapped-operand GEMMs of gemm_swap.cuh.)
//
// L1 epilogue: h = min(g,c) * sigmoid(min(g,c)) * clamp(u,-c,c) is formed in
// registers, the accumulator is released, then h is re-quantised (BF16 by
// rounding; FP8 per 128 columns with scale amax/448; NVFP4 per 16 columns
// with an E4M3 scale against the per-expert c_input_scales; MXFP8 per 32
// columns with the power-of-two scale 2^(floor(log2 amax) - 8); FP8T
// against the per-expert c_input_scales) and stored in expert order for L2.
// L2 epilogue: the row is read into registers, the accumulator released, and
// the row, times its router weight, added into the token-ordered FP32
// accumulator -- float4 atomics through a 32 x 32 transpose (BF16, FP8, MXFP8) or
// TMA bulk reduce-adds (NVFP4); no (M*k, H) staging buffer -- or, in staged
// mode, stored per row.
//
// Every wait is bounded; a wait that runs out records MOE_ERR_TIMEOUT in the
// workspace status word, raises a CTA-wide abort flag, drains the copies and
// MMAs already in flight, frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace moe {

enum { FMT_BF16 = 0, FMT_FP8 = 1, FMT_NVFP4 = 2, FMT_MXFP8 = 3, FMT_FP8T = 4 };
enum { EPI_L1 = 0, EPI_L2_ACC = 1, EPI_L2_STAGED = 2 };

constexpr int kBM = 128;          // MMA M: rows of A (routed rows) per tile
constexpr int kBN = 256;          // MMA N: rows of B (weight rows) per tile
constexpr int kBK = 128;          // bytes of K per row per stage (one swizzle span)
constexpr int kAStage = kBM * kBK;            // 16 KB
constexpr int kBStage = kBN * kBK;            // 32 KB
constexpr int kSFTile = 512;                  // 128 rows x 4 scale bytes
constexpr int kSFAStage = 4 * kSFTile;        // 4 K-steps of 64 e2m1
constexpr int kSFBStage = 2 * 4 * kSFTile;    // 2 row blocks x 4 K-steps
constexpr int kMxSFAStage = kSFTile;          // MXFP8: 4 scales (128 E4M3) per row
constexpr int kMxSFBStage = 2 * kSFTile;      // MXFP8: 2 row blocks
constexpr int kTmemCols = 512;
// Block-scale factors in TMEM: one buffer of 48 columns per shared-memory
// stage after the accumulator (4 x 48 + 256 <= 512).  NVFP4: A scales (16
// columns) then B scales (32 columns); MXFP8: A in columns 0..3, B in
// columns 16..23.  Buffer s belongs to stage s, so the copier needs no
// release barrier: stage s's data lands only after the producer refilled
// it, which it did only after the MMAs of the stage's previous use -- the
// last readers of buffer s -- completed.
constexpr int kSFCol0 = 256;
constexpr int kSFBufCols = 48;
constexpr int kSFBOff = 16;
constexpr int kEpiWarps = 8;

// Bytes of one prepared B block (one stage of one tile).
__host__ __device__ constexpr int b_block_bytes(int fmt) {
  return kBStage + (fmt == FMT_NVFP4 ? kSFBStage : fmt == FMT_MXFP8 ? kMxSFBStage : 0);
}

// Formats whose block scales the tensor cores apply from TMEM.
__host__ __device__ constexpr bool hw_scaled(int fmt) { return fmt == FMT_NVFP4 || fmt == FMT_MXFP8; }

// Gate/up interleave of the prepared gate_up tiles: groups of G gate rows
// followed by the G matching up rows, so that every 2G accumulator columns
// hold matching gate and up columns (the epilogue threads read 128 columns
// each, G = 64, in every format).
__host__ __device__ constexpr int l1_group(int) { return 64; }

// Logical weight row held by row r (0..255) of L1 tile nt: gate and up rows
// of intermediate columns 128*nt .. 128*nt+127 in groups of G.
__host__ __device__ inline int l1_tile_row(int nt, int r, int I, int G) {
  const int g = r / G, o = r % G;
  const int col = 128 * nt + (g >> 1) * G + o;
  return (g & 1) ? I + col : col;
}

// Tile row of the gate row of intermediate column c (0..127 within the
// tile); the matching up row is G rows further.
__host__ __device__ inline int l1_gate_row(int c, int G) { return (c / G) * 2 * G + c % G; }

template <int FMT, int EPI>
struct GemmCfg {
  // L2 gives 36 KB of shared memory to the epilogue's transpose buffers
  static constexpr int kStages = (EPI == EPI_L1) ? 4 : 3;
  // accumulator (BF16/NVFP4) or partial (FP8) buffers of 256 TMEM columns
  static constexpr int kAccBufs = hw_scaled(FMT) ? 1 : 2;
  // bytes one stage's copies bring in
  static constexpr int kStageLoadBytes =
      kAStage + kBStage + ((FMT == FMT_NVFP4)   ? (kSFBStage + kSFAStage)
                           : (FMT == FMT_MXFP8) ? (kMxSFBStage + kMxSFAStage)
                                                : 0);
  // stage stride: every stage's A tile starts on a 1024-byte boundary (the
  // 128-byte swizzle's period)
  static constexpr int kStageBytes = (kStageLoadBytes + 1023) / 1024 * 1024;
  // warp 0 producer, warp 1 MMA issuer, (NVFP4, MXFP8) warp 2 scale-factor
  // copier, then the epilogue warps
  static constexpr int kFirstEpiWarp = hw_scaled(FMT) ? 3 : 2;
  static constexpr int kThreads = (kFirstEpiWarp + kEpiWarps) * 32;
  static constexpr int kBarrierBytes = 4096;
  static constexpr int kXposeStride = 36;   // floats per row of a 32 x 32 transpose buffer
  // L2: per-warp 32 x 32 FP32 transposes.  FP8 L1: per-quarter staging of
  // the 32 rows x 128 h bytes the quarter's two warps produce, so that the
  // rows leave as whole 128-byte segments (rows padded to 144 bytes against
  // bank conflicts).
  static constexpr int kHStageStride = 144;
  static constexpr int kXposeBytes = (EPI != EPI_L1)        ? kEpiWarps * 32 * kXposeStride * 4
                                     : (FMT == FMT_FP8) ? 4 * 32 * kHStageStride
                                                        : 0;
  static constexpr int kHeaderBytes = 1024;   // TMEM address, abort flag (kept across phases)
  static constexpr int kPhaseBytes = kStages * kStageBytes + kBarrierBytes + kXposeBytes;
  static constexpr int kSmemBytes = 1024 /*align*/ + kHeaderBytes + kPhaseBytes;
};

struct GemmArgs {
  int k_stages;       // K bytes / 128
  int n_tiles;        // tiles along N: I/128 (L1, 128 h columns per tile) or H/256 (L2)
  int n_group;        // n tiles per group of the tile order (1 .. n_tiles, see decode_tile)
  int I, H, topk;
  float clamp;
  int fast_math;
  // the L1 activation min(g,c) * sigmoid(act_a*min(g,c)) * (clamp(u,-c,c) + act_b):
  // act_a = 1, act_b = 0 (clamped SwiGLU) or the slope and 1 (swigluoai)
  float act_a, act_b;
  // layout (device, from the permute step)
  const int* expert_ids;
  const int* num_active;
  const int* starts;            // expert_start_indices
  const int* a_scale_offsets;
  const int* tile_offsets;       // tile table: m tiles of tile_rows rows per active expert, prefix summed
  int tile_rows;                 // 128 (kBM), or kNT for the swapped-operand GEMM
  const int* src_info;
  const float* topk_weights;
  // prepared weights: [E][n_tiles][k_stages] blocks of b_block_bytes(FMT)
  const uint8_t* wB;
  // NVFP4 / MXFP8 A scales: 512-byte tiles [row block][K/64 | K/128]
  const uint8_t* sfa;
  int sfa_kc;
  // FP8 scales: A transposed [K/128][sa_ld] (padded rows), B [E][N/128][K/128]
  const float* sa_t;
  int sa_ld;
  const float* sb;
  int sb_nb, sb_kb;
  // NVFP4 per-expert scalars: gate_up_expert_scales (L1) or
  // down_expert_scales (L2); FP8T: the experts' weight scales, times
  // alpha_scalar[0] (L1: the activation scale) or alpha_e2[e] (L2:
  // c_input_scales) when those are set
  const float* alpha;
  const float* alpha_scalar;
  const float* alpha_e2;
  const uint16_t* x_row_scale;   // NVFP4 L1: BF16 per-token rowwise scales of x, or null
  const float* c_in;    // c_input_scales (L1 re-quant)
  // L1 output: the re-quantised intermediate, expert order
  uint8_t* h_out;
  int h_row_bytes;
  uint8_t* h_sf;        // NVFP4 / MXFP8 scale tiles [P/128][I/64 | I/128]
  int h_sf_kc;
  float* h_scale_t;     // FP8 scales transposed [I/128][h_scale_ld]
  int h_scale_ld;
  // L2 output
  float* out;           // accumulate: [M][H]; staged: [R][H]
  int* status;
  // small-M gate_up reading the routed rows in place (no gather): token rows
  // of x, row_bytes each, and FP8 activation scales [M][x_sc_ld]
  const uint8_t* x_rows;
  int x_row_bytes;
  const float* x_sc;
  int x_sc_ld;
  // ... and (NVFP4, MXFP8) the byte scales of x, [M][x_sf_ld]
  const uint8_t* x_sf_rows;
  int x_sf_ld;
};

struct TileInfo {
  int e;       // expert
  int row0;    // first routed row (expert order)
  int rows;    // valid rows in this tile (1..128)
  int srow0;   // first padded scale row
  int n_tile;
};

// Tile T -> (expert, m tile, n tile).  The n tiles are taken in groups of
// n_group; inside a group the order is expert-major with m fastest, so
// concurrently running CTAs share one expert's activation panel and weight
// tiles.  One group of all n tiles is plain expert-major order (gate_up).
// The down leg adds into the FP32 accumulator: with n_group small the CTAs
// work on an accumulator slice of n_group*256 columns of every token at a
// time, which stays in L2, at the price of reading the intermediate once per
// group.

// Search key of tile T inside its group, the group's width `scale` (the
// multiplier of tile_offsets) and its first n tile.
__device__ __forceinline__ int tile_key(const GemmArgs& p, int na, int T, int& scale, int& nbase) {
  const int G = p.n_group;
  if (G >= p.n_tiles) {
    scale = p.n_tiles;
    nbase = 0;
    return T;
  }
  const int per_group = __ldg(p.tile_offsets + na) * G;
  const int gi = T / per_group;
  nbase = gi * G;
  scale = min(G, p.n_tiles - nbase);
  return T - gi * per_group;
}

// The rest of the decode once the active-expert slot `lo` of the key is known
// (tile_offsets[lo]*scale <= g < tile_offsets[lo+1]*scale).
__device__ __forceinline__ void tile_finish(const GemmArgs& p, int lo, int g, int scale, int nbase, TileInfo& t) {
  const int mt0 = __ldg(p.tile_offsets + lo);
  const int nm = __ldg(p.tile_offsets + lo + 1) - mt0;
  const int local = g - mt0 * scale;
  const int n_in = local / nm;
  const int mt = local - n_in * nm;
  t.n_tile = nbase + n_in;
  t.e = __ldg(p.expert_ids + lo);
  const int start = __ldg(p.starts + t.e);
  const int cnt = __ldg(p.starts + t.e + 1) - start;
  t.row0 = start + mt * p.tile_rows;
  t.rows = min(p.tile_rows, cnt - mt * p.tile_rows);
  t.srow0 = __ldg(p.a_scale_offsets + t.e) + mt * p.tile_rows;
}

// Tile T -> (expert, m tile, n tile) by one thread: binary search over the
// active experts' tile offsets.
__device__ __forceinline__ void decode_tile(const GemmArgs& p, int na, int T, TileInfo& t) {
  int scale, nbase;
  const int g = tile_key(p, na, T, scale, nbase);
  int lo = 0, hi = na;  // tile_offsets[lo]*scale <= g < tile_offsets[hi]*scale
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.tile_offsets + mid) * scale <= g) lo = mid; else hi = mid;
  }
  tile_finish(p, lo, g, scale, nbase, t);
}

// The same decode by a whole converged warp: each round probes 32 evenly
// spaced offsets at once and keeps the bucket the key falls in, so up to
// 1024 active experts take two dependent loads instead of ten.
__device__ __forceinline__ void decode_tile_warp(const GemmArgs& p, int na, int T, TileInfo& t, int lane) {
  int scale, nbase;
  const int g = tile_key(p, na, T, scale, nbase);
  int base = 0, len = na;  // the slot lies in [base, base + len); offsets[base]*scale <= g
  while (len > 1) {
    const int step = (len + 31) >> 5;
    const bool le = lane * step < len && __ldg(p.tile_offsets + base + lane * step) * scale <= g;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, le);
    const int j = 31 - __clz(m);
    base += j * step;
    len = min(step, len - j * step);
  }
  tile_finish(p, base, g, scale, nbase, t);
}

// A wait used while tearing down after an abort: ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// The L1 activation of gate g and up u with clamp c, slope a and up bias b:
// min(g,c) * sigmoid(a*min(g,c)) * (clamp(u,-c,c) + b).  a = 1, b = 0 is the
// clamped SwiGLU (both exact no-ops); b = 1 with the caller's slope is the
// clamped "swigluoai" of Struct_mega_ffn_ep_combine_send clamp_activation.
template <bool FAST>
__device__ __forceinline__ float l1_act(float g, float u, float c, float a, float b) {
  const float gc = fminf(g, c);
  const float uc = fminf(fmaxf(u, -c), c);
  const float z = __fmul_rn(a, gc);
  const float s = FAST ? __fdividef(gc, 1.0f + __expf(-z)) : __fdiv_rn(gc, 1.0f + expf(-z));
  return __fmul_rn(s, __fadd_rn(uc, b));
}

// h[i] = the activation of (gate acc[i], up acc[64 + i]), i < 64.  The
// precision switch is taken once, outside the unrolled loop, so only one of
// the two sequences runs.
__device__ __forceinline__ void swiglu_row(const float (&acc)[128], float (&h)[64], const GemmArgs& p) {
  if (p.fast_math) {
#pragma unroll
    for (int i = 0; i < 64; ++i) h[i] = l1_act<true>(acc[i], acc[64 + i], p.clamp, p.act_a, p.act_b);
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) h[i] = l1_act<false>(acc[i], acc[64 + i], p.clamp, p.act_a, p.act_b);
  }
}

// Byte offset of (padded row pr, scale column j) inside the 512-byte scale
// tiles [pr/128][j/4]: 32 rows x 16 bytes, row pr%32, 4-byte group
// (pr%128)/32, byte j%4.
__device__ __forceinline__ size_t sf_tile_offset(int pr, int j, int kc) {
  return (static_cast<size_t>(pr >> 7) * kc + (j >> 2)) * kSFTile + (pr & 31) * 16 +
         ((pr >> 5) & 3) * 4 + (j & 3);
}

// Packed FP32 pair FMA: (d0, d1) += (a0, a1) * (b0, b1).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, c;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%0, %1};\n\tfma.rn.f32x2 c, a, b, c;\n\tmov.b64 {%0, %1}, c;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// One GEMM over all its tiles by the calling CTA (tiles cta, cta + ncta, ...).
// `smem` is this phase's 1024-byte-aligned shared memory (kPhaseBytes),
// `tmem` a 512-column TMEM allocation, `abort_flag` the CTA's abort flag.
// Ends with a block-wide barrier; no copy or MMA of the phase is in flight
// when it returns.
template <int FMT, int EPI>
__device__ __forceinline__ void gemm_phase(const GemmArgs& p, const CUtensorMap* tmA, uint8_t* smem,
                                           uint32_t tmem, volatile int* abort_flag, int cta, int ncta) {
  using Cfg = GemmCfg<FMT, EPI>;
  constexpr int S = Cfg::kStages;
  constexpr int NACC = Cfg::kAccBufs;
  constexpr int SB = Cfg::kStageBytes;
  constexpr int BB = b_block_bytes(FMT);

  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * SB);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* final_bar = acc_empty + NACC;
  uint64_t* xbar = final_bar + 1;  // FP8 L1: one per TMEM lane quarter
  uint64_t* sf_full = xbar + 4;    // NVFP4 / MXFP8: scale buffer s holds stage s's scales
  uint64_t* sf_final = sf_full + 4;   // NVFP4 / MXFP8: the copier's last copies completed
  uint64_t* hbar = sf_final + 1;      // FP8 L1: one per TMEM lane quarter (h rows staged)
  float* xbuf = reinterpret_cast<float*>(smem + S * SB + 1024);  // FP8 L1: [2][2][128] amax
  float* xpose = reinterpret_cast<float*>(smem + S * SB + Cfg::kBarrierBytes);  // L2: per-warp 32 x 32

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(final_bar, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 64);
    for (int i = 0; i < S; ++i) mbar_init(&sf_full[i], 1);
    mbar_init(sf_final, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&hbar[i], 64);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(tmA);
  __syncthreads();

  const int na = *p.num_active;
  const int total = (na > 0) ? __ldg(p.tile_offsets + na) * p.n_tiles : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int T = cta; T < total; T += ncta) {
        TileInfo t;
        decode_tile(p, na, T, t);
        const uint8_t* wb =
            p.wB + (static_cast<size_t>(t.e) * p.n_tiles + t.n_tile) * p.k_stages * BB;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, 1)) goto producer_done;
          uint8_t* sa = smem + stage * SB;
          uint8_t* sbp = sa + kAStage;
          mbar_arrive_expect_tx(&full[stage], Cfg::kStageLoadBytes);
          tma_load_2d(sa, tmA, &full[stage], ks * kBK, t.row0);
          bulk_load(sbp, wb + static_cast<size_t>(ks) * BB, BB, &full[stage]);
          if (FMT == FMT_NVFP4) {
            bulk_load(sbp + BB,
                      p.sfa + (static_cast<size_t>(t.srow0 >> 7) * p.sfa_kc + ks * 4) * kSFTile,
                      kSFAStage, &full[stage]);
          } else if (FMT == FMT_MXFP8) {
            bulk_load(sbp + BB, p.sfa + (static_cast<size_t>(t.srow0 >> 7) * p.sfa_kc + ks) * kSFTile,
                      kMxSFAStage, &full[stage]);
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
      constexpr uint32_t kIdesc = (FMT == FMT_BF16)    ? idesc_dense(1, 1, kBN)
                                  : (FMT == FMT_FP8 || FMT == FMT_FP8T) ? idesc_dense(0, 0, kBN)
                                  : (FMT == FMT_NVFP4) ? idesc_nvf4(kBN)
                                                       : idesc_mxf8(kBN, 0);
      int stage = 0;
      uint32_t phase = 0;
      int ab = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int T = cta; T < total && ok; T += ncta) {
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
          const uint32_t sfa_t = tmem + kSFCol0 + kSFBufCols * stage;
          if (hw_scaled(FMT)) {
            if (!mbar_wait(&sf_full[stage], phase, abort_flag, p.status, 8)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            const uint32_t acc = (FMT == FMT_FP8) ? (kc > 0) : ((ks | kc) != 0);
            const uint64_t a = adesc + static_cast<uint64_t>(2 * kc);
            const uint64_t b = bdesc + static_cast<uint64_t>(2 * kc);
            if (FMT == FMT_BF16) mma_f16(d, a, b, kIdesc, acc);
            else if (FMT == FMT_FP8 || FMT == FMT_FP8T) mma_f8(d, a, b, kIdesc, acc);
            else if (FMT == FMT_NVFP4) mma_nvf4(d, a, b, kIdesc, sfa_t + 4 * kc, sfa_t + kSFBOff + 8 * kc, acc);
            // one UE8M0 scale per 32-wide K step: byte kc of the stage's scale words
            else mma_mxf8(d, a, b, idesc_mxf8(kBN, kc), sfa_t, sfa_t + kSFBOff, acc);
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
  } else if (hw_scaled(FMT) && warp == 2) {
    // ------------------------------------------------------------ scale copier
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int T = cta; T < total; T += ncta) {
        bool ok = true;
        for (int ks = 0; ks < p.k_stages; ++ks) {
          // The stage's data has landed, so the MMAs that last read its scale
          // buffer (the stage's previous use) have completed: the producer
          // refilled the stage only after they released it.
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, 9)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfb_s = smem_u32(smem + stage * SB + kAStage + kBStage);
          const uint32_t dst = tmem + kSFCol0 + kSFBufCols * stage;
          if (FMT == FMT_NVFP4) {
            const uint32_t sfa_s = sfb_s + kSFBStage;
#pragma unroll
            for (int kc = 0; kc < 4; ++kc) {
              tmem_copy_sf(dst + 4 * kc, sdesc_sf_tile(sfa_s + kc * kSFTile));
              tmem_copy_sf(dst + kSFBOff + 8 * kc, sdesc_sf_tile(sfb_s + kc * kSFTile));
              tmem_copy_sf(dst + kSFBOff + 8 * kc + 4, sdesc_sf_tile(sfb_s + 4 * kSFTile + kc * kSFTile));
            }
          } else {
            // MXFP8: one tile per 128 rows covers the stage's four K steps
            tmem_copy_sf(dst, sdesc_sf_tile(sfb_s + kMxSFBStage));
            tmem_copy_sf(dst + kSFBOff, sdesc_sf_tile(sfb_s));
            tmem_copy_sf(dst + kSFBOff + 4, sdesc_sf_tile(sfb_s + kSFTile));
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
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int half = ew >> 2;             // 128-column half of the accumulator
    const int row_local = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int ab = 0;
    uint32_t aphase = 0;
    int xpar = 0;          // FP8 L1: amax exchange buffer / barrier phase
    for (int T = cta; T < total; T += ncta) {
      TileInfo t;
      decode_tile_warp(p, na, T, t, lane);
      const bool valid = row_local < t.rows;
      const int r = t.row0 + row_local;
      const int pr = t.srow0 + row_local;
      // Down leg: the row's flat slot is loaded now and its router weight
      // once the first partial has been taken, so neither load's latency
      // falls on the epilogue's tail (and, likewise, the NVFP4 gate_up's
      // per-token rowwise scale of x).
      const bool gather_wgt = EPI == EPI_L2_ACC && valid;
      const bool row_scaled = EPI == EPI_L1 && FMT == FMT_NVFP4 && p.x_row_scale != nullptr;
      const int s_flat = (gather_wgt || (row_scaled && valid)) ? __ldg(p.src_info + r) : 0;
      float wgt = 1.0f;

      // acc[0..127]: this thread's row, columns 128*half .. 128*half+127 of
      // the tile (L1: 64 gate then 64 up; L2: output columns)
      float acc[128];
      if constexpr (FMT == FMT_FP8) {
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
        const float* sbe = p.sb + static_cast<size_t>(t.e) * p.sb_nb * p.sb_kb;
        int nb_lo, nb_hi;  // weight blocks of acc[0..63] and acc[64..127]
        if (EPI == EPI_L1) {
          nb_lo = t.n_tile;
          nb_hi = (p.I >> 7) + t.n_tile;
        } else {
          nb_lo = nb_hi = (t.n_tile * kBN + half * 128) >> 7;
        }
        bool ok = true;
        // The activation scale of K block ks+1 (a per-row load from L2) is
        // issued before block ks is waited for, taking its latency off the
        // per-block critical path; the weight scales are warp-uniform L1 hits.
        const float* sa_col = p.sa_t + pr;
        float nx_sa = sa_col[0];
        for (int ks = 0; ks < p.k_stages; ++ks) {
          const float sa = nx_sa;
          if (ks + 1 < p.k_stages) nx_sa = sa_col[static_cast<size_t>(ks + 1) * p.sa_ld];
          if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 5)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float s_lo = sa * __ldg(sbe + nb_lo * p.sb_kb + ks);
          const float s_hi = sa * __ldg(sbe + nb_hi * p.sb_kb + ks);
          const uint32_t base = tmem + ab * kBN + half * 128 + lane_off;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float v[16];
            __syncwarp();
            tmem_ld16(base + 16 * c, v);
            const float s = (c < 4) ? s_lo : s_hi;
#pragma unroll
            for (int i = 0; i < 8; ++i) ffma2(acc[16 * c + 2 * i], acc[16 * c + 2 * i + 1], v[2 * i], v[2 * i + 1], s, s);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          if (++ab == NACC) {
            ab = 0;
            aphase ^= 1u;
          }
          if (ks == 0 && gather_wgt) wgt = __ldg(p.topk_weights + s_flat);
        }
        if (!ok) break;
      } else {
        // BF16 / NVFP4 / MXFP8 / FP8T: the whole K sum is in TMEM; read it, release it.
        if (!mbar_wait(&acc_full[ab], aphase, abort_flag, p.status, 6)) break;
        tc_fence_after();
        if (gather_wgt) wgt = __ldg(p.topk_weights + s_flat);
        const uint32_t base = tmem + ab * kBN + half * 128 + lane_off;
        {
          // all 128 columns in one TMEM round trip
          uint32_t r0[32], r1[32], r2[32], r3[32];
          __syncwarp();
          tmem_ld32_async(base, r0);
          tmem_ld32_async(base + 32, r1);
          tmem_ld32_async(base + 64, r2);
          tmem_ld32_async(base + 96, r3);
          tmem_wait_ld(r0);
          tmem_wait_ld(r1);
          tmem_wait_ld(r2);
          tmem_wait_ld(r3);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            acc[i] = __uint_as_float(r0[i]);
            acc[32 + i] = __uint_as_float(r1[i]);
            acc[64 + i] = __uint_as_float(r2[i]);
            acc[96 + i] = __uint_as_float(r3[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (++ab == NACC) {
          ab = 0;
          aphase ^= 1u;
        }
        if (FMT == FMT_FP8T) {
          // (activation scale x weight scale) or (re-quant scale x weight scale)
          float alpha = __ldg(p.alpha + t.e);
          if (p.alpha_scalar) alpha = __fmul_rn(__ldg(p.alpha_scalar), alpha);
          if (p.alpha_e2) alpha = __fmul_rn(__ldg(p.alpha_e2 + t.e), alpha);
#pragma unroll
          for (int i = 0; i < 128; ++i) acc[i] = __fmul_rn(acc[i], alpha);
        }
        if (FMT == FMT_NVFP4) {
          float alpha = __ldg(p.alpha + t.e);
          if (row_scaled && valid)
            alpha = __fmul_rn(alpha, __uint_as_float(static_cast<uint32_t>(__ldg(p.x_row_scale + s_flat / p.topk)) << 16));
#pragma unroll
          for (int i = 0; i < 128; ++i) acc[i] = __fmul_rn(acc[i], alpha);
        }
      }

      if (EPI == EPI_L1) {
        // h for intermediate columns j0 + 64*half + i, i < 64
        const int hcol0 = t.n_tile * 128 + half * 64;
        float h[64];
        swiglu_row(acc, h, p);
        uint8_t* hrow = p.h_out + static_cast<size_t>(r) * p.h_row_bytes;
        if constexpr (FMT == FMT_FP8) {
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(h[i]));
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
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[4 * i], inv), __fmul_rn(h[4 * i + 1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(h[4 * i + 2], inv), __fmul_rn(h[4 * i + 3], inv));
            w[i] = (s != 0.0f) ? (lo | (hi << 16)) : 0u;
          }
          // this thread's 64 bytes into the quarter's staging rows; once both
          // warps of the quarter are in, each stores 16 whole rows (8 lanes
          // x 16 bytes per row, 4 rows per instruction)
          uint8_t* stg = reinterpret_cast<uint8_t*>(xpose) + q * (32 * Cfg::kHStageStride);
          uint4* srow = reinterpret_cast<uint4*>(stg + lane * Cfg::kHStageStride + half * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) srow[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          if (valid && half == 0) p.h_scale_t[static_cast<size_t>(t.n_tile) * p.h_scale_ld + pr] = s;
          mbar_arrive(&hbar[q]);
          if (!mbar_wait(&hbar[q], static_cast<uint32_t>(xpar ^ 1), abort_flag, p.status, 11)) break;
          const int rows_here = t.rows - q * 32;
          uint8_t* hbase = p.h_out + static_cast<size_t>(t.row0 + q * 32) * p.h_row_bytes + t.n_tile * 128;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int row = half * 16 + it * 4 + (lane >> 3);
            const int c16 = lane & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(stg + row * Cfg::kHStageStride + c16 * 16);
            if (row < rows_here)
              *reinterpret_cast<uint4*>(hbase + static_cast<size_t>(row) * p.h_row_bytes + c16 * 16) = v;
          }
        } else if constexpr (FMT == FMT_FP8T) {
          // one static scale per expert: codes e4m3(h * (1 / G)), saturating
          const float inv = __frcp_rn(__ldg(p.c_in + t.e));
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[4 * i], inv), __fmul_rn(h[4 * i + 1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(h[4 * i + 2], inv), __fmul_rn(h[4 * i + 3], inv));
            w[i] = lo | (hi << 16);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + hcol0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        } else if constexpr (FMT == FMT_MXFP8) {
          // two 32-column blocks: scale 2^X, X = floor(log2 amax) - 8 clamped
          // to [-127, 127] (read off amax's exponent field; a zero or
          // subnormal amax gives -127), codes e4m3(h * 2^-X) saturating --
          // the scaling by a power of two is exact
          uint32_t w[16];
          uint32_t sfw = 0;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(h[32 * b + j]));
            const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
            const int X = ex == 0 ? -127 : max(ex - 135, -127);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);   // 2^-X
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t lo = cvt_e4m3x2(__fmul_rn(h[32 * b + 4 * i], inv), __fmul_rn(h[32 * b + 4 * i + 1], inv));
              const uint32_t hi =
                  cvt_e4m3x2(__fmul_rn(h[32 * b + 4 * i + 2], inv), __fmul_rn(h[32 * b + 4 * i + 3], inv));
              w[8 * b + i] = lo | (hi << 16);
            }
            sfw |= static_cast<uint32_t>(X + 127) << (8 * b);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + hcol0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            // scale columns hcol0/32 and hcol0/32 + 1 (even) share a 4-byte group
            *reinterpret_cast<uint16_t*>(p.h_sf + sf_tile_offset(pr, hcol0 >> 5, p.h_sf_kc)) =
                static_cast<uint16_t>(sfw);
          }
        } else if constexpr (FMT == FMT_BF16) {
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + hcol0 * 2);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_uint4(pack_bf16x2(h[8 * i], h[8 * i + 1]), pack_bf16x2(h[8 * i + 2], h[8 * i + 3]),
                                  pack_bf16x2(h[8 * i + 4], h[8 * i + 5]), pack_bf16x2(h[8 * i + 6], h[8 * i + 7]));
          }
        } else {
          const float G = __ldg(p.c_in + t.e);
          const float denom6 = __fmul_rn(6.0f, G);
          uint32_t codes[8];
          uint32_t sfw = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(h[16 * b + j]));
            const uint32_t sf_code = cvt_e4m3x2(__fdiv_rn(amax, denom6), 0.0f) & 0xFFu;
            const float sf = e4m3_to_f32(sf_code);
            uint32_t w0 = 0, w1 = 0;
            if (sf != 0.0f) {
              const float inv = __frcp_rn(__fmul_rn(sf, G));
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                w0 |= cvt_e2m1x2(__fmul_rn(h[16 * b + 2 * j], inv), __fmul_rn(h[16 * b + 2 * j + 1], inv)) << (8 * j);
                w1 |= cvt_e2m1x2(__fmul_rn(h[16 * b + 8 + 2 * j], inv), __fmul_rn(h[16 * b + 9 + 2 * j], inv))
                      << (8 * j);
              }
            }
            codes[2 * b] = w0;
            codes[2 * b + 1] = w1;
            sfw |= sf_code << (8 * b);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + hcol0 / 2);
            dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
            // the 4 scale bytes of columns hcol0/16 .. +3 are contiguous in one tile
            *reinterpret_cast<uint32_t*>(p.h_sf + sf_tile_offset(pr, hcol0 >> 4, p.h_sf_kc)) = sfw;
          }
        }
      } else if constexpr (EPI == EPI_L2_ACC && FMT == FMT_NVFP4) {
        // L2, accumulate (NVFP4): each thread's router-weighted row segment goes
        // through its own 128-byte shared-memory slot into asynchronous bulk
        // reduce-adds (32 columns each) on the token's FP32 accumulator row;
        // the warp moves on to the next tile while the TMA engine finishes
        // the reductions.
        const int n0 = t.n_tile * kBN + half * 128;
        const int tok = gather_wgt ? s_flat / p.topk : r;
        float* slot = xpose + (ew * 32 + lane) * Cfg::kXposeStride;
        float* grow = p.out + static_cast<size_t>(tok) * p.H + n0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          bulk_wait_read();   // the slot's previous contents have been read
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(slot)[i] =
                make_float4(acc[32 * c + 4 * i] * wgt, acc[32 * c + 4 * i + 1] * wgt,
                            acc[32 * c + 4 * i + 2] * wgt, acc[32 * c + 4 * i + 3] * wgt);
          fence_async_smem();
          if (valid) {
            bulk_reduce_add_f32(grow + 32 * c, slot, 128);
            bulk_commit();
          }
        }
      } else {
        // L2, staged or accumulate: write the rows through a per-warp 32 x 32
        // transpose so that one warp instruction covers four whole 128-byte
        // row segments (8 lanes per row) instead of 32 scattered 16-byte
        // pieces; accumulate mode adds them with float4 atomics.
        const int n0 = t.n_tile * kBN + half * 128;
        const int tok = gather_wgt ? s_flat / p.topk : r;
        float* xb = xpose + ew * (32 * Cfg::kXposeStride);
        const int rows_here = t.rows - q * 32;   // valid rows of this warp's quarter
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float4* wrow = reinterpret_cast<float4*>(xb + lane * Cfg::kXposeStride);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            wrow[i] = make_float4(acc[32 * c + 4 * i], acc[32 * c + 4 * i + 1], acc[32 * c + 4 * i + 2],
                                  acc[32 * c + 4 * i + 3]);
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int row = it * 4 + (lane >> 3);
            const int c4 = lane & 7;
            const int rtok = __shfl_sync(0xFFFFFFFFu, tok, row);
            const float rw = __shfl_sync(0xFFFFFFFFu, wgt, row);
            const float4 v = *reinterpret_cast<const float4*>(xb + row * Cfg::kXposeStride + 4 * c4);
            if (row < rows_here) {
              float4* dst = reinterpret_cast<float4*>(p.out + static_cast<size_t>(rtok) * p.H + n0 + 32 * c) + c4;
              if (EPI == EPI_L2_ACC) atomicAdd(dst, make_float4(v.x * rw, v.y * rw, v.z * rw, v.w * rw));
              else *dst = v;
            }
          }
          __syncwarp();
        }
      }
    }
    // every bulk reduction of this thread has landed before the phase ends
    if (EPI == EPI_L2_ACC && FMT == FMT_NVFP4) bulk_wait_done();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// Shared-memory header of every kernel that runs GEMM phases: the TMEM
// address, the CTA's abort flag and, in the word after it, the bounded
// waits' limit in microseconds (0: the default; mbar_wait reads it there).
struct SmemHeader {
  uint32_t tmem;
  int abort;
  int wait_us;
};

__device__ __forceinline__ uint8_t* smem_base_1024() {
  extern __shared__ uint8_t smem_raw[];
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

template <int FMT, int EPI>
__global__ void __launch_bounds__(GemmCfg<FMT, EPI>::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmArgs p, const __grid_constant__ CUtensorMap tmA) {
  uint8_t* base = smem_base_1024();
  SmemHeader* hdr = reinterpret_cast<SmemHeader*>(base);
  if (threadIdx.x == 0) hdr->abort = 0;
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&hdr->tmem, kTmemCols);
  pdl_trigger();
  pdl_wait();   // the layout, activations, accumulator and header come from earlier kernels
  if (threadIdx.x == 0) hdr->wait_us = wait_limit_us(p.status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hdr->tmem;
  gemm_phase<FMT, EPI>(p, &tmA, base + GemmCfg<FMT, EPI>::kHeaderBytes, tmem, &hdr->abort, blockIdx.x,
                       gridDim.x);
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Weight preparation: logical K-major weights [E][N][Kb] (+ NVFP4 scales
// [E][N][K/16], MXFP8 scales [E][N][K/32]) -> blocks [E][n_tiles][k_stages]
// of b_block_bytes(fmt).  One thread per 16-byte chunk of block data; the
// scale tiles follow.
// ---------------------------------------------------------------------------
struct PrepArgs {
  const uint8_t* w;        // logical weights
  const uint8_t* sf;       // NVFP4 / MXFP8 logical scales, else null
  uint8_t* out;
  int E, N, Kb;            // experts, rows per expert, bytes per row
  int ksf;                 // scale columns per row (NVFP4 K/16, MXFP8 K/32)
  int n_tiles, k_stages;
  int l1;                  // 1: gate/up interleaved L1 tiles (N = 2I)
  int fmt;
};

__device__ __forceinline__ int prep_row(const PrepArgs& a, int nt, int r) {
  return a.l1 ? l1_tile_row(nt, r, a.N / 2, l1_group(a.fmt)) : nt * kBN + r;
}

__global__ void __launch_bounds__(256) prepare_weights_kernel(PrepArgs a) {
  pdl_trigger();
  pdl_wait();
  const int bb = b_block_bytes(a.fmt);
  const int64_t blocks = static_cast<int64_t>(a.E) * a.n_tiles * a.k_stages;
  const int64_t n16 = blocks * (kBStage / 16);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = i / (kBStage / 16);
    const int within = static_cast<int>(i - blk * (kBStage / 16));
    const int r = within >> 3, cpos = within & 7;
    const int ks = static_cast<int>(blk % a.k_stages);
    const int64_t et = blk / a.k_stages;
    const int nt = static_cast<int>(et % a.n_tiles);
    const int e = static_cast<int>(et / a.n_tiles);
    const int row = prep_row(a, nt, r);
    const int c = cpos ^ (r & 7);
    const uint4* src = reinterpret_cast<const uint4*>(
        a.w + (static_cast<size_t>(e) * a.N + row) * a.Kb + static_cast<size_t>(ks) * kBK + 16 * c);
    *reinterpret_cast<uint4*>(a.out + blk * bb + within * 16) = *src;
  }
  if (!hw_scaled(a.fmt)) return;
  // per row block: NVFP4 four tiles (K steps kc), MXFP8 one
  const int tiles_per_rb = a.fmt == FMT_NVFP4 ? 4 : 1;
  const int sf_block = bb - kBStage;
  const int64_t nsf = blocks * sf_block;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nsf;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = i / sf_block;
    const int o = static_cast<int>(i - blk * sf_block);
    const int rb = o / (tiles_per_rb * kSFTile), kc = (o / kSFTile) % tiles_per_rb, b = o & (kSFTile - 1);
    const int ks = static_cast<int>(blk % a.k_stages);
    const int64_t et = blk / a.k_stages;
    const int nt = static_cast<int>(et % a.n_tiles);
    const int e = static_cast<int>(et / a.n_tiles);
    const int tile_row = 128 * rb + ((b & 15) >> 2) * 32 + (b >> 4);
    const int row = prep_row(a, nt, tile_row);
    const int col = ks * 4 * tiles_per_rb + kc * 4 + (b & 3);
    a.out[blk * bb + kBStage + o] = a.sf[(static_cast<size_t>(e) * a.N + row) * a.ksf + col];
  }
}

}  // namespace moe

// aux_kernels.cuh -- the memory-bound steps around the expert GEMMs:
// routing from logits, the counting-sort permutation, the activation gather
// into expert order, accumulator zeroing, the BF16 finalise and the staged
// (deterministic) combine.
//
// Each step is a __device__ function over a "virtual block" (an index and the
// calling block's threads), wrapped by a small __global__ kernel; the
// single-launch fused kernel calls the same functions between grid barriers.
#pragma once

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Routing (flashinfer.fused_moe.MoEActivationPack, routing_input_mode
// FromLogits): one warp per token.  Each lane holds up to PER experts as
// 64-bit keys (order-preserving bits of score = logit + bias, then the
// complemented expert id), so one warp max picks the highest score with the
// lower id on ties; NaN scores map to the smallest key.  The weights are the
// softmax of the unbiased logits over the chosen k.
// ---------------------------------------------------------------------------
struct RouteArgs {
  const float* logits;   // [M][E]
  const float* bias;     // [E] or null
  int64_t M;
  int E, k;
  int64_t* idx_out;      // [M][out_k]
  float* w_out;          // [M][out_k]
  int out_k;             // k, or k + 1 with a shared expert
  int shared;            // 1: column k is the shared expert (index E, weight 1)
};

__device__ __forceinline__ uint64_t route_key(float s, int e) {
  if (s == 0.0f) s = 0.0f;  // -0 and +0 are the same score
  const uint32_t b = __float_as_uint(s);
  const uint32_t ord = (s != s) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
  return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - e);
}

// Routes token t with the calling (full) warp, from its logits already in
// registers (lane l holds experts l, l+32, ...) and the bias of those experts.
template <int PER>
__device__ __forceinline__ void route_token(const RouteArgs& a, int64_t t, const float (&lg)[PER],
                                            const float (&bias)[PER], int lane) {
  uint64_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < a.E) key[i] = route_key(__fadd_rn(lg[i], bias[i]), e);
  }
  int my_e = 0;
  for (int j = 0; j < a.k; ++j) {
    uint64_t best = 0;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (key[i] > best) {
        best = key[i];
        bi = i;
      }
    uint64_t m = best;
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, m, off);
      m = (o > m) ? o : m;
    }
    const int e = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(m));
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (i == bi && best == m) key[i] = 0;
    if (lane == j) my_e = e;
  }
  // the unbiased logit of this lane's chosen expert, from the lane that holds it
  const bool mine = lane < a.k;
  float l = -INFINITY;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float v = __shfl_sync(0xFFFFFFFFu, lg[i], my_e & 31);
    if (mine && (my_e >> 5) == i) l = v;
  }
  float mx = l;
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  const float ex = mine ? expf(l - mx) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
  if (mine) {
    a.idx_out[t * a.out_k + lane] = my_e;
    a.w_out[t * a.out_k + lane] = __fdiv_rn(ex, sum);
  }
  if (a.shared && lane == 0) {
    a.idx_out[t * a.out_k + a.k] = a.E;
    a.w_out[t * a.out_k + a.k] = 1.0f;
  }
}

// Tokens warp_id, warp_id + nwarps, ... (all lanes of the calling warp),
// with the logits of B tokens loaded before any of them is routed, so their
// memory latencies overlap.
template <int PER>
__device__ __forceinline__ void route_tokens_per(const RouteArgs& a, int64_t warp_id, int64_t nwarps, int lane) {
  constexpr int B = PER <= 4 ? 4 : (PER <= 8 ? 2 : 1);
  float bias[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    bias[i] = (a.bias && e < a.E) ? a.bias[e] : 0.0f;
  }
  for (int64_t t0 = warp_id; t0 < a.M; t0 += nwarps * B) {
    float lg[B][PER];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int64_t t = t0 + b * nwarps;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        lg[b][i] = (t < a.M && e < a.E) ? a.logits[t * a.E + e] : 0.0f;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int64_t t = t0 + b * nwarps;
      if (t < a.M) route_token<PER>(a, t, lg[b], bias, lane);
    }
  }
}

// Experts per lane (32-expert groups) of a routing problem.
__host__ __device__ inline int route_per(int E) {
  const int per = (E + 31) / 32;
  return per <= 1 ? 1 : per <= 2 ? 2 : per <= 4 ? 4 : per <= 8 ? 8 : per <= 16 ? 16 : 32;
}

__device__ __forceinline__ void route_tokens(const RouteArgs& a, int64_t warp_id, int64_t nwarps, int lane) {
  switch (route_per(a.E)) {
    case 1: route_tokens_per<1>(a, warp_id, nwarps, lane); break;
    case 2: route_tokens_per<2>(a, warp_id, nwarps, lane); break;
    case 4: route_tokens_per<4>(a, warp_id, nwarps, lane); break;
    case 8: route_tokens_per<8>(a, warp_id, nwarps, lane); break;
    case 16: route_tokens_per<16>(a, warp_id, nwarps, lane); break;
    default: route_tokens_per<32>(a, warp_id, nwarps, lane); break;
  }
}

// One kernel per expert-group count, so the register allocation (and the
// occupancy) is that of the problem's own width.
template <int PER>
__global__ void __launch_bounds__(256) route_kernel(RouteArgs a) {
  pdl_trigger();
  pdl_wait();
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  route_tokens_per<PER>(a, (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5, nw,
                        threadIdx.x & 31);
}

// ---------------------------------------------------------------------------
// Per-token dynamic NVFP4 quantisation of BF16 activations (EPConfig,
// nvfp4_dyn_global_scales): one warp per token; lane l owns the 16-value
// blocks l, l+32, ...  Pass 1 finds the token's largest magnitude, pass 2
// re-reads each block and quantises it against G = rowmax / 2688 with the
// same FP32 steps as the intermediate's NVFP4 re-quant.
// ---------------------------------------------------------------------------
struct QuantRowArgs {
  const uint16_t* x;     // BF16 [M][H]
  int64_t M;
  int H;
  uint8_t* codes;        // [M][H/2]
  uint8_t* scales;       // E4M3 [M][H/16]
  uint16_t* rowwise;     // BF16 [M]
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__global__ void __launch_bounds__(256) quantize_rowwise_kernel(QuantRowArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int nblk = a.H / 16;
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < a.M; t += nw) {
    const uint4* row = reinterpret_cast<const uint4*>(a.x + t * a.H);
    float rowmax = 0.0f;
    for (int b = lane; b < nblk; b += 32) {
      const uint4 u0 = __ldg(row + 2 * b), u1 = __ldg(row + 2 * b + 1);
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        rowmax = fmaxf(rowmax, fmaxf(fabsf(bf16_bits_to_f32(w[i] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[i] >> 16))));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(0xFFFFFFFFu, rowmax, off));
    const float G = __fdiv_rn(rowmax, 2688.0f);
    const float denom6 = __fmul_rn(6.0f, G);
    uint32_t* crow = reinterpret_cast<uint32_t*>(a.codes + t * (a.H / 2));
    for (int b = lane; b < nblk; b += 32) {
      const uint4 u0 = __ldg(row + 2 * b), u1 = __ldg(row + 2 * b + 1);
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float v[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
      }
      uint32_t c0 = 0, c1 = 0, sf_code = 0;
      if (rowmax > 0.0f) {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        sf_code = cvt_e4m3x2(__fdiv_rn(amax, denom6), 0.0f) & 0xFFu;
        const float sf = e4m3_to_f32(sf_code);
        if (sf != 0.0f) {
          const float inv = __frcp_rn(__fmul_rn(sf, G));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            c0 |= cvt_e2m1x2(__fmul_rn(v[2 * j], inv), __fmul_rn(v[2 * j + 1], inv)) << (8 * j);
            c1 |= cvt_e2m1x2(__fmul_rn(v[8 + 2 * j], inv), __fmul_rn(v[9 + 2 * j], inv)) << (8 * j);
          }
        }
      }
      crow[2 * b] = c0;
      crow[2 * b + 1] = c1;
      a.scales[t * nblk + b] = static_cast<uint8_t>(sf_code);
    }
    if (lane == 0) a.rowwise[t] = rowmax > 0.0f ? static_cast<uint16_t>(pack_bf16x2(G, 0.0f) & 0xFFFFu) : 0;
  }
}

// ---------------------------------------------------------------------------
// Permutation (Struct_mega_ffn_ep_combine_send: expert_start_indices,
// expert_ids, a_scale_offsets, src_info, num_active_experts): a stable
// counting sort of the flat slots s = t*k + j by expert.
//   small problems: one block; warp w owns a contiguous run of slots and
//           counts it into its own histogram row; the rows' prefix sums in
//           (expert, warp) order give every warp its first row per expert,
//           and a second ordered pass over each run writes the rows.
//   large problems, pass 1: per 1024-slot chunk, count slots per expert.
//   large problems, pass 2: per chunk, the expert totals and this chunk's
//           offset within each expert give every slot its row; one warp walks
//           the chunk in order, ranking equal experts inside each 32-slot
//           round with __match_any_sync, so rows ascend in slot index.
// Chunk 0 (or the one block) also writes the per-expert arrays and the GEMM
// tile table.
// ---------------------------------------------------------------------------
constexpr int kPermChunk = 1024;
constexpr int kPermSmallMax = 16384;
constexpr int kPermBatch = 8;       // rounds of 32 slots whose loads one warp issues together
constexpr int kPermSmallMaxE = 256;

struct PermOut {
  int* expert_counts;
  int* expert_start_indices;
  int* src_info;
  int* slot_to_row;
  int* expert_ids;
  int* num_active;
  int* a_scale_offsets;
  int* tile_offsets;
  int* tiles32;          // optional: the small-M GEMMs' 32-row tile table (E+1)
};

struct PermArgs {
  const int64_t* idx;    // [R]
  int64_t R;
  int E;
  int nblk;              // chunks of kPermChunk slots
  int* block_counts;     // [nblk][E]
  PermOut o;
  int* status;
};

__host__ __device__ inline bool perm_small_case(int64_t R, int E) {
  return R <= kPermSmallMax && E <= kPermSmallMaxE;
}

// Shared-memory ints of the two-pass (per chunk) and the one-block permutation.
__host__ __device__ inline int perm_chunk_smem_ints(int E) { return 3 * E + 1 + kPermChunk; }
// One-block problems with few experts whose experts x slots fit a 16 KB
// bitmap take the bitmap path (perm_bitmap_block); with many experts its
// per-expert row scans cost more than the per-warp histograms.
constexpr int kPermBitmapWords = 4096;
constexpr int kPermBitmapMaxE = 64;
__host__ __device__ inline int perm_bitmap_words(int64_t R, int E) {
  return E * static_cast<int>((R + 31) / 32);
}
__host__ __device__ inline bool perm_bitmap_case(int64_t R, int E) {
  return perm_small_case(R, E) && E <= kPermBitmapMaxE && perm_bitmap_words(R, E) <= kPermBitmapWords;
}
__host__ __device__ inline int perm_small_smem_ints(int64_t R, int E, int nwarps) {
  const int hist = nwarps * E + 2 * E + 1;
  const int bitmap = 2 * perm_bitmap_words(R, E) + 2 * E + 1;
  return perm_bitmap_case(R, E) && bitmap > hist ? bitmap : hist;
}

// Exclusive scan of v[0..n) by one warp (n <= 1024); writes out[0..n] (n+1
// entries, out[n] = total).  Each lane owns a contiguous run of entries.
// One warp turns the per-expert totals (shared memory, E entries) into
// start[0..E] (shared memory: the exclusive scan, start[E] = routed rows) and,
// when `tables` is set, the layout arrays in global memory: expert_counts,
// expert_start_indices, a_scale_offsets (scan of the counts padded to 128),
// expert_ids (active experts in order, -1 after them), num_active and
// tile_offsets (scan of the active experts' 128-row m tiles), and when asked
// the small-M GEMMs' table of 32-row tiles.  The scans run together: each
// lane takes E/32 consecutive experts, sums them, and one round of shuffles
// scans all the sums at once.
__device__ void expert_tables_warp(const int* total, int* start, int E, const PermOut& o, bool tables, int lane) {
  const int per = (E + 31) >> 5;
  const int b = min(E, lane * per), e_end = min(E, b + per);
  int c = 0, pad = 0, act = 0, mt = 0, m32 = 0;
  for (int e = b; e < e_end; ++e) {
    const int t = total[e];
    const int m = (t + 127) >> 7;
    c += t;
    pad += m << 7;
    act += t > 0 ? 1 : 0;
    mt += m;
    m32 += (t + 31) >> 5;
  }
  int ic = c, ip = pad, ia = act, im = mt, i32 = m32;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int xc = __shfl_up_sync(0xFFFFFFFFu, ic, off);
    const int xp = __shfl_up_sync(0xFFFFFFFFu, ip, off);
    const int xa = __shfl_up_sync(0xFFFFFFFFu, ia, off);
    const int xm = __shfl_up_sync(0xFFFFFFFFu, im, off);
    const int x32 = __shfl_up_sync(0xFFFFFFFFu, i32, off);
    if (lane >= off) {
      ic += xc;
      ip += xp;
      ia += xa;
      im += xm;
      i32 += x32;
    }
  }
  const int na = __shfl_sync(0xFFFFFFFFu, ia, 31);
  // exclusive bases of this lane
  int rc = ic - c, rp = ip - pad, ra = ia - act, rm = im - mt, r32 = i32 - m32;
  for (int e = b; e < e_end; ++e) {
    const int t = total[e];
    const int m = (t + 127) >> 7;
    start[e] = rc;
    if (tables) {
      o.expert_counts[e] = t;
      o.expert_start_indices[e] = rc;
      o.a_scale_offsets[e] = rp;
      if (t > 0) {
        o.expert_ids[ra] = e;
        o.tile_offsets[ra] = rm;
        if (o.tiles32) o.tiles32[ra] = r32;
      }
      if (e >= na) o.expert_ids[e] = -1;
    }
    rc += t;
    rp += m << 7;
    if (t > 0) {
      ++ra;
      rm += m;
      r32 += (t + 31) >> 5;
    }
  }
  if (lane == 31) {
    start[E] = ic;
    if (tables) {
      o.expert_start_indices[E] = ic;
      o.a_scale_offsets[E] = ip;
      *o.num_active = na;
      o.tile_offsets[na] = im;
      if (o.tiles32) o.tiles32[na] = i32;
    }
  }
}

// Pass 1 of the large case for chunk c.
__device__ void perm_count_chunk(const PermArgs& a, int c, int* sm) {
  int* cnt = sm;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(c) * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x) {
    const int64_t s = base + i;
    if (s < a.R) {
      const int64_t v = a.idx[s];
      if (v >= 0 && v < a.E) atomicAdd(&cnt[v], 1);
      else if (v != -1) record_error(a.status, MOE_ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    a.block_counts[static_cast<size_t>(c) * a.E + e] = cnt[e];
  __syncthreads();
}

// Pass 2 of the large case for chunk c.
__device__ void perm_scatter_chunk(const PermArgs& a, int c, int* sm) {
  const int E = a.E;
  int* total = sm;                 // [E]
  int* start = total + E;          // [E+1]
  int* cursor = start + E + 1;     // [E]
  int* sidx = cursor + E;          // [kPermChunk] this chunk's expert ids
  const int64_t base = static_cast<int64_t>(c) * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x) {
    const int64_t s = base + i;
    int v = -1;
    if (s < a.R) {
      const int64_t x = a.idx[s];
      v = (x >= 0 && x < E) ? static_cast<int>(x) : -1;
    }
    sidx[i] = v;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int tot = 0, before = 0;
#pragma unroll 8
    for (int b = 0; b < a.nblk; ++b) {
      const int n = __ldg(a.block_counts + static_cast<size_t>(b) * E + e);
      tot += n;
      before += (b < c) ? n : 0;
    }
    total[e] = tot;
    cursor[e] = before;
  }
  __syncthreads();
  if (threadIdx.x < 32) expert_tables_warp(total, start, E, a.o, c == 0, threadIdx.x);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] += start[e];
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const unsigned lt = (1u << lane) - 1u;
    for (int rnd = 0; rnd < kPermChunk / 32; ++rnd) {
      const int64_t s = base + rnd * 32 + lane;
      if (base + rnd * 32 >= a.R) break;
      const int v = sidx[rnd * 32 + lane];
      const bool valid = v >= 0;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? v : (E + lane));
      int row = -1;
      if (valid) {
        row = cursor[v] + __popc(peers & lt);
        a.o.src_info[row] = static_cast<int>(s);
      }
      if (s < a.R) a.o.slot_to_row[s] = row;
      __syncwarp();
      if (valid && lane == 31 - __clz(peers)) cursor[v] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
}

// The whole small case in the calling block.
// One block, bitmap form: bit s of expert e's row is set when slot s routes
// to e.  A slot's rank inside its expert (the stable order) is the prefix
// popcount of its expert's row below it: per-word prefix counts of each row,
// then one popcount of the slot's own word.  Every step is a parallel pass
// over the slots, the words or the experts.
__device__ void perm_bitmap_block(const PermArgs& a, int* sm) {
  const int E = a.E;
  const int R = static_cast<int>(a.R);
  const int W = (R + 31) >> 5;                            // words per expert row
  uint32_t* bits = reinterpret_cast<uint32_t*>(sm);        // [E][W]
  int* wpre = sm + E * W;                                  // [E][W] set bits of the row before word w
  int* total = wpre + E * W;                               // [E]
  int* start = total + E;                                  // [E+1]
  const int nthr = blockDim.x, nw = nthr >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < E * W; i += nthr) bits[i] = 0u;
  __syncthreads();
  for (int s = threadIdx.x; s < R; s += nthr) {
    const int64_t x = a.idx[s];
    if (x >= 0 && x < E) atomicOr(&bits[static_cast<int>(x) * W + (s >> 5)], 1u << (s & 31));
    else if (x != -1) record_error(a.status, MOE_ERR_BAD_INDEX);
  }
  __syncthreads();
  // per expert row: exclusive prefix of the words' popcounts, and the total
  const int per = (W + 31) >> 5;
  for (int e = warp; e < E; e += nw) {
    const int b = min(W, lane * per), w_end = min(W, b + per);
    int sum = 0;
    for (int w = b; w < w_end; ++w) sum += __popc(bits[e * W + w]);
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - sum;
    for (int w = b; w < w_end; ++w) {
      wpre[e * W + w] = run;
      run += __popc(bits[e * W + w]);
    }
    if (lane == 31) total[e] = incl;
  }
  __syncthreads();
  if (warp == 0) expert_tables_warp(total, start, E, a.o, true, lane);
  __syncthreads();
  for (int s = threadIdx.x; s < R; s += nthr) {
    const int64_t x = a.idx[s];
    int row = -1;
    if (x >= 0 && x < E) {
      const int e = static_cast<int>(x), w = s >> 5;
      row = start[e] + wpre[e * W + w] + __popc(bits[e * W + w] & ((1u << (s & 31)) - 1u));
      a.o.src_info[row] = s;
    }
    a.o.slot_to_row[s] = row;
  }
  __syncthreads();
}

__device__ void perm_small_block(const PermArgs& a, int* sm) {
  if (perm_bitmap_case(a.R, a.E)) {
    perm_bitmap_block(a, sm);
    return;
  }
  const int E = a.E;
  const int R = static_cast<int>(a.R);
  const int nw = blockDim.x >> 5;
  int* hist = sm;                  // [nw][E]: counts, then each warp's running offset inside the expert
  int* total = hist + nw * E;      // [E]
  int* start = total + E;          // [E+1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  for (int i = threadIdx.x; i < nw * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int per = (R + nw - 1) / nw;
  const int b0 = min(R, warp * per), b1 = min(R, b0 + per);
  int* my = hist + warp * E;
  // Each warp's slots go in batches of kPermBatch rounds of 32: a batch's
  // index loads are issued together.  A warp whose slots fit in one batch
  // keeps them in registers for the second pass.
  const bool one_batch = b1 - b0 <= 32 * kPermBatch;
  int v[kPermBatch];
  for (int base = b0; base < b1; base += 32 * kPermBatch) {
#pragma unroll
    for (int j = 0; j < kPermBatch; ++j) {
      const int s = base + 32 * j + lane;
      v[j] = -1;
      if (s < b1) {
        const int64_t x = a.idx[s];
        if (x >= 0 && x < E) v[j] = static_cast<int>(x);
        else if (x != -1) record_error(a.status, MOE_ERR_BAD_INDEX);
      }
    }
#pragma unroll
    for (int j = 0; j < kPermBatch; ++j) {
      if (base + 32 * j >= b1) break;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, v[j] >= 0 ? v[j] : E + lane);
      if (v[j] >= 0 && lane == 31 - __clz(peers)) my[v[j]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  // per expert: each warp's offset inside the expert (exclusive over warps)
  // and the expert's total
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < nw; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    total[e] = run;
  }
  __syncthreads();
  if (warp == 0) expert_tables_warp(total, start, E, a.o, true, lane);
  __syncthreads();
  for (int base = b0; base < b1; base += 32 * kPermBatch) {
    if (!one_batch) {
#pragma unroll
      for (int j = 0; j < kPermBatch; ++j) {
        const int s = base + 32 * j + lane;
        v[j] = -1;
        if (s < b1) {
          const int64_t x = a.idx[s];
          if (x >= 0 && x < E) v[j] = static_cast<int>(x);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kPermBatch; ++j) {
      if (base + 32 * j >= b1) break;
      const int s = base + 32 * j + lane;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, v[j] >= 0 ? v[j] : E + lane);
      int row = -1;
      if (v[j] >= 0) {
        row = start[v[j]] + my[v[j]] + __popc(peers & lt);
        a.o.src_info[row] = s;
      }
      if (s < b1) a.o.slot_to_row[s] = row;
      __syncwarp();
      if (v[j] >= 0 && lane == 31 - __clz(peers)) my[v[j]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) perm_count_kernel(PermArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  perm_count_chunk(a, blockIdx.x, sm);
}

__global__ void __launch_bounds__(256) perm_scatter_kernel(PermArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  perm_scatter_chunk(a, blockIdx.x, sm);
}

__global__ void __launch_bounds__(1024) perm_small_kernel(PermArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  perm_small_block(a, sm);
}

// ---------------------------------------------------------------------------
// Gather of activation rows into expert order (the A operand of the gate_up
// GEMM) with their block scales in the padded per-expert scale layout
// (Struct_mega_ffn_ep_combine_send: a_scale_offsets).  One warp per row.
// ---------------------------------------------------------------------------
struct GatherArgs {
  const uint8_t* x;          // [M][row_bytes]
  const void* x_scale;       // FP8: fp32 [M][H/128]; NVFP4: e4m3 [M][H/16]; MXFP8: ue8m0 [M][H/32]
  const int* src_info;
  const int* starts;
  const int* a_scale_offsets;
  int64_t R;                 // rows allocated (M*k)
  int E;
  int row_bytes;
  int topk;
  int H;
  int fmt;                   // FMT_*
  uint8_t* x_perm;           // [R][row_bytes]
  float* sa_t;               // FP8: [H/128][ld]
  uint8_t* sfa;              // NVFP4 / MXFP8: tiles [P/128][H/64 | H/128]
  int ld;                    // padded rows allocated
  // small-M GEMMs: their tile table (32-row tiles), built here; null otherwise
  const int* expert_ids;
  const int* num_active;
  int* tiles32;
  int skip_rows;             // the GEMM reads the routed rows of x itself: no row / scale copies
};

// Tile table of the small-M GEMMs: tiles32[a] = 32-row tiles of the active
// experts before slot a, tiles32[num_active] = all of them.  One warp.
__device__ void small_tile_table(const GatherArgs& g, int lane) {
  const int na = *g.num_active;
  const int per = (na + 31) >> 5;
  const int b = min(na, lane * per), e_end = min(na, b + per);
  int sum = 0;
  for (int a = b; a < e_end; ++a) {
    const int e = g.expert_ids[a];
    sum += (g.starts[e + 1] - g.starts[e] + 31) >> 5;
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += x;
  }
  int run = incl - sum;
  for (int a = b; a < e_end; ++a) {
    g.tiles32[a] = run;
    const int e = g.expert_ids[a];
    run += (g.starts[e + 1] - g.starts[e] + 31) >> 5;
  }
  if (lane == 31) g.tiles32[na] = incl;
}

// The expert owning row r: the largest e with starts[e] <= r (empty experts
// before it have smaller ids, those after it start past r).
__device__ __forceinline__ int gather_expert_of(const GatherArgs& g, int64_t r) {
  int lo = 0, hi = g.E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (g.starts[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// Copies rows r0 and r1 (r1 < 0: none) of x into expert order with all of a
// lane's loads of both 4 KB slices in flight before any store.
__device__ __forceinline__ void gather_copy2(const GatherArgs& g, int64_t r0, int64_t t0, int64_t r1, int64_t t1,
                                             int lane) {
  const int nvec = g.row_bytes / 16;
  const uint4* __restrict__ s0 = reinterpret_cast<const uint4*>(g.x + t0 * g.row_bytes);
  const uint4* __restrict__ s1 = reinterpret_cast<const uint4*>(g.x + (r1 >= 0 ? t1 : t0) * g.row_bytes);
  uint4* __restrict__ d0 = reinterpret_cast<uint4*>(g.x_perm + r0 * g.row_bytes);
  uint4* __restrict__ d1 = reinterpret_cast<uint4*>(g.x_perm + (r1 >= 0 ? r1 : r0) * g.row_bytes);
  for (int i0 = 0; i0 < nvec; i0 += 256) {
    uint4 v0[8], v1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + lane + 32 * j;
      if (i < nvec) {
        v0[j] = __ldg(s0 + i);
        if (r1 >= 0) v1[j] = __ldg(s1 + i);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + lane + 32 * j;
      if (i < nvec) {
        d0[i] = v0[j];
        if (r1 >= 0) d1[i] = v1[j];
      }
    }
  }
}

// The block scales of routed row r (token t, padded scale row pr).
__device__ __forceinline__ void gather_scales(const GatherArgs& g, int64_t t, int pr, int lane) {
  if (g.fmt == 1) {
    const float* xs = static_cast<const float*>(g.x_scale) + t * (g.H / 128);
    for (int kb = lane; kb < g.H / 128; kb += 32) g.sa_t[static_cast<size_t>(kb) * g.ld + pr] = xs[kb];
  } else if (g.fmt == 2 || g.fmt == 3) {
    // one byte per 16 (NVFP4) or 32 (MXFP8) elements, four per tile row
    const int cols = g.fmt == 2 ? g.H / 16 : g.H / 32;
    const uint8_t* xs = static_cast<const uint8_t*>(g.x_scale) + t * cols;
    const int kc = cols / 4;
    for (int j = lane; j < cols; j += 32) {
      const size_t off = (static_cast<size_t>(pr >> 7) * kc + (j >> 2)) * 512 + (pr & 31) * 16 +
                         ((pr >> 5) & 3) * 4 + (j & 3);
      g.sfa[off] = xs[j];
    }
  }
}

// The calling warp's contiguous run of rows (an equal share of the valid
// slots, warp_id-th of nwarps), two rows per step.  Consecutive rows share
// their expert, so its search runs once per run and the expert then only
// advances; each row's token comes from src_info.
__device__ __forceinline__ void gather_rows(const GatherArgs& g, int64_t warp_id, int64_t nwarps, int lane) {
  const int64_t valid = g.starts[g.E];
  const int64_t per = (valid + nwarps - 1) / nwarps;
  const int64_t rb = warp_id * per;
  const int64_t re = min(valid, rb + per);
  if (rb >= re) return;
  int e = gather_expert_of(g, rb);
  int64_t e_end = g.starts[e + 1];
  int64_t sbase = g.a_scale_offsets[e] - g.starts[e];   // padded scale row = sbase + r
  for (int64_t r0 = rb; r0 < re; r0 += 2) {
    const int64_t r1 = (r0 + 1 < re) ? r0 + 1 : -1;
    while (r0 >= e_end) {
      ++e;
      e_end = g.starts[e + 1];
      sbase = g.a_scale_offsets[e] - g.starts[e];
    }
    const int p0 = static_cast<int>(sbase + r0);
    int p1 = 0;
    if (r1 >= 0) {
      while (r1 >= e_end) {
        ++e;
        e_end = g.starts[e + 1];
        sbase = g.a_scale_offsets[e] - g.starts[e];
      }
      p1 = static_cast<int>(sbase + r1);
    }
    const int64_t t0 = g.src_info[r0] / g.topk;
    const int64_t t1 = (r1 >= 0) ? g.src_info[r1] / g.topk : 0;
    gather_copy2(g, r0, t0, r1, t1, lane);
    if (g.fmt == 2 || g.fmt == 3) {
      gather_scales(g, t0, p0, lane);
      if (r1 >= 0) gather_scales(g, t1, p1, lane);
    }
  }
  if (g.fmt == 1) {
    // FP8 scales, transposed [H/128][padded rows]: lane l takes row r + l of
    // each 32-row group, so every K block's 32 scales are written as
    // consecutive padded rows
    const int kbs = g.H / 128;
    int le = gather_expert_of(g, rb);
    for (int64_t r = rb + lane; r - lane < re; r += 32) {
      if (r < re) {
        while (r >= g.starts[le + 1]) ++le;
        const size_t pr = static_cast<size_t>(g.a_scale_offsets[le] + (r - g.starts[le]));
        const float* xs = static_cast<const float*>(g.x_scale) + static_cast<int64_t>(g.src_info[r] / g.topk) * kbs;
        for (int kb = 0; kb < kbs; ++kb) g.sa_t[static_cast<size_t>(kb) * g.ld + pr] = __ldg(xs + kb);
      }
    }
  }
}

__global__ void __launch_bounds__(256) gather_kernel(GatherArgs g) {
  pdl_trigger();
  pdl_wait();
  if (g.tiles32 && blockIdx.x == 0 && threadIdx.x < 32) small_tile_table(g, threadIdx.x);
  if (g.skip_rows) return;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  gather_rows(g, (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5, nw, threadIdx.x & 31);
}

__device__ __forceinline__ void zero_range(float4* __restrict__ p, int64_t n4, int64_t i0, int64_t stride) {
  for (int64_t i = i0; i < n4; i += stride) p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(256) zero_kernel(float4* __restrict__ p, int64_t n4) {
  pdl_trigger();
  pdl_wait();
  zero_range(p, n4, static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x,
             static_cast<int64_t>(gridDim.x) * blockDim.x);
}

// FP32 accumulator [n] -> BF16, round to nearest even; 8 elements per item,
// four items' loads in flight per thread.
__device__ __forceinline__ void finalize_range(const float4* __restrict__ acc, uint4* __restrict__ out, int64_t n8,
                                               int64_t i0, int64_t stride) {
  for (int64_t ib = i0; ib < n8; ib += 4 * stride) {
    float4 a[4], b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = ib + j * stride;
      if (i < n8) {
        a[j] = acc[2 * i];
        b[j] = acc[2 * i + 1];
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = ib + j * stride;
      if (i < n8)
        out[i] = make_uint4(pack_bf16x2(a[j].x, a[j].y), pack_bf16x2(a[j].z, a[j].w), pack_bf16x2(b[j].x, b[j].y),
                            pack_bf16x2(b[j].z, b[j].w));
    }
  }
}

__global__ void __launch_bounds__(256) finalize_kernel(const float4* __restrict__ acc,
                                                       uint4* __restrict__ out, int64_t n8) {
  pdl_trigger();
  pdl_wait();
  finalize_range(acc, out, n8, static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x,
                 static_cast<int64_t>(gridDim.x) * blockDim.x);
}

// Staged combine (DistributedEPCombine): out[t] = bf16(sum_j w[t,j] *
// in[slot_to_row[t*k+j]]), j ascending, FP32 sums; 8 columns per step.
__global__ void __launch_bounds__(256) combine_staged_kernel(const float* __restrict__ in,
                                                             const int* __restrict__ slot_to_row,
                                                             const float* __restrict__ w,
                                                             int64_t M, int H, int k,
                                                             uint4* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int64_t n8 = M * (H / 8);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / (H / 8);
    const int c = static_cast<int>(i - t * (H / 8)) * 8;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int row = slot_to_row[t * k + j];
      if (row < 0) continue;
      const float wt = w[t * k + j];
      const float4* src = reinterpret_cast<const float4*>(in + static_cast<int64_t>(row) * H + c);
      const float4 a = src[0], b = src[1];
      s[0] = fmaf(wt, a.x, s[0]); s[1] = fmaf(wt, a.y, s[1]);
      s[2] = fmaf(wt, a.z, s[2]); s[3] = fmaf(wt, a.w, s[3]);
      s[4] = fmaf(wt, b.x, s[4]); s[5] = fmaf(wt, b.y, s[5]);
      s[6] = fmaf(wt, b.z, s[6]); s[7] = fmaf(wt, b.w, s[7]);
    }
    out[i] = make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]),
                        pack_bf16x2(s[4], s[5]), pack_bf16x2(s[6], s[7]));
  }
}

}  // namespace moe

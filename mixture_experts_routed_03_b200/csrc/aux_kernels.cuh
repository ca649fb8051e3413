// aux_kernels.cuh -- the memory-bound steps around the expert GEMMs:
// routing from logits, the counting-sort permutation, the activation gather
// into expert order, accumulator zeroing, the BF16 finalise and the staged
// (deterministic) combine, and the one-time NVFP4 scale-tile preparation.
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
__device__ __forceinline__ uint64_t route_key(float s, int e) {
  if (s == 0.0f) s = 0.0f;  // -0 and +0 are the same score
  const uint32_t b = __float_as_uint(s);
  const uint32_t ord = (s != s) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
  return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - e);
}

template <int PER>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias, int64_t M,
                                                    int E, int k, int64_t* __restrict__ idx_out,
                                                    float* __restrict__ w_out) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  const float* row = logits + t * E;
  uint64_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < E) key[i] = route_key(__fadd_rn(row[e], bias ? bias[e] : 0.0f), e);
  }
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
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
  const bool mine = lane < k;
  const float l = mine ? row[my_e] : -INFINITY;
  float mx = l;
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  const float ex = mine ? expf(l - mx) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
  if (mine) {
    idx_out[t * k + lane] = my_e;
    w_out[t * k + lane] = __fdiv_rn(ex, sum);
  }
}

// ---------------------------------------------------------------------------
// Permutation (Struct_mega_ffn_ep_combine_send: expert_start_indices,
// expert_ids, a_scale_offsets, src_info, num_active_experts): a stable
// counting sort of the flat slots s = t*k + j by expert.
//   pass 1: per 1024-slot chunk, count slots per expert (shared atomics)
//   pass 2: per chunk, the expert totals and this chunk's offset within each
//           expert give every slot its row; one warp walks the chunk in
//           order, ranking equal experts inside each 32-slot round with
//           __match_any_sync, so rows ascend in slot index.  Chunk 0 also
//           writes the per-expert arrays and the GEMM tile table.
// ---------------------------------------------------------------------------
constexpr int kPermChunk = 1024;

__global__ void __launch_bounds__(256) perm_count_kernel(const int64_t* __restrict__ idx,
                                                         int64_t R, int E,
                                                         int* __restrict__ block_counts,
                                                         int* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x) {
    const int64_t s = base + i;
    if (s < R) {
      const int64_t v = idx[s];
      if (v >= 0 && v < E) atomicAdd(&cnt[v], 1);
      else if (v != -1) record_error(status, MOE_ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_counts[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

struct PermOut {
  int* expert_counts;
  int* expert_start_indices;
  int* src_info;
  int* slot_to_row;
  int* expert_ids;
  int* num_active;
  int* a_scale_offsets;
  int* tile_offsets;
};

// Exclusive scan of v[0..n) by one warp (n <= 1024); writes out[0..n] (n+1
// entries, out[n] = total).  Each lane owns a contiguous run of entries.
__device__ void warp_exclusive_scan(const int* v, int* out, int n) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  const int b = min(n, lane * per), e = min(n, b + per);
  int local = 0;
  for (int i = b; i < e; ++i) local += v[i];
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  int run = incl - local;
  for (int i = b; i < e; ++i) {
    out[i] = run;
    run += v[i];
  }
  if (lane == 31) out[n] = incl;
}

// Writes expert_counts, expert_start_indices, a_scale_offsets, expert_ids,
// num_active and tile_offsets from the per-expert totals and their exclusive
// scan (start, E+1 entries).  Called by every thread of one block; tmp and
// tmp2 are E+1-entry shared scratch arrays.
__device__ void write_expert_arrays(const int* total, const int* start, int* tmp, int* tmp2, int E,
                                    const PermOut& o) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    o.expert_counts[e] = total[e];
    o.expert_start_indices[e] = start[e];
    tmp[e] = (total[e] + 127) / 128 * 128;  // padded rows
    tmp2[e] = (total[e] > 0) ? 1 : 0;
  }
  if (threadIdx.x == 0) o.expert_start_indices[E] = start[E];
  __syncthreads();
  if (threadIdx.x < 32) warp_exclusive_scan(tmp, o.a_scale_offsets, E);
  __syncthreads();
  // active experts: compact with a scan of the flags (tmp becomes the ranks)
  if (threadIdx.x < 32) warp_exclusive_scan(tmp2, tmp, E);
  __syncthreads();
  const int na = tmp[E];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (total[e] > 0) {
      o.expert_ids[tmp[e]] = e;
      tmp2[tmp[e]] = (total[e] + 127) / 128;  // m tiles of the a-th active expert
    }
    if (e >= na) o.expert_ids[e] = -1;
  }
  if (threadIdx.x == 0) *o.num_active = na;
  __syncthreads();
  if (threadIdx.x < 32) warp_exclusive_scan(tmp2, o.tile_offsets, na);
}

__global__ void __launch_bounds__(256) perm_scatter_kernel(const int64_t* __restrict__ idx,
                                                           int64_t R, int E, int nblk,
                                                           const int* __restrict__ block_counts,
                                                           PermOut o) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  int* total = sm;                 // [E]
  int* start = total + E;          // [E+1]
  int* cursor = start + E + 1;     // [E]
  int* tmp = cursor + E;           // [E+1]
  int* tmp2 = tmp + E + 1;         // [E+1]
  int* sidx = tmp2 + E + 1;        // [kPermChunk] this chunk's expert ids
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += blockDim.x) {
    const int64_t s = base + i;
    int v = -1;
    if (s < R) {
      const int64_t x = idx[s];
      v = (x >= 0 && x < E) ? static_cast<int>(x) : -1;
    }
    sidx[i] = v;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int tot = 0, before = 0;
    for (int b = 0; b < nblk; ++b) {
      const int c = block_counts[static_cast<size_t>(b) * E + e];
      tot += c;
      if (b < static_cast<int>(blockIdx.x)) before += c;
    }
    total[e] = tot;
    cursor[e] = before;
  }
  __syncthreads();
  if (threadIdx.x < 32) warp_exclusive_scan(total, start, E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] += start[e];

  if (blockIdx.x == 0) write_expert_arrays(total, start, tmp, tmp2, E, o);
  __syncthreads();

  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const unsigned lt = (1u << lane) - 1u;
    for (int rnd = 0; rnd < kPermChunk / 32; ++rnd) {
      const int64_t s = base + rnd * 32 + lane;
      if (base + rnd * 32 >= R) break;
      const int v = sidx[rnd * 32 + lane];
      const bool valid = v >= 0;
      const int key = valid ? v : (E + lane);
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
      int row = -1;
      if (valid) {
        row = cursor[v] + __popc(peers & lt);
        o.src_info[row] = static_cast<int>(s);
      }
      if (s < R) o.slot_to_row[s] = row;
      __syncwarp();
      if (valid && lane == 31 - __clz(peers)) cursor[v] += __popc(peers);
      __syncwarp();
    }
  }
}

// Single-launch permutation for small problems (R <= kPermSmallMax slots,
// E <= kPermSmallMaxE): one block of 32 warps; warp w owns a contiguous run
// of slots and counts it into its own histogram row; the rows' prefix sums in
// (expert, warp) order give every warp its first row per expert, so a second
// ordered pass over each run yields the same stable order as the two-kernel
// path.
constexpr int kPermSmallMax = 16384;
constexpr int kPermSmallMaxE = 256;

__global__ void __launch_bounds__(1024) perm_small_kernel(const int64_t* __restrict__ idx, int R, int E,
                                                          PermOut o, int* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int sm[];
  int* hist = sm;                  // [32][E]: counts, then each warp's running cursor
  int* total = hist + 32 * E;      // [E]
  int* start = total + E;          // [E+1]
  int* tmp = start + E + 1;        // [E+1]
  int* tmp2 = tmp + E + 1;         // [E+1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int per = (R + 31) / 32;
  const int b0 = min(R, warp * per), b1 = min(R, b0 + per);
  int* my = hist + warp * E;
  for (int base = b0; base < b1; base += 32) {
    const int s = base + lane;
    int v = -1;
    if (s < b1) {
      const int64_t x = idx[s];
      if (x >= 0 && x < E) v = static_cast<int>(x);
      else if (x != -1) record_error(status, MOE_ERR_BAD_INDEX);
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, v >= 0 ? v : E + lane);
    if (v >= 0 && lane == 31 - __clz(peers)) my[v] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int t = 0;
    for (int w = 0; w < 32; ++w) t += hist[w * E + e];
    total[e] = t;
  }
  __syncthreads();
  if (threadIdx.x < 32) warp_exclusive_scan(total, start, E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = start[e];
    for (int w = 0; w < 32; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  write_expert_arrays(total, start, tmp, tmp2, E, o);
  for (int base = b0; base < b1; base += 32) {
    const int s = base + lane;
    int v = -1;
    if (s < b1) {
      const int64_t x = idx[s];
      if (x >= 0 && x < E) v = static_cast<int>(x);
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, v >= 0 ? v : E + lane);
    int row = -1;
    if (v >= 0) {
      row = my[v] + __popc(peers & lt);
      o.src_info[row] = s;
    }
    if (s < b1) o.slot_to_row[s] = row;
    __syncwarp();
    if (v >= 0 && lane == 31 - __clz(peers)) my[v] += __popc(peers);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Gather of activation rows into expert order (the A operand of the gate_up
// GEMM) with their block scales in the padded per-expert scale layout
// (Struct_mega_ffn_ep_combine_send: a_scale_offsets).  One warp per row.
// ---------------------------------------------------------------------------
struct GatherArgs {
  const uint8_t* x;          // [M][row_bytes]
  const void* x_scale;       // FP8: fp32 [M][H/128]; NVFP4: e4m3 [M][H/16]
  const int* src_info;
  const int* starts;
  const int* a_scale_offsets;
  int64_t R;                 // rows allocated (M*k)
  int row_bytes;
  int topk;
  int H;
  int fmt;                   // FMT_*
  uint8_t* x_perm;           // [R][row_bytes]
  float* sa_t;               // FP8: [H/128][ld]
  uint8_t* sfa;              // NVFP4: tiles [P/128][H/64]
  int ld;                    // padded rows allocated
};

__global__ void __launch_bounds__(256) gather_kernel(GatherArgs g, int E) {
  pdl_trigger();
  pdl_wait();
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= g.R) return;
  if (r >= g.starts[E]) return;  // rows past the valid slots
  const int s = g.src_info[r];
  const int64_t t = s / g.topk;
  // the expert owning row r: starts[e] <= r < starts[e+1]
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (g.starts[mid] <= r) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int pr = g.a_scale_offsets[e] + static_cast<int>(r - g.starts[e]);
  const int nvec = g.row_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(g.x + t * g.row_bytes);
  uint4* dst = reinterpret_cast<uint4*>(g.x_perm + r * g.row_bytes);
  for (int i = lane; i < nvec; i += 32) dst[i] = src[i];
  if (g.fmt == 1) {
    const float* xs = static_cast<const float*>(g.x_scale) + t * (g.H / 128);
    for (int kb = lane; kb < g.H / 128; kb += 32) g.sa_t[static_cast<size_t>(kb) * g.ld + pr] = xs[kb];
  } else if (g.fmt == 2) {
    const uint8_t* xs = static_cast<const uint8_t*>(g.x_scale) + t * (g.H / 16);
    const int kc = g.H / 64;
    for (int j = lane; j < g.H / 16; j += 32) {
      const size_t off = (static_cast<size_t>(pr >> 7) * kc + (j >> 2)) * 512 + (pr & 31) * 16 +
                         ((pr >> 5) & 3) * 4 + (j & 3);
      g.sfa[off] = xs[j];
    }
  }
}

__global__ void __launch_bounds__(256) zero_kernel(float4* __restrict__ p, int64_t n4) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// FP32 accumulator [n] -> BF16, round to nearest even; 8 elements per step.
__global__ void __launch_bounds__(256) finalize_kernel(const float4* __restrict__ acc,
                                                       uint4* __restrict__ out, int64_t n8) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    out[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                        pack_bf16x2(b.z, b.w));
  }
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

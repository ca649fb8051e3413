// moe_api.cu -- the C ABI of include/moe.h: argument validation, workspace
// carving, TMA descriptor set-up and kernel launches.  No memory is
// allocated here; every buffer is the caller's.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "aux_kernels.cuh"
#include "fused.cuh"
#include "gemm.cuh"
#include "gemm_swap.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- validation
int x_row_bytes(int fmt, int H) { return fmt == FMT_BF16 ? 2 * H : (fmt == FMT_NVFP4 ? H / 2 : H); }
int h_row_bytes(int fmt, int I) { return fmt == FMT_BF16 ? 2 * I : (fmt == FMT_NVFP4 ? I / 2 : I); }

// Bytes of the block scales of one padded row of K elements.
size_t scale_row_bytes(int fmt, int K) {
  return fmt == FMT_FP8 ? size_t(K / 128) * 4 : fmt == FMT_NVFP4 ? size_t(K / 16) : fmt == FMT_MXFP8 ? size_t(K / 32) : 0;
}

moe_status_t check_problem(const moe_problem_t* p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens < 0) return MOE_ERR_INVALID_ARG;
  if (p->format < MOE_FMT_BF16 || p->format > MOE_FMT_FP8_PER_TENSOR) return MOE_ERR_INVALID_ARG;
  if (p->hidden <= 0 || p->hidden % 256 != 0) return MOE_ERR_INVALID_ARG;
  if (p->intermediate_hidden <= 0 || p->intermediate_hidden % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (p->num_experts < 1 || p->num_topk < 1 || p->num_topk > p->num_experts) return MOE_ERR_INVALID_ARG;
  if (p->shared_expert != 0 && p->shared_expert != 1) return MOE_ERR_INVALID_ARG;
  if (p->activation != MOE_ACT_SWIGLU && p->activation != MOE_ACT_SWIGLUOAI) return MOE_ERR_INVALID_ARG;
  if (p->activation == MOE_ACT_SWIGLUOAI && !(std::isfinite(p->activation_alpha) && p->activation_alpha > 0.0f))
    return MOE_ERR_INVALID_ARG;
  // with a shared expert: num_experts + 1 experts, num_topk + 1 slots per token
  const int E_all = p->num_experts + p->shared_expert;
  const int k_all = p->num_topk + p->shared_expert;
  if (E_all > 1024) return MOE_ERR_UNSUPPORTED;
  if (std::isnan(p->activation_clamp) || !(p->activation_clamp > 0.0f)) return MOE_ERR_INVALID_ARG;
  if (p->tile_regime < MOE_TILE_AUTO || p->tile_regime > MOE_TILE_SMALL_M) return MOE_ERR_INVALID_ARG;
  if (p->format == MOE_FMT_NVFP4 && p->intermediate_hidden % 256 != 0) return MOE_ERR_UNSUPPORTED;
  const int64_t R = p->num_tokens * k_all;
  if (R > (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  // expert weight row indices are 32-bit in the TMA coordinates
  if (int64_t(E_all) * 2 * p->intermediate_hidden >= (int64_t(1) << 31) ||
      int64_t(E_all) * p->hidden >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// The problem every step after the routing works on: a fused shared expert
// (EPConfig fused_shared_expert) is one more expert, index num_experts, and
// one more slot per token, its last column, so the permutation, the GEMMs
// and the combine treat it as a routed expert that every token chose.
moe_problem_t effective(const moe_problem_t* p) {
  moe_problem_t q = *p;
  q.num_experts += p->shared_expert;
  q.num_topk += p->shared_expert;
  q.shared_expert = 0;
  return q;
}

// ---------------------------------------------------------------- workspace
struct WsLayout {
  int64_t M, R, P;   // tokens, routed rows, padded scale rows
  int nblk;          // permute chunks
  size_t header, route_idx, route_w;
  size_t counts, starts, src_info, slot_to_row, expert_ids, num_active, a_scale_offsets, tile_offsets;
  size_t block_counts, tiles32;
  size_t x_perm, x_sf;
  size_t h, h_sf;
  size_t acc;
  size_t total;
  size_t h_bytes, h_sf_bytes;
};

WsLayout make_layout(const moe_problem_t* p) {
  WsLayout L{};
  const int E = p->num_experts, H = p->hidden, I = p->intermediate_hidden, fmt = p->format;
  L.M = p->num_tokens;
  L.R = L.M * p->num_topk;
  L.P = int64_t(align_up(size_t(L.R), 128)) + 128 * std::min<int64_t>(E, L.R);
  L.nblk = int((L.R + kPermChunk - 1) / kPermChunk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + std::max<size_t>(bytes, 1), kAlign);
    return o;
  };
  L.header = take(sizeof(WsHeader));
  L.route_idx = take(size_t(L.R) * 8);
  L.route_w = take(size_t(L.R) * 4);
  L.counts = take(size_t(E) * 4);
  L.starts = take(size_t(E + 1) * 4);
  L.src_info = take(size_t(L.R) * 4);
  L.slot_to_row = take(size_t(L.R) * 4);
  L.expert_ids = take(size_t(E) * 4);
  L.num_active = take(4);
  L.a_scale_offsets = take(size_t(E + 1) * 4);
  L.tile_offsets = take(size_t(E + 1) * 4);
  L.block_counts = take(size_t(L.nblk) * E * 4);
  L.tiles32 = take(size_t(E + 1) * 4);
  L.x_perm = take(size_t(L.R) * x_row_bytes(fmt, H));
  L.x_sf = take(size_t(L.P) * scale_row_bytes(fmt, H));
  L.h_bytes = size_t(L.R) * h_row_bytes(fmt, I);
  L.h_sf_bytes = size_t(L.P) * scale_row_bytes(fmt, I);
  L.h = take(L.h_bytes);
  L.h_sf = take(L.h_sf_bytes);
  L.acc = take(size_t(L.M) * H * 4);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- TMA maps
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

// 2-D byte tensor [rows][row_bytes], boxes of 128 bytes x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_bytes & 15) || rows == 0) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- timing
struct Timing {
  bool on = false;
  int cap = 0;            // event pairs per slot
  int used[MOE_NUM_SLOTS] = {0};
  cudaEvent_t* ev = nullptr;  // [MOE_NUM_SLOTS][cap][2]
  std::mutex mu;
};
Timing g_tim;

// Records the start event of `slot` on `st`; returns the pair index or -1.
int tim_begin(int slot, cudaStream_t st) {
  if (!g_tim.on) return -1;
  std::lock_guard<std::mutex> lk(g_tim.mu);
  const int i = g_tim.used[slot];
  if (i >= g_tim.cap) return -1;
  g_tim.used[slot] = i + 1;
  cudaEventRecord(g_tim.ev[(size_t(slot) * g_tim.cap + i) * 2], st);
  return i;
}

void tim_end(int slot, int i, cudaStream_t st) {
  if (i < 0) return;
  cudaEventRecord(g_tim.ev[(size_t(slot) * g_tim.cap + i) * 2 + 1], st);
}

struct TimScope {
  int slot, i;
  cudaStream_t st;
  TimScope(int s, cudaStream_t stream) : slot(s), i(tim_begin(s, stream)), st(stream) {}
  ~TimScope() { tim_end(slot, i, st); }
};

// ---------------------------------------------------------------- launches
// Every kernel is launched with programmatic stream serialisation: it may be
// scheduled while the previous kernel of the stream drains, runs its
// prologue, and waits (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int FMT, int EPI>
cudaError_t set_gemm_attr() {
  return cudaFuncSetAttribute(moe_gemm_kernel<FMT, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GemmCfg<FMT, EPI>::kSmemBytes);
}

template <int FMT, int EPI>
cudaError_t set_swap_attr() {
  return cudaFuncSetAttribute(moe_gemm_swap_kernel<FMT, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              SwapCfg<FMT, EPI>::kSmemBytes);
}

template <int FMT>
cudaError_t set_swap_attrs_fmt() {
  cudaError_t e;
  if ((e = set_swap_attr<FMT, EPI_L1>()) != cudaSuccess) return e;
  if ((e = set_swap_attr<FMT, EPI_L2_ACC>()) != cudaSuccess) return e;
  if ((e = set_swap_attr<FMT, EPI_L2_STAGED>()) != cudaSuccess) return e;
  return cudaFuncSetAttribute(moe_fused_kernel<FMT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              fused_smem_bytes<FMT, true>());
}

template <int FMT>
cudaError_t set_attrs_fmt() {
  cudaError_t e;
  if ((e = set_gemm_attr<FMT, EPI_L1>()) != cudaSuccess) return e;
  if ((e = set_gemm_attr<FMT, EPI_L2_ACC>()) != cudaSuccess) return e;
  return set_gemm_attr<FMT, EPI_L2_STAGED>();
}

template <int FMT>
cudaError_t set_fused_attr() {
  return cudaFuncSetAttribute(moe_fused_kernel<FMT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              fused_smem_bytes<FMT, false>());
}

cudaError_t set_all_attrs() {
  cudaError_t e;
  if ((e = set_fused_attr<FMT_BF16>()) != cudaSuccess) return e;
  if ((e = set_fused_attr<FMT_FP8>()) != cudaSuccess) return e;
  if ((e = set_fused_attr<FMT_NVFP4>()) != cudaSuccess) return e;
  if ((e = set_fused_attr<FMT_MXFP8>()) != cudaSuccess) return e;
  if ((e = set_fused_attr<FMT_FP8T>()) != cudaSuccess) return e;
  if ((e = set_attrs_fmt<FMT_BF16>()) != cudaSuccess) return e;
  if ((e = set_attrs_fmt<FMT_FP8>()) != cudaSuccess) return e;
  if ((e = set_attrs_fmt<FMT_NVFP4>()) != cudaSuccess) return e;
  if ((e = set_attrs_fmt<FMT_MXFP8>()) != cudaSuccess) return e;
  if ((e = set_attrs_fmt<FMT_FP8T>()) != cudaSuccess) return e;
  if ((e = set_swap_attrs_fmt<FMT_BF16>()) != cudaSuccess) return e;
  if ((e = set_swap_attrs_fmt<FMT_FP8>()) != cudaSuccess) return e;
  if ((e = set_swap_attrs_fmt<FMT_NVFP4>()) != cudaSuccess) return e;
  if ((e = set_swap_attrs_fmt<FMT_MXFP8>()) != cudaSuccess) return e;
  return set_swap_attrs_fmt<FMT_FP8T>();
}

bool ensure_init() {
  static int inited_mask[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && inited_mask[dev]) return true;
  if (set_all_attrs() != cudaSuccess) return false;
  if (dev >= 0 && dev < 64) inited_mask[dev] = 1;
  return true;
}

template <int FMT, int EPI>
cudaError_t launch_gemm(const GemmArgs& a, const CUtensorMap& ta, int grid, cudaStream_t st) {
  return launch_k(moe_gemm_kernel<FMT, EPI>, grid, GemmCfg<FMT, EPI>::kThreads, GemmCfg<FMT, EPI>::kSmemBytes,
                  st, a, ta);
}

template <int FMT, int EPI>
cudaError_t launch_swap(const GemmArgs& a, const CUtensorMap& ta, int grid, cudaStream_t st) {
  return launch_k(moe_gemm_swap_kernel<FMT, EPI>, grid, SwapCfg<FMT, EPI>::kThreads,
                  SwapCfg<FMT, EPI>::kSmemBytes, st, a, ta);
}

template <int EPI>
cudaError_t launch_gemm_fmt(int fmt, bool swap, const GemmArgs& a, const CUtensorMap& ta, int grid,
                            cudaStream_t st) {
  if (swap) {
    switch (fmt) {
      case FMT_BF16: return launch_swap<FMT_BF16, EPI>(a, ta, grid, st);
      case FMT_FP8: return launch_swap<FMT_FP8, EPI>(a, ta, grid, st);
      case FMT_MXFP8: return launch_swap<FMT_MXFP8, EPI>(a, ta, grid, st);
      case FMT_FP8T: return launch_swap<FMT_FP8T, EPI>(a, ta, grid, st);
      default: return launch_swap<FMT_NVFP4, EPI>(a, ta, grid, st);
    }
  }
  switch (fmt) {
    case FMT_BF16: return launch_gemm<FMT_BF16, EPI>(a, ta, grid, st);
    case FMT_FP8: return launch_gemm<FMT_FP8, EPI>(a, ta, grid, st);
    case FMT_MXFP8: return launch_gemm<FMT_MXFP8, EPI>(a, ta, grid, st);
    case FMT_FP8T: return launch_gemm<FMT_FP8T, EPI>(a, ta, grid, st);
    default: return launch_gemm<FMT_NVFP4, EPI>(a, ta, grid, st);
  }
}

// Bytes of the prepared gate_up (L1) and down (L2) weight blobs.
size_t prepared_bytes(const moe_problem_t* p, bool l1) {
  const int fmt = p->format;
  const size_t E = p->num_experts, H = p->hidden, I = p->intermediate_hidden;
  const size_t n_tiles = l1 ? I / 128 : H / 256;
  const size_t k_stages = size_t(l1 ? x_row_bytes(fmt, int(H)) : h_row_bytes(fmt, int(I))) / 128;
  return E * n_tiles * k_stages * size_t(b_block_bytes(fmt));
}

int grid_for(int64_t n, int threads, int cap = 148 * 16) {
  int64_t g = (n + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return int(g);
}

RouteArgs route_args(const moe_problem_t* p, const float* logits, const float* bias, int64_t* idx, float* w) {
  RouteArgs a{};
  a.logits = logits;
  a.bias = bias;
  a.M = p->num_tokens;
  a.E = p->num_experts;
  a.k = p->num_topk;
  a.idx_out = idx;
  a.w_out = w;
  a.shared = p->shared_expert;
  a.out_k = p->num_topk + p->shared_expert;
  return a;
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  TimScope ts(MOE_SLOT_ROUTE, st);
  const int grid = grid_for(a.M * 32, 256, 1 << 30);
  switch (route_per(a.E)) {
    case 1: return launch_k(route_kernel<1>, grid, 256, 0, st, a);
    case 2: return launch_k(route_kernel<2>, grid, 256, 0, st, a);
    case 4: return launch_k(route_kernel<4>, grid, 256, 0, st, a);
    case 8: return launch_k(route_kernel<8>, grid, 256, 0, st, a);
    case 16: return launch_k(route_kernel<16>, grid, 256, 0, st, a);
    default: return launch_k(route_kernel<32>, grid, 256, 0, st, a);
  }
}

PermArgs perm_args(const moe_problem_t* p, const int64_t* idx, const PermOut& o, int* block_counts, int nblk,
                   int* status) {
  PermArgs a{};
  a.idx = idx;
  a.R = p->num_tokens * p->num_topk;
  a.E = p->num_experts;
  a.nblk = nblk;
  a.block_counts = block_counts;
  a.o = o;
  a.status = status;
  return a;
}

cudaError_t launch_permute(const PermArgs& a, cudaStream_t st) {
  TimScope ts(MOE_SLOT_PERMUTE, st);
  if (perm_small_case(a.R, a.E))
    return launch_k(perm_small_kernel, 1, 1024, perm_small_smem_ints(a.R, a.E, 32) * sizeof(int), st, a);
  cudaError_t e = launch_k(perm_count_kernel, a.nblk, 256, a.E * sizeof(int), st, a);
  if (e != cudaSuccess) return e;
  return launch_k(perm_scatter_kernel, a.nblk, 256, perm_chunk_smem_ints(a.E) * sizeof(int), st, a);
}

struct FfnBuffers {
  // layout
  const int *counts, *starts, *src_info, *slot_to_row, *expert_ids, *num_active, *a_scale_offsets, *tile_offsets;
  // scratch
  uint8_t *x_perm, *x_sf, *h, *h_sf;
  int* tiles32;     // small-M tile table (workspace)
  int64_t P;
  int* status;
};

// Everything the FFN kernels need: the gather, the two GEMMs and their A maps.
struct FfnPlan {
  GatherArgs g;
  GemmArgs l1, l2;
  CUtensorMap ta1, ta2;
  int grid1, grid2;
  bool swap;        // small-M (swapped-operand) GEMMs
};

// The GEMMs' tile regime for this problem (MOE_TILE_AUTO resolved).
bool small_m_tiles(const moe_problem_t* p) {
  if (p->tile_regime == MOE_TILE_SMALL_M) return true;
  if (p->tile_regime == MOE_TILE_LARGE_M) return false;
  return p->num_tokens * p->num_topk <= int64_t(64) * p->num_experts;
}

moe_status_t plan_ffn(const moe_problem_t* p, const moe_act_t* act, const moe_weights_t* w, const FfnBuffers& b,
                      const float* topk_weights, float* out, FfnPlan& pl) {
  const int fmt = p->format, H = p->hidden, I = p->intermediate_hidden, E = p->num_experts, k = p->num_topk;
  const int64_t M = p->num_tokens, R = M * k;
  const int nsm = sm_count();
  pl.swap = small_m_tiles(p);
  const int tile_rows = pl.swap ? kNT : kBM;

  GatherArgs& g = pl.g;
  g = GatherArgs{};
  g.x = static_cast<const uint8_t*>(act->x);
  g.x_scale = act->x_scale;
  g.src_info = b.src_info;
  g.starts = b.starts;
  g.a_scale_offsets = b.a_scale_offsets;
  g.R = R;
  g.E = E;
  g.row_bytes = x_row_bytes(fmt, H);
  g.topk = k;
  g.H = H;
  g.fmt = fmt;
  g.x_perm = b.x_perm;
  g.sa_t = reinterpret_cast<float*>(b.x_sf);
  g.sfa = b.x_sf;
  g.ld = int(b.P);
  g.expert_ids = b.expert_ids;
  g.num_active = b.num_active;
  g.tiles32 = pl.swap ? b.tiles32 : nullptr;
  // the small-M gate_up copies its routed rows straight from x: no gathered
  // copy (a large-M tile's 128 rows per K block arrive faster as one tiled
  // copy of gathered rows than as 32 four-row gathers from x)
  const bool direct_l1 = pl.swap;
  g.skip_rows = direct_l1 ? 1 : 0;

  // L1: gate_up (its A map, over the gathered rows, is unused by the
  // small-M tiles, which copy x rows themselves)
  if (!make_map(&pl.ta1, b.x_perm, x_row_bytes(fmt, H), uint64_t(R), uint32_t(tile_rows))) return MOE_ERR_CUDA;
  GemmArgs& a = pl.l1;
  a = GemmArgs{};
  a.k_stages = x_row_bytes(fmt, H) / 128;
  a.n_tiles = I / 128;
  a.n_group = a.n_tiles;   // expert-major
  a.wB = static_cast<const uint8_t*>(w->w13);
  a.I = I;
  a.H = H;
  a.topk = k;
  a.clamp = p->activation_clamp;
  a.fast_math = p->fast_math;
  const bool oai = p->activation == MOE_ACT_SWIGLUOAI;
  a.act_a = oai ? p->activation_alpha : 1.0f;
  a.act_b = oai ? 1.0f : 0.0f;
  a.expert_ids = b.expert_ids;
  a.num_active = b.num_active;
  a.starts = b.starts;
  a.a_scale_offsets = b.a_scale_offsets;
  a.tile_offsets = pl.swap ? b.tiles32 : b.tile_offsets;
  a.tile_rows = tile_rows;
  if (direct_l1) {
    a.x_rows = static_cast<const uint8_t*>(act->x);
    a.x_row_bytes = x_row_bytes(fmt, H);
    a.x_sc = static_cast<const float*>(act->x_scale);   // FP8; null for BF16
    a.x_sc_ld = H / 128;
    if (fmt == FMT_NVFP4 || fmt == FMT_MXFP8) {
      a.x_sf_rows = static_cast<const uint8_t*>(act->x_scale);
      a.x_sf_ld = fmt == FMT_NVFP4 ? H / 16 : H / 32;
    }
  }
  a.src_info = b.src_info;
  a.topk_weights = topk_weights;
  a.sfa = b.x_sf;
  a.sfa_kc = fmt == FMT_MXFP8 ? H / 128 : H / 64;   // scale tiles per 128-row block
  a.sa_t = reinterpret_cast<const float*>(b.x_sf);
  a.sa_ld = int(b.P);
  a.sb = static_cast<const float*>(w->w13_scale);
  a.sb_nb = 2 * I / 128;
  a.sb_kb = H / 128;
  // per-expert output scaling: NVFP4's products, or FP8 per-tensor's weight
  // scales times the activation scale (L1) / the re-quant scale (L2)
  const bool per_tensor = fmt == FMT_FP8T;
  a.alpha = per_tensor ? static_cast<const float*>(w->w13_scale) : w->gate_up_expert_scales;
  a.alpha_scalar = per_tensor ? static_cast<const float*>(act->x_scale) : nullptr;
  a.alpha_e2 = nullptr;
  a.x_row_scale = static_cast<const uint16_t*>(act->x_rowwise_scale);
  a.c_in = w->c_input_scales;
  a.h_out = b.h;
  a.h_row_bytes = h_row_bytes(fmt, I);
  a.h_sf = b.h_sf;
  a.h_sf_kc = fmt == FMT_MXFP8 ? I / 128 : I / 64;
  a.h_scale_t = reinterpret_cast<float*>(b.h_sf);
  a.h_scale_ld = int(b.P);
  a.status = b.status;
  const int64_t mtiles_bound = (R + tile_rows - 1) / tile_rows + std::min<int64_t>(E, R);
  pl.grid1 = std::max(1, int(std::min<int64_t>(nsm, mtiles_bound * a.n_tiles)));

  // L2: down
  if (!make_map(&pl.ta2, b.h, h_row_bytes(fmt, I), uint64_t(R), uint32_t(tile_rows))) return MOE_ERR_CUDA;
  GemmArgs& a2 = pl.l2;
  a2 = a;
  a2.x_rows = nullptr;   // the down leg reads the intermediate through its TMA map
  a2.x_sc = nullptr;
  a2.x_sf_rows = nullptr;
  a2.x_row_scale = nullptr;
  a2.k_stages = h_row_bytes(fmt, I) / 128;
  a2.n_tiles = H / 256;
  // Output n tiles in groups: a group's slice of the FP32 accumulator
  // (M x 256*group floats) stays in L2 while its tiles add into it, and the
  // intermediate is read once per group.  While the intermediate itself fits
  // in L2 the re-reads are free and one n tile per group is best.
  // When it does not fit, FP8 (whose down leg is paced by the promotion of
  // its partial sums) stays expert-major -- on M = 16384, H = 4096, 16 n
  // tiles, groups of 2 to 6 were 4-8% slower -- while MXFP8, whose down leg
  // is paced by the reductions into the accumulator, runs groups of 4 (a
  // 64 MB slice; 9% faster than expert-major on the same problem).
  const size_t kL2Budget = size_t(48) << 20;
  const bool h_fits = size_t(R) * h_row_bytes(fmt, I) <= kL2Budget;
  a2.n_group = h_fits ? 1 : (fmt == FMT_MXFP8 ? std::min(a2.n_tiles, 4) : a2.n_tiles);
  a2.wB = static_cast<const uint8_t*>(w->w2);
  a2.sfa = b.h_sf;
  a2.sfa_kc = a.h_sf_kc;
  a2.sa_t = reinterpret_cast<const float*>(b.h_sf);
  a2.sb = static_cast<const float*>(w->w2_scale);
  a2.sb_nb = H / 128;
  a2.sb_kb = I / 128;
  a2.alpha = per_tensor ? static_cast<const float*>(w->w2_scale) : w->down_expert_scales;
  a2.alpha_scalar = nullptr;
  a2.alpha_e2 = per_tensor ? w->c_input_scales : nullptr;
  a2.out = out;
  pl.grid2 = std::max(1, int(std::min<int64_t>(nsm, mtiles_bound * a2.n_tiles)));
  return MOE_OK;
}

moe_status_t run_ffn(const moe_problem_t* p, const moe_act_t* act, const moe_weights_t* w,
                     const FfnBuffers& b, const float* topk_weights,
                     int out_mode, float* out, cudaStream_t st) {
  const int fmt = p->format;
  const int64_t M = p->num_tokens, R = M * p->num_topk, H = p->hidden;
  FfnPlan pl;
  moe_status_t s = plan_ffn(p, act, w, b, topk_weights, out, pl);
  if (s != MOE_OK) return s;
  if (!pl.g.skip_rows || pl.g.tiles32) {
    TimScope ts(MOE_SLOT_GATHER, st);
    // eight 256-thread blocks per SM: each warp copies a run of rows
    if (launch_k(gather_kernel, grid_for(R * 32, 256, sm_count() * 8), 256, 0, st, pl.g) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  {
    TimScope ts(MOE_SLOT_GEMM1, st);
    if (launch_gemm_fmt<EPI_L1>(fmt, pl.swap, pl.l1, pl.ta1, pl.grid1, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (out_mode == MOE_OUT_ACCUMULATE) {
    TimScope ts(MOE_SLOT_ZERO, st);
    if (launch_k(zero_kernel, grid_for(M * H / 4, 256), 256, 0, st, reinterpret_cast<float4*>(out),
                 int64_t(M * H / 4)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  TimScope ts2(MOE_SLOT_GEMM2, st);
  cudaError_t e = (out_mode == MOE_OUT_ACCUMULATE)
                      ? launch_gemm_fmt<EPI_L2_ACC>(fmt, pl.swap, pl.l2, pl.ta2, pl.grid2, st)
                      : launch_gemm_fmt<EPI_L2_STAGED>(fmt, pl.swap, pl.l2, pl.ta2, pl.grid2, st);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The single-launch layer: a cooperative launch of moe_fused_kernel<FMT>.
template <int FMT, bool SWAP>
cudaError_t launch_fused_fmt(const FusedArgs& f, const FfnPlan& pl, int grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(FusedShape<FMT, SWAP>::kThreads);
  cfg.dynamicSmemBytes = fused_smem_bytes<FMT, SWAP>();
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_fused_kernel<FMT, SWAP>, f, pl.ta1, pl.ta2);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

moe_status_t check_act_weights(const moe_problem_t* p, const moe_act_t* act, const moe_weights_t* w) {
  if (!act || !w || !act->x || !w->w13 || !w->w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(act->x) || !aligned16(w->w13) || !aligned16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (p->format != MOE_FMT_BF16 && !act->x_scale) return MOE_ERR_INVALID_ARG;
  // the scales are read a 4-byte word at a time (the small-M gate_up copies
  // a row's NVFP4 / MXFP8 scale words straight from x_scale)
  if ((reinterpret_cast<uintptr_t>(act->x_scale) & 3) != 0) return MOE_ERR_INVALID_ARG;
  if (p->format == MOE_FMT_FP8_E4M3_B128 && (!w->w13_scale || !w->w2_scale)) return MOE_ERR_INVALID_ARG;
  if (p->format == MOE_FMT_NVFP4 &&
      (!w->gate_up_expert_scales || !w->down_expert_scales || !w->c_input_scales))
    return MOE_ERR_INVALID_ARG;
  if (p->format == MOE_FMT_FP8_PER_TENSOR && (!w->w13_scale || !w->w2_scale || !w->c_input_scales))
    return MOE_ERR_INVALID_ARG;
  // rowwise activation scales exist for NVFP4 only
  if (act->x_rowwise_scale && p->format != MOE_FMT_NVFP4) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

bool layout_ok(const moe_layout_t* l) {
  return l && l->expert_counts && l->expert_start_indices && l->src_info && l->slot_to_row && l->expert_ids &&
         l->num_active && l->a_scale_offsets && l->tile_offsets;
}


// ------------------------------------------------------ allocation-free permute
// Scratch of moe_permute_noalloc, the entry point for callers that cannot
// allocate device memory (a host runtime without a device allocator, a
// serving loop that must not allocate per request): the per-chunk expert
// counts of the two-pass permutation live in this file-scope device array,
// which every GPU that loads the library holds until the process exits.
// kNoAllocCountEntries bounds chunks x experts.  Pass 1 rewrites every entry
// it covers, so no clearing is needed; concurrent calls race on the array.
constexpr int kNoAllocCountEntries = 32768;   // 128 KB
static __device__ __align__(256) int g_noalloc_counts[kNoAllocCountEntries];

// Device address of g_noalloc_counts per device, looked up with that device
// current (host code cannot use the symbol itself): once per device and
// primary context -- a cudaDeviceReset gives the device a new context, in
// which the array has a new address, so the lookup is repeated then.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn get_ctx_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

int* noalloc_counts_ptr() {
  static int* ptrs[64] = {nullptr};
  static CUcontext ctxs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  CtxGetCurrentFn get_ctx = get_ctx_fn();
  CUcontext ctx = nullptr;
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev] || !ctx || ctxs[dev] != ctx) {
    // (the lookup also makes the device's context current if no runtime
    // call of this thread has yet)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_counts) != cudaSuccess) return nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
    ctxs[dev] = ctx;
  }
  return ptrs[dev];
}

__global__ void set_int_kernel(int* p, int v) { *p = v; }

__global__ void set_hooks_kernel(int* hdr, int wait_limit_us, int skip_arrival) {
  hdr[kWsWaitLimitWord] = wait_limit_us;
  hdr[kWsSkipArrivalWord] = skip_arrival;
}

}  // namespace

// =============================================================== C ABI
extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_BAD_INDEX: return "MOE_ERR_BAD_INDEX";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status_t moe_init(int device) {
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
  const bool ok = ensure_init() && get_encode() != nullptr;
  cudaSetDevice(prev);
  return ok ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_get_workspace_offsets(const moe_problem_t* p, moe_workspace_offsets_t* o) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!o) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  o->status = L.header;
  o->topk_idx = L.route_idx;
  o->topk_weights = L.route_w;
  o->expert_counts = L.counts;
  o->expert_start_indices = L.starts;
  o->src_info = L.src_info;
  o->slot_to_row = L.slot_to_row;
  o->expert_ids = L.expert_ids;
  o->num_active = L.num_active;
  o->a_scale_offsets = L.a_scale_offsets;
  o->tile_offsets = L.tile_offsets;
  o->intermediate = L.h;
  o->intermediate_scales = L.h_sf;
  o->scale_rows = L.P;
  o->accumulator = L.acc;
  return MOE_OK;
}

moe_status_t moe_get_workspace_size(const moe_problem_t* p, size_t* bytes) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(p).total;
  return MOE_OK;
}

moe_status_t moe_get_tile_regime(const moe_problem_t* p, int32_t* regime) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!regime) return MOE_ERR_INVALID_ARG;
  *regime = small_m_tiles(p) ? MOE_TILE_SMALL_M : MOE_TILE_LARGE_M;
  return MOE_OK;
}

moe_status_t moe_get_intermediate_size(const moe_problem_t* p, size_t* bytes, size_t* scale_offset) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!bytes || !scale_offset) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  *scale_offset = align_up(std::max<size_t>(L.h_bytes, 1), kAlign);
  *bytes = *scale_offset + align_up(std::max<size_t>(L.h_sf_bytes, 1), kAlign);
  return MOE_OK;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < sizeof(WsHeader)) return MOE_ERR_INVALID_ARG;
  zero_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<float4*>(ws),
                                                               int64_t(sizeof(WsHeader) / 16));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_workspace_test_hooks(void* ws, size_t ws_bytes, int32_t wait_limit_us, int32_t skip_arrival,
                                      void* stream) {
  if (!ws || ws_bytes < sizeof(WsHeader) || wait_limit_us < 0 || (skip_arrival != 0 && skip_arrival != 1))
    return MOE_ERR_INVALID_ARG;
  set_hooks_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(ws), wait_limit_us,
                                                                    skip_arrival);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_get_prepared_weights_size(const moe_problem_t* p, size_t* w13_bytes, size_t* w2_bytes) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!w13_bytes || !w2_bytes) return MOE_ERR_INVALID_ARG;
  *w13_bytes = prepared_bytes(p, true);
  *w2_bytes = prepared_bytes(p, false);
  return MOE_OK;
}

moe_status_t moe_prepare_weights(const moe_problem_t* p, const moe_weights_t* logical, void* out_w13,
                                 void* out_w2, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (!logical || !logical->w13 || !logical->w2 || !out_w13 || !out_w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(logical->w13) || !aligned16(logical->w2) || !aligned16(out_w13) || !aligned16(out_w2))
    return MOE_ERR_INVALID_ARG;
  if ((p->format == MOE_FMT_NVFP4 || p->format == MOE_FMT_MXFP8) && (!logical->w13_scale || !logical->w2_scale))
    return MOE_ERR_INVALID_ARG;
  if (!ensure_init()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int fmt = p->format, E = p->num_experts, H = p->hidden, I = p->intermediate_hidden;
  PrepArgs a{};
  a.fmt = fmt;
  a.E = E;
  // gate_up: 2I rows, K = H
  a.w = static_cast<const uint8_t*>(logical->w13);
  a.sf = static_cast<const uint8_t*>(logical->w13_scale);
  a.out = static_cast<uint8_t*>(out_w13);
  a.N = 2 * I;
  a.Kb = x_row_bytes(fmt, H);
  a.ksf = fmt == FMT_MXFP8 ? H / 32 : H / 16;
  a.n_tiles = I / 128;
  a.k_stages = a.Kb / 128;
  a.l1 = 1;
  if (launch_k(prepare_weights_kernel, grid_for(int64_t(prepared_bytes(p, true)) / 16, 256), 256, 0, st, a) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  // down: H rows, K = I
  a.w = static_cast<const uint8_t*>(logical->w2);
  a.sf = static_cast<const uint8_t*>(logical->w2_scale);
  a.out = static_cast<uint8_t*>(out_w2);
  a.N = H;
  a.Kb = h_row_bytes(fmt, I);
  a.ksf = fmt == FMT_MXFP8 ? I / 32 : I / 16;
  a.n_tiles = H / 256;
  a.k_stages = a.Kb / 128;
  a.l1 = 0;
  return launch_k(prepare_weights_kernel, grid_for(int64_t(prepared_bytes(p, false)) / 16, 256), 256, 0, st, a) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_route(const moe_problem_t* p, const float* logits, const float* bias, int64_t* topk_idx,
                       float* topk_weights, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  if (p->num_topk > 32) return MOE_ERR_UNSUPPORTED;
  if (p->num_tokens == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_weights) return MOE_ERR_INVALID_ARG;
  return launch_route(route_args(p, logits, bias, topk_idx, topk_weights), static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_quantize_nvfp4_rowwise(const moe_problem_t* p, const void* x_bf16, void* codes, void* block_scales,
                                        void* rowwise_scales, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  if (p->num_tokens == 0) return MOE_OK;
  if (!x_bf16 || !codes || !block_scales || !rowwise_scales || !aligned16(x_bf16) || !aligned16(codes))
    return MOE_ERR_INVALID_ARG;
  QuantRowArgs a{};
  a.x = static_cast<const uint16_t*>(x_bf16);
  a.M = p->num_tokens;
  a.H = p->hidden;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = static_cast<uint8_t*>(block_scales);
  a.rowwise = static_cast<uint16_t*>(rowwise_scales);
  return launch_k(quantize_rowwise_kernel, grid_for(a.M * 32, 256, sm_count() * 16), 256, 0,
                  static_cast<cudaStream_t>(stream), a) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_permute(const moe_problem_t* p, const int64_t* topk_idx, const moe_layout_t* layout, void* ws,
                         size_t ws_bytes, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (p->num_tokens == 0) return MOE_OK;
  if (!topk_idx || !layout_ok(layout) || !ws) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  PermOut o{layout->expert_counts, layout->expert_start_indices, layout->src_info, layout->slot_to_row,
            layout->expert_ids,    layout->num_active,           layout->a_scale_offsets, layout->tile_offsets};
  return launch_permute(perm_args(p, topk_idx, o, reinterpret_cast<int*>(base + L.block_counts), L.nblk,
                                  reinterpret_cast<int*>(base + L.header)),
                        static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_ffn(const moe_problem_t* p, const moe_act_t* act, const moe_weights_t* w,
                     const moe_layout_t* layout, const float* topk_weights, int32_t out_mode, void* out,
                     void* intermediate, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (out_mode != MOE_OUT_ACCUMULATE && out_mode != MOE_OUT_STAGED) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens == 0) return MOE_OK;
  if ((s = check_act_weights(p, act, w)) != MOE_OK) return s;
  if (!layout_ok(layout) || !out || !ws || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (out_mode == MOE_OUT_ACCUMULATE && !topk_weights) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!ensure_init()) return MOE_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(ws);
  FfnBuffers b{};
  b.counts = layout->expert_counts;
  b.starts = layout->expert_start_indices;
  b.src_info = layout->src_info;
  b.slot_to_row = layout->slot_to_row;
  b.expert_ids = layout->expert_ids;
  b.num_active = layout->num_active;
  b.a_scale_offsets = layout->a_scale_offsets;
  b.tile_offsets = layout->tile_offsets;
  b.x_perm = base + L.x_perm;
  b.x_sf = base + L.x_sf;
  size_t so = 0, isz = 0;
  moe_get_intermediate_size(p, &isz, &so);
  b.h = intermediate ? static_cast<uint8_t*>(intermediate) : base + L.h;
  b.h_sf = intermediate ? static_cast<uint8_t*>(intermediate) + so : base + L.h_sf;
  b.tiles32 = reinterpret_cast<int*>(base + L.tiles32);
  b.P = L.P;
  b.status = reinterpret_cast<int*>(base + L.header);
  return run_ffn(p, act, w, b, topk_weights, out_mode, static_cast<float*>(out),
                 static_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine(const moe_problem_t* p, const moe_layout_t* layout, const float* topk_weights,
                         const void* in, int32_t in_mode, void* out_bf16, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (in_mode != MOE_IN_ACCUMULATED && in_mode != MOE_IN_STAGED) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens == 0) return MOE_OK;
  if (!in || !out_bf16 || !aligned16(in) || !aligned16(out_bf16)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t M = p->num_tokens, H = p->hidden;
  TimScope ts(in_mode == MOE_IN_ACCUMULATED ? MOE_SLOT_FINALIZE : MOE_SLOT_COMBINE, st);
  cudaError_t e;
  if (in_mode == MOE_IN_ACCUMULATED) {
    e = launch_k(finalize_kernel, grid_for(M * H / 8, 256), 256, 0, st, static_cast<const float4*>(in),
                 static_cast<uint4*>(out_bf16), int64_t(M * H / 8));
  } else {
    if (!layout || !layout->slot_to_row || !topk_weights) return MOE_ERR_INVALID_ARG;
    e = launch_k(combine_staged_kernel, grid_for(M * H / 8, 256), 256, 0, st, static_cast<const float*>(in),
                 static_cast<const int*>(layout->slot_to_row), topk_weights, M, int(H), p->num_topk,
                 static_cast<uint4*>(out_bf16));
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_fused(const moe_problem_t* p, const moe_act_t* act, const moe_weights_t* w,
                       const int64_t* topk_idx, const float* topk_weights, const float* logits,
                       const float* bias, void* out_bf16, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  // the routing chooses among the routed experts; every later step works on
  // the effective problem (a shared expert is one more expert and slot)
  const moe_problem_t* p_route = p;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (p->num_tokens == 0) return MOE_OK;
  if ((s = check_act_weights(p, act, w)) != MOE_OK) return s;
  const bool pre = topk_idx != nullptr && topk_weights != nullptr;
  const bool from_logits = logits != nullptr;
  if (pre == from_logits || (!pre && (topk_idx || topk_weights))) return MOE_ERR_INVALID_ARG;
  if (from_logits && p_route->num_topk > 32) return MOE_ERR_UNSUPPORTED;
  if (!out_bf16 || !aligned16(out_bf16) || !ws) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!ensure_init()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base + L.header);
  FusedArgs f{};
  const int64_t* idx = topk_idx;
  const float* wts = topk_weights;
  if (from_logits) {
    int64_t* ridx = reinterpret_cast<int64_t*>(base + L.route_idx);
    float* rw = reinterpret_cast<float*>(base + L.route_w);
    f.route = route_args(p_route, logits, bias, ridx, rw);
    f.do_route = 1;
    idx = ridx;
    wts = rw;
  }
  PermOut o{reinterpret_cast<int*>(base + L.counts),     reinterpret_cast<int*>(base + L.starts),
            reinterpret_cast<int*>(base + L.src_info),   reinterpret_cast<int*>(base + L.slot_to_row),
            reinterpret_cast<int*>(base + L.expert_ids), reinterpret_cast<int*>(base + L.num_active),
            reinterpret_cast<int*>(base + L.a_scale_offsets), reinterpret_cast<int*>(base + L.tile_offsets)};
  // small-M tiles: the permutation also writes their tile table, and as the
  // GEMMs read the routed rows of x themselves there is no gather phase
  const bool small_m = small_m_tiles(p);
  if (small_m) o.tiles32 = reinterpret_cast<int*>(base + L.tiles32);
  // no gather phase when the gate_up GEMM reads x itself (small-M tiles)
  f.gather_phase = small_m ? 0 : 1;
  f.perm = perm_args(p, idx, o, reinterpret_cast<int*>(base + L.block_counts), L.nblk, status);
  f.perm_small = perm_small_case(f.perm.R, f.perm.E) ? 1 : 0;
  FfnBuffers b{};
  b.counts = o.expert_counts;
  b.starts = o.expert_start_indices;
  b.src_info = o.src_info;
  b.slot_to_row = o.slot_to_row;
  b.expert_ids = o.expert_ids;
  b.num_active = o.num_active;
  b.a_scale_offsets = o.a_scale_offsets;
  b.tile_offsets = o.tile_offsets;
  b.x_perm = base + L.x_perm;
  b.x_sf = base + L.x_sf;
  b.h = base + L.h;
  b.h_sf = base + L.h_sf;
  b.tiles32 = reinterpret_cast<int*>(base + L.tiles32);
  b.P = L.P;
  b.status = status;
  float* acc = reinterpret_cast<float*>(base + L.acc);
  FfnPlan pl;
  if ((s = plan_ffn(p, act, w, b, wts, acc, pl)) != MOE_OK) return s;
  const int64_t M = p->num_tokens, H = p->hidden;
  f.gather = pl.g;
  f.acc = reinterpret_cast<float4*>(acc);
  f.acc_n4 = M * H / 4;
  f.out = static_cast<uint4*>(out_bf16);
  f.out_n8 = M * H / 8;
  f.l1 = pl.l1;
  f.l2 = pl.l2;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base + L.header);
  f.gbar = hdr->grid_bar;
  f.status = status;
  f.phase_ns = hdr->phase_ns;
  const int grid = sm_count();
  TimScope ts(MOE_SLOT_FUSED, st);
  cudaError_t e;
  switch (p->format) {
    case FMT_BF16:
      e = pl.swap ? launch_fused_fmt<FMT_BF16, true>(f, pl, grid, st) : launch_fused_fmt<FMT_BF16, false>(f, pl, grid, st);
      break;
    case FMT_FP8:
      e = pl.swap ? launch_fused_fmt<FMT_FP8, true>(f, pl, grid, st) : launch_fused_fmt<FMT_FP8, false>(f, pl, grid, st);
      break;
    case FMT_MXFP8:
      e = pl.swap ? launch_fused_fmt<FMT_MXFP8, true>(f, pl, grid, st) : launch_fused_fmt<FMT_MXFP8, false>(f, pl, grid, st);
      break;
    case FMT_FP8T:
      e = pl.swap ? launch_fused_fmt<FMT_FP8T, true>(f, pl, grid, st) : launch_fused_fmt<FMT_FP8T, false>(f, pl, grid, st);
      break;
    default:
      e = pl.swap ? launch_fused_fmt<FMT_NVFP4, true>(f, pl, grid, st) : launch_fused_fmt<FMT_NVFP4, false>(f, pl, grid, st);
      break;
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_permute_noalloc(const moe_problem_t* p, const int64_t* topk_idx, const moe_layout_t* layout,
                                 int32_t* device_status, void* stream) {
  moe_status_t s = check_problem(p);
  if (s != MOE_OK) return s;
  const moe_problem_t pe = effective(p);
  p = &pe;
  if (p->num_tokens == 0) return MOE_OK;
  if (!topk_idx || !layout_ok(layout) || !device_status) return MOE_ERR_INVALID_ARG;
  const int64_t R = p->num_tokens * p->num_topk;
  const int E = p->num_experts;
  const int64_t nblk = (R + kPermChunk - 1) / kPermChunk;
  const bool small = perm_small_case(R, E);
  if (!small && nblk * E > kNoAllocCountEntries) return MOE_ERR_UNSUPPORTED;
  int* counts = small ? nullptr : noalloc_counts_ptr();
  if (!small && !counts) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word must start at zero; the counts are fully rewritten by pass 1
  set_int_kernel<<<1, 1, 0, st>>>(device_status, MOE_OK);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  PermOut o{layout->expert_counts, layout->expert_start_indices, layout->src_info, layout->slot_to_row,
            layout->expert_ids,    layout->num_active,           layout->a_scale_offsets, layout->tile_offsets};
  return launch_permute(perm_args(p, topk_idx, o, counts, int(nblk), device_status), st) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status_t moe_timing_enable(int enable, int max_calls) {
  std::lock_guard<std::mutex> lk(g_tim.mu);
  if (!enable) {
    g_tim.on = false;
    return MOE_OK;
  }
  if (max_calls < 1) return MOE_ERR_INVALID_ARG;
  if (!g_tim.ev || g_tim.cap < max_calls) {
    if (g_tim.ev) {
      for (int i = 0; i < MOE_NUM_SLOTS * g_tim.cap * 2; ++i) cudaEventDestroy(g_tim.ev[i]);
      delete[] g_tim.ev;
      g_tim.ev = nullptr;
    }
    g_tim.ev = new cudaEvent_t[size_t(MOE_NUM_SLOTS) * max_calls * 2];
    for (int i = 0; i < MOE_NUM_SLOTS * max_calls * 2; ++i)
      if (cudaEventCreate(&g_tim.ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
    g_tim.cap = max_calls;
  }
  for (int s = 0; s < MOE_NUM_SLOTS; ++s) g_tim.used[s] = 0;
  g_tim.on = true;
  return MOE_OK;
}

moe_status_t moe_timing_read(float* ms, int* launches) {
  if (!ms || !launches) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_tim.mu);
  for (int s = 0; s < MOE_NUM_SLOTS; ++s) {
    ms[s] = 0.0f;
    launches[s] = g_tim.used[s];
    for (int i = 0; i < g_tim.used[s]; ++i) {
      cudaEvent_t a = g_tim.ev[(size_t(s) * g_tim.cap + i) * 2];
      cudaEvent_t b = g_tim.ev[(size_t(s) * g_tim.cap + i) * 2 + 1];
      if (cudaEventSynchronize(b) != cudaSuccess) return MOE_ERR_CUDA;
      float t = 0.0f;
      if (cudaEventElapsedTime(&t, a, b) != cudaSuccess) return MOE_ERR_CUDA;
      ms[s] += t;
    }
    g_tim.used[s] = 0;
  }
  return MOE_OK;
}

moe_status_t moe_read_status(const void* ws, void* stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status_t>(v);
}

}  // extern "C"

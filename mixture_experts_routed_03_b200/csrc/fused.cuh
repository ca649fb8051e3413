// fused.cuh -- the whole routed-MoE layer in one launch.
//
// A cooperative, persistent kernel (one CTA per SM, all resident) runs the
// steps of the layer as phases separated by grid-wide barriers (the GEMM
// phases use the large-M tiles, or with SWAP the small-M swapped-operand
// tiles):
//
//   route (when routing from logits)  ->  permute (one block, or two passes
//   over 1024-slot chunks)  ->  gather into expert order  ->  gate_up GEMM
//   with the clamped-SwiGLU + re-quant epilogue, then zero the FP32
//   accumulator  ->  down GEMM with the router-weighted scatter-reduce
//   epilogue  ->  BF16 finalise
//
// (EPConfig, fused_moe_ready: dispatch, FFN and combine as one launch; the
// expert-parallel exchange of that op is out of scope here.)  Every phase is
// the same device code the unfused entry points launch one kernel each for.
// The grid barrier counts arrivals and bumps a generation word in the
// workspace; a wait that exceeds the bound records MOE_ERR_TIMEOUT, raises
// the CTA's abort flag and the remaining phases are skipped.  Generic-proxy
// writes that a later phase reads through TMA are fenced with
// fence.proxy.async before and after each barrier.
#pragma once

#include "aux_kernels.cuh"
#include "gemm.cuh"
#include "gemm_swap.cuh"

namespace moe {

struct FusedArgs {
  RouteArgs route;
  int do_route;
  PermArgs perm;
  int perm_small;
  int gather_phase;     // 0: the small-M GEMMs read x themselves and the permute built their tile table
  GatherArgs gather;
  float4* acc;
  int64_t acc_n4;
  uint4* out;
  int64_t out_n8;
  GemmArgs l1, l2;
  int* gbar;            // [2]: arrivals, generation (workspace header)
  int* status;
  unsigned long long* phase_ns;  // [8]: %globaltimer at each phase boundary (CTA 0)
};

// Grid-wide barrier for a cooperative launch; returns false after an abort.
// (Test hook: with the header's skip_arrival set, CTA 0 withholds its
// arrival once -- clearing the flag -- so the others' wait runs out.)
__device__ bool grid_barrier(int* gbar, volatile int* abort_flag, int* status) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* gen = gbar + 1;
    const int g = *gen;
    __threadfence();
    const bool skip = blockIdx.x == 0 && atomicExch(status + kWsSkipArrivalWord, 0) == 1;
    const unsigned long long limit = limit_ns_of(abort_flag[1]);
    if (!skip && atomicAdd(gbar, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(gbar, 0);
      __threadfence();
      atomicAdd(gbar + 1, 1);
    } else {
      const unsigned long long t0 = globaltimer_ns();
      while (*gen == g) {
        if (*abort_flag) break;
        if (globaltimer_ns() - t0 > limit) {
          *abort_flag = 1;
          if (atomicCAS(status, 0, MOE_ERR_TIMEOUT) == 0) status[1] = 100;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
  }
  __syncthreads();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return *abort_flag == 0;
}

// Indices of the calling thread for the grid-stride steps (recomputed per
// phase so nothing but the abort flag stays live across the GEMM phases).
struct GridIdx {
  int64_t gw, tw, gt, tt;
  int lane;
};
__device__ __forceinline__ GridIdx grid_idx() {
  GridIdx g;
  const int64_t nw = blockDim.x >> 5;
  g.gw = static_cast<int64_t>(blockIdx.x) * nw + (threadIdx.x >> 5);
  g.tw = static_cast<int64_t>(gridDim.x) * nw;
  g.gt = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  g.tt = static_cast<int64_t>(gridDim.x) * blockDim.x;
  g.lane = threadIdx.x & 31;
  return g;
}

__device__ __forceinline__ void stamp(const FusedArgs& f, int i) {
  if (blockIdx.x == 0 && threadIdx.x == 0) f.phase_ns[i] = globaltimer_ns();
}

// Block shape of the single launch: that of its GEMM phases (large-M tiles,
// or the swapped-operand small-M tiles).
template <int FMT, bool SWAP>
struct FusedShape {
  static constexpr int kThreads = GemmCfg<FMT, EPI_L1>::kThreads;
  static constexpr int kHeaderBytes = GemmCfg<FMT, EPI_L1>::kHeaderBytes;
  static constexpr int kSmemBytes = GemmCfg<FMT, EPI_L1>::kSmemBytes > GemmCfg<FMT, EPI_L2_ACC>::kSmemBytes
                                        ? GemmCfg<FMT, EPI_L1>::kSmemBytes
                                        : GemmCfg<FMT, EPI_L2_ACC>::kSmemBytes;
  static_assert(GemmCfg<FMT, EPI_L1>::kThreads == GemmCfg<FMT, EPI_L2_ACC>::kThreads, "one block shape");
};
template <int FMT>
struct FusedShape<FMT, true> {
  static constexpr int kThreads = SwapCfg<FMT, EPI_L1>::kThreads;
  static constexpr int kHeaderBytes = SwapCfg<FMT, EPI_L1>::kHeaderBytes;
  static constexpr int kSmemBytes = SwapCfg<FMT, EPI_L1>::kSmemBytes > SwapCfg<FMT, EPI_L2_ACC>::kSmemBytes
                                        ? SwapCfg<FMT, EPI_L1>::kSmemBytes
                                        : SwapCfg<FMT, EPI_L2_ACC>::kSmemBytes;
  static_assert(SwapCfg<FMT, EPI_L1>::kThreads == SwapCfg<FMT, EPI_L2_ACC>::kThreads, "one block shape");
};

template <int FMT, bool SWAP>
__global__ void __launch_bounds__(FusedShape<FMT, SWAP>::kThreads, 1)
    moe_fused_kernel(const __grid_constant__ FusedArgs f, const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ CUtensorMap tmA2) {
  constexpr int kHdr = FusedShape<FMT, SWAP>::kHeaderBytes;
  SmemHeader* hdr = reinterpret_cast<SmemHeader*>(smem_base_1024());
  if (threadIdx.x == 0) {
    hdr->abort = 0;
    hdr->wait_us = wait_limit_us(f.status);
  }
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&hdr->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  stamp(f, 0);
  bool ok = true;
  if (f.do_route) {
    const GridIdx g = grid_idx();
    route_tokens(f.route, g.gw, g.tw, g.lane);
    ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  }
  stamp(f, 1);
  if (ok) {
    int* sm_int = reinterpret_cast<int*>(smem_base_1024() + kHdr);
    if (f.perm_small) {
      if (blockIdx.x == 0) perm_small_block(f.perm, sm_int);
    } else {
      for (int c = blockIdx.x; c < f.perm.nblk; c += gridDim.x) perm_count_chunk(f.perm, c, sm_int);
      ok = grid_barrier(f.gbar, &hdr->abort, f.status);
      if (ok)
        for (int c = blockIdx.x; c < f.perm.nblk; c += gridDim.x) perm_scatter_chunk(f.perm, c, sm_int);
    }
  }
  if (ok) ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  stamp(f, 2);
  if (ok && f.gather_phase) {
    if (f.gather.tiles32 && blockIdx.x == 0 && threadIdx.x < 32) small_tile_table(f.gather, threadIdx.x);
    if (!f.gather.skip_rows) {
      const GridIdx g = grid_idx();
      gather_rows(f.gather, g.gw, g.tw, g.lane);
    }
    ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  }
  stamp(f, 3);
  if (ok) {
    if constexpr (SWAP)
      gemm_phase_swap<FMT, EPI_L1>(f.l1, &tmA1, smem_base_1024() + kHdr, hdr->tmem, &hdr->abort, blockIdx.x,
                                   gridDim.x);
    else
      gemm_phase<FMT, EPI_L1>(f.l1, &tmA1, smem_base_1024() + kHdr, hdr->tmem, &hdr->abort, blockIdx.x, gridDim.x);
    // the accumulator is zeroed last, just before the down GEMM adds into it
    const GridIdx g = grid_idx();
    zero_range(f.acc, f.acc_n4, g.gt, g.tt);
    ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  }
  stamp(f, 4);
  if (ok) {
    if constexpr (SWAP)
      gemm_phase_swap<FMT, EPI_L2_ACC>(f.l2, &tmA2, smem_base_1024() + kHdr, hdr->tmem, &hdr->abort, blockIdx.x,
                                       gridDim.x);
    else
      gemm_phase<FMT, EPI_L2_ACC>(f.l2, &tmA2, smem_base_1024() + kHdr, hdr->tmem, &hdr->abort, blockIdx.x,
                                  gridDim.x);
    ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  }
  stamp(f, 5);
  if (ok) {
    const GridIdx g = grid_idx();
    finalize_range(f.acc, f.out, f.out_n8, g.gt, g.tt);
    ok = grid_barrier(f.gbar, &hdr->abort, f.status);
  }
  stamp(f, 6);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(hdr->tmem, kTmemCols);
}

template <int FMT, bool SWAP>
__host__ __device__ constexpr int fused_smem_bytes() {
  return FusedShape<FMT, SWAP>::kSmemBytes;
}

}  // namespace moe

// mma_peak.cu -- dense tensor-core throughput of this GPU, for the roofline.
//
// A measurement tool, not part of the layer: every CTA keeps one operand
// stage resident in shared memory and one thread issues tcgen05.mma back to
// back into one TMEM accumulator, the way the grouped GEMMs issue their K
// steps, so the achieved rate is the tensor pipe's own, with no memory
// traffic.  Shapes: M = 128 per CTA (cta_group::1) or M = 256 per CTA pair
// (cta_group::2, each CTA holding its 128 rows of A and half of B's N rows),
// N = 128 or 256, K = one 32-byte step per instruction (BF16 K = 16, E4M3
// K = 32, block-scaled E2M1 K = 64).  Operands are zero, so no value can
// slow the pipe down.  Every wait is bounded (status 6 on a time-out).
//
// extern "C" moe_peak_mma(kind, n, pair, iters, scratch, stream, *tflops, *cycles)
//   kind   0 BF16 (kind::f16), 1 E4M3 (kind::f8f6f4), 2 NVFP4
//          (kind::mxf4nvf4.block_scale.scale_vec::4X; cta_group::1 only),
//          3 MXFP8 (kind::mxf8f6f4.block_scale.scale_vec::1X; cta_group::1 only)
//   iters  K blocks of 4 instructions each CTA (or pair) issues
//   scratch device buffer of at least 16 bytes x grid (status, cycles)
// Returns 0 on success; *tflops = dense FLOPs / event time over the whole
// grid (one CTA per SM), *cycles = SM cycles per instruction of one CTA.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace {

using namespace moe;

constexpr int kPeakThreads = 128;
constexpr int kOffA = 0;            // 128 rows x 128 bytes
constexpr int kOffB = 16384;        // up to 256 rows x 128 bytes
constexpr int kOffSF = 49152;       // NVFP4: 12 scale tiles of 512 bytes
constexpr int kOffBar = 55296;
constexpr int kPeakSmem = 56320 + 1024;

__device__ __forceinline__ void mma_f16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(1u)
      : "memory");
}

__device__ __forceinline__ void mma_f8_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(1u)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int KIND, int N, bool PAIR>
__global__ void __launch_bounds__(kPeakThreads, 1) mma_peak_kernel(int iters, int* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* done = reinterpret_cast<uint64_t*>(base + kOffBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(base + kOffBar + 64);
  int* status = reinterpret_cast<int*>(base + kOffBar + 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool leader = !PAIR || cluster_rank() == 0;

  for (int i = threadIdx.x; i < kOffBar / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *status = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                   "r"(512)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      tmem_alloc(tslot, 512);
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  long long t0 = 0, t1 = 0;
  if (leader && warp == 1 && lane == 0) {
    if (KIND == 2) {
      // scale factors of 4 K steps for A (16 columns) and B (32 columns),
      // issued by this thread ahead of its MMAs
      for (int t = 0; t < 12; ++t)
        tmem_copy_sf(tmem + 256 + 4 * t, sdesc_sf_tile(smem_u32(base + kOffSF + 512 * t)));
    } else if (KIND == 3) {
      // one scale tile for A (4 columns) and two for B's 256 rows, which
      // serve all four K steps (byte kc of each word)
      for (int t = 0; t < 3; ++t)
        tmem_copy_sf(tmem + 256 + (t ? 12 + 4 * t : 0), sdesc_sf_tile(smem_u32(base + kOffSF + 512 * t)));
    }
    constexpr uint32_t M = PAIR ? 256 : 128;
    constexpr uint32_t idesc_m = (M >> 4) << 24;
    const uint32_t idesc = (KIND == 0)   ? ((idesc_dense(1, 1, N) & ~(31u << 24)) | idesc_m)
                           : (KIND == 1) ? ((idesc_dense(0, 0, N) & ~(31u << 24)) | idesc_m)
                                         : idesc_nvf4(N);   // (KIND 3 builds its own per K step)
    const uint64_t adesc = sdesc_sw128(smem_u32(base + kOffA));
    const uint64_t bdesc = sdesc_sw128(smem_u32(base + kOffB));
    t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        const uint64_t a = adesc + static_cast<uint64_t>(2 * kc);
        const uint64_t b = bdesc + static_cast<uint64_t>(2 * kc);
        if (KIND == 0) {
          if (PAIR) mma_f16_pair(tmem, a, b, idesc); else mma_f16(tmem, a, b, idesc, 1u);
        } else if (KIND == 1) {
          if (PAIR) mma_f8_pair(tmem, a, b, idesc); else mma_f8(tmem, a, b, idesc, 1u);
        } else if (KIND == 2) {
          mma_nvf4(tmem, a, b, idesc, tmem + 256 + 4 * kc, tmem + 256 + 16 + 8 * kc, 1u);
        } else {
          mma_mxf8(tmem, a, b, idesc_mxf8(N, kc), tmem + 256, tmem + 256 + 16, 1u);
        }
      }
    }
    if (PAIR) {
      asm volatile(
          "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
          "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
              smem_u32(done))
          : "memory");
    } else {
      mma_commit(done);
    }
  }
  // every thread waits for the MMAs to finish (bounded)
  {
    const unsigned long long g0 = globaltimer_ns();
    while (!mbar_test(done, 0)) {
      if (globaltimer_ns() - g0 > kWaitLimitNs) {
        *status = MOE_ERR_TIMEOUT;
        break;
      }
    }
  }
  if (leader && warp == 1 && lane == 0) {
    t1 = clock64();
    out[4 * blockIdx.x + 0] = *status;
    reinterpret_cast<long long*>(out)[2 * blockIdx.x + 1] = t1 - t0;
  } else if (!leader && threadIdx.x == 0) {
    out[4 * blockIdx.x + 0] = *status;
    reinterpret_cast<long long*>(out)[2 * blockIdx.x + 1] = 0;
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    else
      tmem_dealloc(tmem, 512);
  }
}

template <int KIND, int N, bool PAIR>
int run_peak(int iters, int* scratch, cudaStream_t st, float* tflops, float* cycles) {
  auto kern = mma_peak_kernel<KIND, N, PAIR>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPeakSmem) != cudaSuccess) return 4;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kPeakThreads);
  cfg.dynamicSmemBytes = kPeakSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int grid = nsm;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) return 4;
    grid = 2 * clusters;
  }
  cfg.gridDim = dim3(grid);
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  // one short warm-up launch, then the timed one
  if (cudaLaunchKernelEx(&cfg, kern, 64, scratch) != cudaSuccess) return 4;
  cudaEventRecord(e0, st);
  if (cudaLaunchKernelEx(&cfg, kern, iters, scratch) != cudaSuccess) return 4;
  cudaEventRecord(e1, st);
  if (cudaEventSynchronize(e1) != cudaSuccess) return 4;
  float ms = 0.0f;
  cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  int* host = new int[4 * grid];
  cudaMemcpy(host, scratch, sizeof(int) * 4 * grid, cudaMemcpyDeviceToHost);
  int status = 0;
  double cyc = 0.0;
  int n = 0;
  for (int b = 0; b < grid; ++b) {
    if (host[4 * b]) status = host[4 * b];
    const long long c = reinterpret_cast<long long*>(host)[2 * b + 1];
    if (c > 0) {
      cyc += static_cast<double>(c);
      ++n;
    }
  }
  delete[] host;
  const double k = (KIND == 0) ? 16.0 : (KIND == 2 ? 64.0 : 32.0);
  const double m = PAIR ? 256.0 : 128.0;
  const double issuers = PAIR ? grid / 2 : grid;
  const double flops = 2.0 * m * N * k * 4.0 * iters * issuers;
  *tflops = static_cast<float>(flops / (ms * 1e-3) / 1e12);
  *cycles = n ? static_cast<float>(cyc / n / (4.0 * iters)) : 0.0f;
  return status;
}

// ---------------------------------------------------------------------------
// Main-loop probe: the grouped GEMMs' operand feed without their epilogue.
// Each CTA streams K blocks of A (128 rows x 128 bytes) and B (256 weight
// rows x 128 bytes, or its 128-row half in a CTA pair) from an L2-resident
// source by bulk copies into a 4-stage ring, and (mma = 1) issues the E4M3
// MMAs of each block (M128 x N256 per CTA, or M256 x N256 per pair), or
// (mma = 0) releases each stage as soon as it lands.  In a pair, the second
// CTA's stages are relayed to the first CTA's MMA thread by a remote
// mbarrier arrive, and the MMA's commit releases the stage in both CTAs.
// ---------------------------------------------------------------------------
constexpr int kLoopStages = 4;

__device__ __forceinline__ uint32_t mapa_rank0(uint32_t saddr) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(saddr));
  return r;
}

__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_test_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; on a time-out sets *status and returns false.
__device__ __forceinline__ bool probe_wait(uint64_t* bar, uint32_t parity, int* status, bool cluster_scope) {
  const unsigned long long g0 = globaltimer_ns();
  while (!(cluster_scope ? mbar_test_cluster(bar, parity) : mbar_test(bar, parity))) {
    if (*status) return false;
    if (globaltimer_ns() - g0 > kWaitLimitNs) {
      *status = MOE_ERR_TIMEOUT;
      return false;
    }
  }
  return true;
}

template <bool PAIR, bool MMA>
__global__ void __launch_bounds__(kPeakThreads, 1)
    mainloop_probe_kernel(int iters, const uint8_t* src, long long src_blocks, int* out) {
  constexpr int kA = 16384;
  constexpr int kB = PAIR ? 16384 : 32768;
  constexpr int kStage = kA + kB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kLoopStages * kStage);
  uint64_t* empty = full + kLoopStages;
  uint64_t* peer_full = empty + kLoopStages;
  uint64_t* done = peer_full + kLoopStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* status = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0;
  const bool leader = rank == 0;
  const int unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;   // CTA or pair index

  if (threadIdx.x == 0) {
    for (int i = 0; i < kLoopStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&peer_full[i], 1);
    }
    mbar_init(done, 1);
    *status = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (MMA && warp == 0) {
    if (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                   "r"(512)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      tmem_alloc(tslot, 512);
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = MMA ? *tslot : 0;

  long long t0 = 0, t1 = 0;
  if (warp == 0 && lane == 0) {
    // producer: block (unit, it) of this CTA's half comes from a spread-out,
    // L2-resident offset
    int stage = 0;
    uint32_t phase = 0;
    for (int it = 0; it < iters; ++it) {
      if (!probe_wait(&empty[stage], phase ^ 1u, status, false)) break;
      const long long blk = (static_cast<long long>(unit) * 7919 + it * 13 + rank * 5) % src_blocks;
      uint8_t* sa = base + stage * kStage;
      mbar_arrive_expect_tx(&full[stage], kStage);
      bulk_load(sa, src + blk * 49152, kA, &full[stage]);
      bulk_load(sa + kA, src + blk * 49152 + kA, kB, &full[stage]);
      if (++stage == kLoopStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // consumer: the MMAs of each stage (or an immediate release)
    constexpr uint32_t M = PAIR ? 256 : 128;
    const uint32_t idesc = (idesc_dense(0, 0, 256) & ~(31u << 24)) | ((M >> 4) << 24);
    int stage = 0;
    uint32_t phase = 0;
    t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if (!probe_wait(&full[stage], phase, status, false)) break;
      if (PAIR && !probe_wait(&peer_full[stage], phase, status, true)) break;
      tc_fence_after();
      uint8_t* sa = base + stage * kStage;
      if (MMA) {
        const uint64_t adesc = sdesc_sw128(smem_u32(sa));
        const uint64_t bdesc = sdesc_sw128(smem_u32(sa + kA));
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          if (PAIR) mma_f8_pair(tmem, adesc + 2 * kc, bdesc + 2 * kc, idesc);
          else mma_f8(tmem, adesc + 2 * kc, bdesc + 2 * kc, idesc, 1u);
        }
        if (PAIR) {
          asm volatile(
              "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
              "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
                  smem_u32(&empty[stage]))
              : "memory");
        } else {
          mma_commit(&empty[stage]);
        }
      } else {
        mbar_arrive(&empty[stage]);
        if (PAIR) {
          // the second CTA's stage too
          uint32_t r;
          asm volatile("mapa.shared::cluster.u32 %0, %1, 1;" : "=r"(r) : "r"(smem_u32(&empty[stage])));
          remote_arrive(r);
        }
      }
      if (++stage == kLoopStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    t1 = clock64();
    if (MMA) {
      if (PAIR) {
        asm volatile(
            "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
                smem_u32(done))
            : "memory");
      } else {
        mma_commit(done);
      }
    } else {
      mbar_arrive(done);
      if (PAIR) {
        uint32_t r;
        asm volatile("mapa.shared::cluster.u32 %0, %1, 1;" : "=r"(r) : "r"(smem_u32(done)));
        remote_arrive(r);
      }
    }
  } else if (PAIR && !leader && warp == 2 && lane == 0) {
    // relay: this CTA's landed stages to the first CTA's MMA thread
    int stage = 0;
    uint32_t phase = 0;
    for (int it = 0; it < iters; ++it) {
      if (!probe_wait(&full[stage], phase, status, false)) break;
      remote_arrive(mapa_rank0(smem_u32(&peer_full[stage])));
      if (++stage == kLoopStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // everyone: the last stage consumed (bounded)
  if (threadIdx.x == 64) probe_wait(done, 0, status, PAIR);
  __syncthreads();
  if (threadIdx.x == 32 && leader) {
    out[4 * blockIdx.x + 0] = *status;
    reinterpret_cast<long long*>(out)[2 * blockIdx.x + 1] = t1 - t0;
  } else if (threadIdx.x == 0 && !leader) {
    out[4 * blockIdx.x + 0] = *status;
    reinterpret_cast<long long*>(out)[2 * blockIdx.x + 1] = 0;
  }
  tc_fence_before();
  if (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (MMA && warp == 0) {
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    else
      tmem_dealloc(tmem, 512);
  }
}

template <bool PAIR, bool MMA>
int run_mainloop(int iters, const uint8_t* src, long long src_bytes, int* scratch, cudaStream_t st,
                 float* cycles, float* gbs) {
  auto kern = mainloop_probe_kernel<PAIR, MMA>;
  constexpr int kStage = 16384 + (PAIR ? 16384 : 32768);
  const int smem = kLoopStages * kStage + 1024 + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kPeakThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int grid = nsm;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) return 4;
    grid = 2 * clusters;
  }
  cfg.gridDim = dim3(grid);
  const long long src_blocks = src_bytes / 49152;
  if (src_blocks < 1) return 1;
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  if (cudaLaunchKernelEx(&cfg, kern, 64, src, src_blocks, scratch) != cudaSuccess) return 4;
  cudaEventRecord(e0, st);
  if (cudaLaunchKernelEx(&cfg, kern, iters, src, src_blocks, scratch) != cudaSuccess) return 4;
  cudaEventRecord(e1, st);
  if (cudaEventSynchronize(e1) != cudaSuccess) return 4;
  float ms = 0.0f;
  cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  int* host = new int[4 * grid];
  cudaMemcpy(host, scratch, sizeof(int) * 4 * grid, cudaMemcpyDeviceToHost);
  int status = 0;
  double cyc = 0.0;
  int n = 0;
  for (int b = 0; b < grid; ++b) {
    if (host[4 * b]) status = host[4 * b];
    const long long c = reinterpret_cast<long long*>(host)[2 * b + 1];
    if (c > 0) {
      cyc += static_cast<double>(c);
      ++n;
    }
  }
  delete[] host;
  *cycles = n ? static_cast<float>(cyc / n / iters) : 0.0f;
  *gbs = static_cast<float>(static_cast<double>(kStage) * iters * grid / (ms * 1e-3) / 1e9);
  return status;
}

// ---------------------------------------------------------------------------
// TMEM read probe: WARPS warps (a multiple of 4, each reading the 32 lanes of
// its quarter) repeatedly load COLS columns of FP32 with tcgen05.ld 32x32b.x16
// chunks, waiting once per LOADS chunks, and fold them into a register sum.
// Reports the tensor-memory to register rate of one SM.
// ---------------------------------------------------------------------------
template <int WARPS, int LOADS>
__global__ void __launch_bounds__(WARPS * 32, 1) tmem_read_probe_kernel(int iters, int* out) {
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  // each warp of a quarter owns 512 / (WARPS / 4) columns
  constexpr int kCols = 512 / (WARPS / 4);
  const uint32_t col0 = (warp >> 2) * kCols;
  float acc = 0.0f;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    for (int c = 0; c < kCols; c += 16 * LOADS) {
      uint32_t r[LOADS][16];
#pragma unroll
      for (int l = 0; l < LOADS; ++l) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[l][0]), "=r"(r[l][1]), "=r"(r[l][2]), "=r"(r[l][3]), "=r"(r[l][4]), "=r"(r[l][5]),
              "=r"(r[l][6]), "=r"(r[l][7]), "=r"(r[l][8]), "=r"(r[l][9]), "=r"(r[l][10]), "=r"(r[l][11]),
              "=r"(r[l][12]), "=r"(r[l][13]), "=r"(r[l][14]), "=r"(r[l][15])
            : "r"(tmem + lane_off + col0 + c + 16 * l));
      }
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int l = 0; l < LOADS; ++l)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc += __uint_as_float(r[l][i]);
    }
  }
  const long long t1 = clock64();
  if (acc == 1234.5f) out[3] = 1;   // keeps the loads
  if (threadIdx.x == 0) reinterpret_cast<long long*>(out)[0] = t1 - t0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// The same with one tcgen05.ld of WIDTH (32, 64 or 128) columns per wait.
template <int WARPS, int WIDTH>
__global__ void __launch_bounds__(WARPS * 32, 1) tmem_read_wide_kernel(int iters, int* out) {
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  constexpr int kCols = 512 / (WARPS / 4);
  const uint32_t col0 = (warp >> 2) * kCols;
  float acc = 0.0f;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    for (int c = 0; c < kCols; c += WIDTH) {
      uint32_t r[WIDTH];
      if constexpr (WIDTH == 32) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
              "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
              "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
              "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(tmem + lane_off + col0 + c));
      } else {
#pragma unroll
        for (int h = 0; h < WIDTH / 32; ++h)
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
              "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
              "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
              : "=r"(r[32 * h + 0]), "=r"(r[32 * h + 1]), "=r"(r[32 * h + 2]), "=r"(r[32 * h + 3]),
                "=r"(r[32 * h + 4]), "=r"(r[32 * h + 5]), "=r"(r[32 * h + 6]), "=r"(r[32 * h + 7]),
                "=r"(r[32 * h + 8]), "=r"(r[32 * h + 9]), "=r"(r[32 * h + 10]), "=r"(r[32 * h + 11]),
                "=r"(r[32 * h + 12]), "=r"(r[32 * h + 13]), "=r"(r[32 * h + 14]), "=r"(r[32 * h + 15]),
                "=r"(r[32 * h + 16]), "=r"(r[32 * h + 17]), "=r"(r[32 * h + 18]), "=r"(r[32 * h + 19]),
                "=r"(r[32 * h + 20]), "=r"(r[32 * h + 21]), "=r"(r[32 * h + 22]), "=r"(r[32 * h + 23]),
                "=r"(r[32 * h + 24]), "=r"(r[32 * h + 25]), "=r"(r[32 * h + 26]), "=r"(r[32 * h + 27]),
                "=r"(r[32 * h + 28]), "=r"(r[32 * h + 29]), "=r"(r[32 * h + 30]), "=r"(r[32 * h + 31])
              : "r"(tmem + lane_off + col0 + c + 32 * h));
      }
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int i = 0; i < WIDTH; i += 2) acc += __uint_as_float(r[i]) * __uint_as_float(r[i + 1]);
    }
  }
  const long long t1 = clock64();
  if (acc == 1234.5f) out[3] = 1;
  if (threadIdx.x == 0) reinterpret_cast<long long*>(out)[0] = t1 - t0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int WARPS, int WIDTH>
int run_tmem_wide(int iters, int* scratch, cudaStream_t st, float* bytes_per_cycle) {
  tmem_read_wide_kernel<WARPS, WIDTH><<<1, WARPS * 32, 0, st>>>(iters, scratch);
  if (cudaStreamSynchronize(st) != cudaSuccess) return 4;
  long long cyc = 0;
  cudaMemcpy(&cyc, scratch, sizeof(cyc), cudaMemcpyDeviceToHost);
  const double bytes = static_cast<double>(iters) * 128.0 * 512.0 * 4.0;
  *bytes_per_cycle = cyc > 0 ? static_cast<float>(bytes / cyc) : 0.0f;
  return 0;
}

template <int WARPS, int LOADS>
int run_tmem_read(int iters, int* scratch, cudaStream_t st, float* bytes_per_cycle) {
  tmem_read_probe_kernel<WARPS, LOADS><<<1, WARPS * 32, 0, st>>>(iters, scratch);
  if (cudaStreamSynchronize(st) != cudaSuccess) return 4;
  long long cyc = 0;
  cudaMemcpy(&cyc, scratch, sizeof(cyc), cudaMemcpyDeviceToHost);
  // every warp reads 32 lanes x 4 bytes x its columns per iteration
  const double bytes = static_cast<double>(iters) * 128.0 * 512.0 * 4.0;
  *bytes_per_cycle = cyc > 0 ? static_cast<float>(bytes / cyc) : 0.0f;
  return 0;
}

}  // namespace

extern "C" int moe_peak_mma(int kind, int n, int pair, int iters, void* scratch, void* stream, float* tflops,
                            float* cycles) {
  if (!scratch || !tflops || !cycles || iters < 1) return 1;
  int* s = static_cast<int*>(scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kind == 0 && n == 256 && !pair) return run_peak<0, 256, false>(iters, s, st, tflops, cycles);
  if (kind == 0 && n == 128 && !pair) return run_peak<0, 128, false>(iters, s, st, tflops, cycles);
  if (kind == 0 && n == 256 && pair) return run_peak<0, 256, true>(iters, s, st, tflops, cycles);
  if (kind == 1 && n == 256 && !pair) return run_peak<1, 256, false>(iters, s, st, tflops, cycles);
  if (kind == 1 && n == 128 && !pair) return run_peak<1, 128, false>(iters, s, st, tflops, cycles);
  if (kind == 1 && n == 256 && pair) return run_peak<1, 256, true>(iters, s, st, tflops, cycles);
  if (kind == 1 && n == 128 && pair) return run_peak<1, 128, true>(iters, s, st, tflops, cycles);
  if (kind == 2 && n == 256 && !pair) return run_peak<2, 256, false>(iters, s, st, tflops, cycles);
  if (kind == 2 && n == 128 && !pair) return run_peak<2, 128, false>(iters, s, st, tflops, cycles);
  if (kind == 3 && n == 256 && !pair) return run_peak<3, 256, false>(iters, s, st, tflops, cycles);
  return 2;
}

// Main-loop probe (see mainloop_probe_kernel): cycles per K block of the
// issuing CTA and the aggregate L2 -> shared memory rate.  src: device buffer
// of src_bytes (>= 48 KB) to stream from; scratch as for moe_peak_mma.
extern "C" int moe_peak_mainloop(int pair, int mma, int iters, const void* src, long long src_bytes, void* scratch,
                                 void* stream, float* cycles, float* gbs) {
  if (!src || !scratch || !cycles || !gbs || iters < 1) return 1;
  const uint8_t* s8 = static_cast<const uint8_t*>(src);
  int* sc = static_cast<int*>(scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pair && mma) return run_mainloop<true, true>(iters, s8, src_bytes, sc, st, cycles, gbs);
  if (pair && !mma) return run_mainloop<true, false>(iters, s8, src_bytes, sc, st, cycles, gbs);
  if (!pair && mma) return run_mainloop<false, true>(iters, s8, src_bytes, sc, st, cycles, gbs);
  return run_mainloop<false, false>(iters, s8, src_bytes, sc, st, cycles, gbs);
}

// TMEM read probe (see tmem_read_probe_kernel): bytes per SM cycle from
// tensor memory to registers with `warps` warps (4, 8 or 16) and `loads`
// 16-column loads in flight per wait (1, 2 or 4).
extern "C" int moe_peak_tmem_read(int warps, int loads, int iters, void* scratch, void* stream, float* bytes_per_cycle) {
  if (!scratch || !bytes_per_cycle || iters < 1) return 1;
  int* s = static_cast<int*>(scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (warps == 4 && loads == 1) return run_tmem_read<4, 1>(iters, s, st, bytes_per_cycle);
  if (warps == 4 && loads == 4) return run_tmem_read<4, 4>(iters, s, st, bytes_per_cycle);
  if (warps == 8 && loads == 1) return run_tmem_read<8, 1>(iters, s, st, bytes_per_cycle);
  if (warps == 8 && loads == 2) return run_tmem_read<8, 2>(iters, s, st, bytes_per_cycle);
  if (warps == 8 && loads == 4) return run_tmem_read<8, 4>(iters, s, st, bytes_per_cycle);
  if (warps == 16 && loads == 1) return run_tmem_read<16, 1>(iters, s, st, bytes_per_cycle);
  if (warps == 16 && loads == 2) return run_tmem_read<16, 2>(iters, s, st, bytes_per_cycle);
  if (warps == 16 && loads == 4) return run_tmem_read<16, 4>(iters, s, st, bytes_per_cycle);
  // loads >= 32: one load of that many columns per wait
  if (warps == 4 && loads == 32) return run_tmem_wide<4, 32>(iters, s, st, bytes_per_cycle);
  if (warps == 4 && loads == 64) return run_tmem_wide<4, 64>(iters, s, st, bytes_per_cycle);
  if (warps == 8 && loads == 32) return run_tmem_wide<8, 32>(iters, s, st, bytes_per_cycle);
  if (warps == 8 && loads == 64) return run_tmem_wide<8, 64>(iters, s, st, bytes_per_cycle);
  if (warps == 16 && loads == 32) return run_tmem_wide<16, 32>(iters, s, st, bytes_per_cycle);
  return 2;
}

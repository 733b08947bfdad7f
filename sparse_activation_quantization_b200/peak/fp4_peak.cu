// fp4_peak.cu - measured tcgen05 FP4 tensor peaks on this GPU (roofline
// denominators).  Every SM runs one CTA that issues back-to-back
// block-scaled FP4 MMAs (128 x N x K) from shared memory into TMEM, the
// instruction forms the SharQ GEMM uses: dense kind::mxf4nvf4 block16
// (K = 64) and 4:8-sparse tcgen05.mma.sp (K = 128 logical).  The pair form
// runs every two SMs as one CTA pair (cluster of 2) issuing the cta_group::2
// MMAs of the prefill GEMM (M = 256, N = 256), whose B operand is split
// between the two CTAs' shared memory.  Operands are zeros with valid
// metadata; throughput does not depend on values.
#include <cuda_runtime.h>

#include "../csrc/sharq_device.cuh"

using namespace sharq;

namespace {

constexpr int kSmem = 64 * 1024;

__global__ void __launch_bounds__(128, 1) fp4_peak_kernel(int sparse, int n256, int iters,
                                                          unsigned long long* ns) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t tbase;
  __shared__ __align__(8) uint64_t bar;
  for (int i = threadIdx.x; i < (kSmem - 1024) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x)   // metadata: pairs 0 and 1
    reinterpret_cast<uint32_t*>(sm + 56 * 1024)[i] = 0x44444444u;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 0) {
    const uint32_t s0 = smem_u32(sm);
    const uint32_t B = s0, A = s0 + 32768, E = s0 + 56 * 1024, SF = s0 + 48 * 1024;
    const int N = n256 ? 256 : 128;
    tc_cp_128x128b(tm + 256 + 48, smem_desc(E, 0, 128, kSwNone));
    for (int j = 0; j < 8; ++j) tc_cp_32x128b_x4(tm + 256 + 4 * j, smem_desc(SF, 0, 128, kSwNone));
    const uint32_t idn = idesc_nvf4(128, N, false), isp = idesc_nvf4(128, N, true);
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 0; it < iters; ++it) {
      if (sparse) {
        for (int j = 0; j < 2; ++j)
          mma_sp_nvf4(tm, smem_desc(A + 32 * j, 16, 512, kSw64), smem_desc(B + 64 * j, 16, 1024, kSw128),
                      tm + 256 + 48 + 2 * j, isp, tm + 256, tm + 256 + 8, 1u);
      } else {
        for (int j = 0; j < 4; ++j)
          mma_nvf4(tm, smem_desc(A + 32 * j, 16, 1024, kSw128), smem_desc(B + 32 * j, 16, 1024, kSw128), idn,
                   tm + 256, tm + 256 + 8, 1u);
      }
    }
    tc_commit(&bar);
    const unsigned long long lim = globaltimer_ns() + 2000000000ull;
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() > lim) break;
    }
    ns[blockIdx.x] = globaltimer_ns() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

__global__ void __launch_bounds__(128, 1) fp4_peak_pair_kernel(int sparse, int iters, unsigned long long* ns) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t tbase;
  __shared__ __align__(8) uint64_t bar;
  // per CTA: B half (128 rows) at 0, A at 16 KB, scales at 32 KB, metadata at 40 KB
  for (int i = threadIdx.x; i < (kSmem - 1024) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x)   // metadata: pairs 0 and 1
    reinterpret_cast<uint32_t*>(sm + 40 * 1024)[i] = 0x44444444u;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc_pair(&tbase, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 0 && cluster_ctarank() == 0) {
    const uint32_t s0 = smem_u32(sm);
    const uint32_t B = s0, A = s0 + 16384, SF = s0 + 32768, E = s0 + 40960;
    tc_cp_pair_128x128b(tm + 256 + 48, smem_desc(E, 0, 128, kSwNone));
    for (int j = 0; j < 8; ++j) tc_cp_pair_32x128b_x4(tm + 256 + 4 * j, smem_desc(SF, 0, 128, kSwNone));
    const uint32_t idn = idesc_nvf4(256, 256, false), isp = idesc_nvf4(256, 256, true);
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 0; it < iters; ++it) {
      if (sparse) {
        for (int j = 0; j < 2; ++j)
          mma_pair_sp_nvf4(tm, smem_desc(A + 32 * j, 16, 512, kSw64), smem_desc(B + 64 * j, 16, 1024, kSw128),
                           tm + 256 + 48 + 2 * j, isp, tm + 256, tm + 256 + 8, 1u);
      } else {
        for (int j = 0; j < 4; ++j)
          mma_pair_nvf4(tm, smem_desc(A + 32 * j, 16, 1024, kSw128), smem_desc(B + 32 * j, 16, 1024, kSw128), idn,
                        tm + 256, tm + 256 + 8, 1u);
      }
    }
    tc_commit_pair(&bar);
    const unsigned long long lim = globaltimer_ns() + 2000000000ull;
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() > lim) break;
    }
    ns[blockIdx.x >> 1] = globaltimer_ns() - t0;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs are done before either CTA frees TMEM
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc_pair(tm, 512);
  }
}

}  // namespace

// Measured FP4 peak of the CTA-pair form (M = 256, N = 256) in FLOP/s
// (logical FLOPs for the sparse form), over every SM pair.  Returns 0 on
// success.
extern "C" int sharq_fp4_peak_pair(int sparse, int iters, double* flops_per_s, double* pair_ns_mean) {
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
    return -4;
  const int pairs = sms / 2;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, sizeof(unsigned long long) * pairs) != cudaSuccess) return -4;
  cudaFuncSetAttribute(fp4_peak_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  for (int rep = 0; rep < 2; ++rep) {  // first launch warms up
    if (cudaLaunchKernelEx(&cfg, fp4_peak_pair_kernel, sparse, iters, d) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(d);
      return -4;
    }
  }
  unsigned long long* h = new unsigned long long[pairs];
  cudaMemcpy(h, d, sizeof(unsigned long long) * pairs, cudaMemcpyDeviceToHost);
  double mean = 0.0;
  for (int i = 0; i < pairs; ++i) mean += (double)h[i];
  mean /= pairs;
  delete[] h;
  cudaFree(d);
  // per iteration: 4 dense 256x256x64 or 2 sparse 256x256x128 (logical) MMAs
  const double flop_iter = 2.0 * 256.0 * 256.0 * 256.0;
  *flops_per_s = flop_iter * iters * pairs / (mean * 1e-9);
  *pair_ns_mean = mean;
  return 0;
}

// Measured FP4 peak in FLOP/s (logical FLOPs for the sparse form), N = 256
// or 128, over every SM.  Returns 0 on success.
extern "C" int sharq_fp4_peak(int sparse, int n256, int iters, double* flops_per_s, double* sm_ns_mean) {
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
    return -4;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, sizeof(unsigned long long) * sms) != cudaSuccess) return -4;
  cudaFuncSetAttribute(fp4_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  double mean = 0.0;
  for (int rep = 0; rep < 2; ++rep) {  // first launch warms up
    fp4_peak_kernel<<<sms, 128, kSmem>>>(sparse, n256, iters, d);
    if (cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(d);
      return -4;
    }
  }
  unsigned long long* h = new unsigned long long[sms];
  cudaMemcpy(h, d, sizeof(unsigned long long) * sms, cudaMemcpyDeviceToHost);
  for (int i = 0; i < sms; ++i) mean += (double)h[i];
  mean /= sms;
  delete[] h;
  cudaFree(d);
  const double N = n256 ? 256.0 : 128.0;
  // per iteration: 4 dense 128xNx64 or 2 sparse 128xNx128 (logical) MMAs
  const double flop_iter = 2.0 * 128.0 * N * 256.0;
  *flops_per_s = flop_iter * iters * sms / (mean * 1e-9);
  *sm_ns_mean = mean;
  return 0;
}

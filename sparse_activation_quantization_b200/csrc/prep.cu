// prep.cu - sharq_prep: the fused activation preparation of SharQ.
//
// xllm-io review of SharQ, section 3.5 ("fused activation preparation":
// RMSNorm/PTS + pair-top-k 4:8 in-pairs mask + sparse compression + dense
// residual construction in one preparation step) and sections 3.2-3.3 for
// what is computed; kasblo.com explainer, steps 1-3 of the recipe.
//
// The per-tensor scale (PTS) is a device-wide max that every quantization
// step needs before it can emit a code.  Two forms:
//   single launch (prep_fused_kernel): a grid that fits the GPU holds the whole
//     tensor in registers -- load, RMSNorm, device-wide max through a bounded
//     grid barrier, then quantize; X is read once.  Used whenever the grid
//     fits on the GPU at once.
//   two launches (larger tensors): prep_stats_kernel (one CTA per row:
//     float64 sum of squares -> 1/rms, row max |Xn| -> atomicMax), then
//     prep_quant_kernel (re-reads X, L2-resident up to ~100 MB).
// Work unit: one thread per run of 8 consecutive K (one 16-byte load, one
// 4:8 in-pairs chunk); rows longer than 8192 give each thread 2 or 4 runs.
// The 32-K backbone block and the 16-K residual block span 4 and 2 such
// threads (adjacent lanes), reduced with warp shuffles.  The residual never
// leaves registers; every output is stored in the MMA-ready tiled layout of
// include/sharq.h.
#include "quant.cuh"

namespace sharq {

namespace {

// Optional phase timeline (compile with -DSHARQ_TRACE): 4 global-timer
// stamps per CTA of the single-launch kernel -- entry, max published,
// barrier passed, exit.
#ifdef SHARQ_TRACE
__device__ unsigned long long* g_trace_prep = nullptr;
#define PREP_TRACE(k)                                                                        \
  do {                                                                                       \
    if (g_trace_prep && threadIdx.x == 0) g_trace_prep[(size_t)blockIdx.x * 4 + (k)] = globaltimer_ns(); \
  } while (0)
#else
#define PREP_TRACE(k) \
  do {                \
  } while (0)
#endif

template <int NW>
__device__ __forceinline__ double block_sum_d(double v, double* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  double r = 0.0;
#pragma unroll
  for (int i = 0; i < NW; ++i) r += sh[i];
  __syncthreads();
  return r;
}

template <int NW>
__device__ __forceinline__ float block_max_f(float v, float* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  float r = 0.0f;
#pragma unroll
  for (int i = 0; i < NW; ++i) r = fmaxf(r, sh[i]);
  return r;
}

constexpr int kStatsThreads = 256;

__global__ void __launch_bounds__(kStatsThreads) prep_stats_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma, float eps,
    const int* __restrict__ row_index, int K, float* __restrict__ inv_rms,
    unsigned int* __restrict__ gmax_bits) {
  __shared__ double sh_d[kStatsThreads / 32];
  __shared__ float sh_f[kStatsThreads / 32];
  const int t = blockIdx.x;
  const int src = row_index ? row_index[t] : t;
  const int nch = K >> 3;
  float inv = 1.0f;
  if (src < 0) {  // zero padding row: Xn = 0 contributes nothing to gmax
    if (threadIdx.x == 0 && gamma) inv_rms[t] = (float)(1.0 / sqrt((double)eps));
    else if (threadIdx.x == 0) inv_rms[t] = 1.0f;
    return;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)src * K);
  const uint4* gr = reinterpret_cast<const uint4*>(gamma);
  if (gamma) {
    double ss = 0.0;
    for (int c = threadIdx.x; c < nch; c += kStatsThreads) {
      float f[8];
      bf16x8_to_float(xr[c], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += (double)f[i] * (double)f[i];
    }
    ss = block_sum_d<kStatsThreads / 32>(ss, sh_d);
    inv = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
  }
  float amax = 0.0f;
  for (int c = threadIdx.x; c < nch; c += kStatsThreads) {
    float f[8];
    bf16x8_to_float(xr[c], f);
    if (gamma) {
      float g[8];
      bf16x8_to_float(gr[c], g);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(norm_one(f[i], inv, g[i])));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
  }
  amax = block_max_f<kStatsThreads / 32>(amax, sh_f);
  if (threadIdx.x == 0) {
    inv_rms[t] = inv;
    atomicMax(gmax_bits, __float_as_uint(amax));  // non-negative floats order as uints
  }
}

// Allow the next kernel in the stream (the GEMM, launched as a programmatic
// dependent) to start its set-up and weight loads now; it waits for this
// grid's completion (griddepcontrol.wait) before reading our outputs.
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Last CTA out resets the device-wide max and the counters (sync words
// 0..2 of the act scalar block), so the next sharq_prep on this buffer
// starts from zero without a memset.  Called by thread 0 of every CTA at its
// end, after the CTA has read the max (so the reset cannot race a reader).
__device__ __forceinline__ void depart_and_reset(unsigned int* sync) {
  if (atomicAdd(sync + 2, 1u) == gridDim.x - 1) {
    sync[0] = 0u;
    sync[1] = 0u;
    sync[2] = 0u;
    __threadfence();
  }
}

constexpr int kQuantThreads = 256;

// Two-launch form, second launch: one thread per 32 consecutive K (four runs
// of 8; every quantization block inside the thread), flat over rows.
template <bool kSharq>
__global__ void __launch_bounds__(kQuantThreads) prep_quant_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma,
    const int* __restrict__ row_index, int T, int Tp, int K, const float* __restrict__ inv_rms,
    const unsigned int* __restrict__ gmax_bits, float* __restrict__ s_g_out, QuantPtrs out) {
  __shared__ float gmax_sh;
  allow_dependents();
  const int segs = K >> 5;
  const long long gid = (long long)blockIdx.x * kQuantThreads + threadIdx.x;
  if (threadIdx.x == 0) gmax_sh = __uint_as_float(*(volatile const unsigned int*)gmax_bits);
  __syncthreads();
  const float gmax = gmax_sh;
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  if (gid == 0) *s_g_out = s;  // published even when there are no rows
  if (gid < (long long)T * segs) {
    const int t = (int)(gid / segs);
    const int c0 = (int)(gid - (long long)t * segs) * 4;
    const int src = row_index ? row_index[t] : t;
    float x[32];
    load_runs<4>(x, X, src, K, c0);
    if (gamma && src >= 0) normalise_runs<4>(x, gamma, c0, inv_rms[t]);
    quant_runs<4, kSharq>(x, t, c0, K, s, __fmul_rn(6.0f, s), out);
  }
  if (threadIdx.x == 0) depart_and_reset(const_cast<unsigned int*>(gmax_bits));
}

// ---------------------------------------------------------------------------
// Single-launch form (cooperative grid; whole rows inside a CTA).
constexpr int kFusedMaxThreads = 1024;
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

template <int NC>
constexpr int fused_max_threads() { return NC == 4 ? 640 : kFusedMaxThreads; }

template <int NC, bool kSharq>
__global__ void __launch_bounds__(fused_max_threads<NC>()) prep_fused_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma, float eps,
    const int* __restrict__ row_index, int T, int Tp, int K, int rows_per_cta, float* __restrict__ inv_rms,
    unsigned int* sync, float* __restrict__ s_g_out, QuantPtrs out) {
  __shared__ double wsum[kFusedMaxThreads / 32];
  __shared__ float wmax[kFusedMaxThreads / 32];
  __shared__ float gmax_sh;
  PREP_TRACE(0);
  allow_dependents();
  if (blockIdx.x == 0 && threadIdx.x == 0) sync[3] = 0u;  // error word of the previous prep
  // threads per row, padded to whole warps (a warp never spans two rows);
  // the padding lanes hold zeros and store nothing
  const int used = (K >> 3) / NC;
  const int tpr = (used + 31) & ~31;
  const int rl = threadIdx.x / tpr;
  const int li = threadIdx.x - rl * tpr;
  const bool has = li < used;
  const int c0 = (has ? li : 0) * NC;
  const int t = blockIdx.x * rows_per_cta + rl;
  const bool live = t < T;  // rows T..Tp-1 (tile padding) are not written
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpr = tpr >> 5;                 // warps per row

  float x[8 * NC];
  int src = -1;
  if (live && has) src = row_index ? row_index[t] : t;
  load_runs<NC>(x, X, src, K, c0);
  // gamma in flight together with X (not after the row reduction)
  uint4 graw[NC];
  if (gamma && src >= 0) {
    const uint4* gr = reinterpret_cast<const uint4*>(gamma) + c0;
#pragma unroll
    for (int c = 0; c < NC; ++c) graw[c] = gr[c];
  }

  if (gamma) {
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 8 * NC; ++i) ss += (double)x[i] * (double)x[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) wsum[warp] = ss;
    __syncthreads();
    double tot = 0.0;
    for (int w = 0; w < wpr; ++w) tot += wsum[rl * wpr + w];  // fixed order
    const float inv = (float)(1.0 / sqrt(tot / (double)K + (double)eps));
    if (live && li == 0) inv_rms[t] = inv;
    if (src >= 0) {
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float g[8];
        bf16x8_to_float(graw[c], g);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[8 * c + e] = norm_one(x[8 * c + e], inv, g[e]);
      }
    }
  } else if (live && li == 0) {
    inv_rms[t] = 1.0f;
  }

  // CTA max |Xn| -> device-wide max
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8 * NC; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) wmax[warp] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
    if (gridDim.x == 1) {
      gmax_sh = m;  // one CTA holds the whole tensor: no grid barrier
    } else {
      atomicMax(sync, __float_as_uint(m));
      // arrival with release semantics: our max is visible before the count
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(sync + 1) : "memory");
      PREP_TRACE(1);
      // grid barrier: every CTA has published its max (bounded spin)
      const uint64_t deadline = globaltimer_ns() + kBarrierLimitNs;
      unsigned seen = 0;
      do {
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(sync + 1) : "memory");
        if (seen >= gridDim.x) break;
        if (globaltimer_ns() > deadline) {
          atomicCAS(reinterpret_cast<int*>(sync + 3), 0, -5);  // SHARQ_ERR_TIMEOUT
          break;
        }
      } while (true);
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      gmax_sh = __uint_as_float(*(volatile unsigned int*)sync);
    }
    PREP_TRACE(2);
  }
  __syncthreads();
  const float gmax = gmax_sh;
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s;
  // rows past T: whole warps (rows span whole warps), so they can skip
  if (live) quant_runs<NC, kSharq>(x, t, c0, K, s, __fmul_rn(6.0f, s), out, has);
  if (threadIdx.x == 0 && gridDim.x > 1) depart_and_reset(sync);
#ifdef SHARQ_TRACE
  __syncthreads();
  PREP_TRACE(3);
#endif
}

// runs of 8 per thread so that a row fits one CTA (<= 1024 threads)
int fused_runs_per_thread(int K) {
  const int runs = K >> 3;
  if (runs <= 1024) return 1;
  if (runs <= 2048 && (runs / 2) % 2 == 0) return 2;
  if (runs <= 4 * 640) return 4;
  return 0;
}

// Prep CTAs use almost no shared memory; ask for the maximum shared-memory
// carveout anyway so that an SM running them keeps room for a GEMM CTA
// (~215 KB) launched early as their programmatic dependent.
template <class F>
void prefer_max_shared(F* fn) {
  cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  cudaGetLastError();
}

template <int NC, bool kSharq>
int fused_max_ctas_t(int threads) {
  static int cache[kFusedMaxThreads + 1][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return 0;
  int& c = cache[threads][dev];
  if (c == 0) {
    prefer_max_shared(prep_fused_kernel<NC, kSharq>);
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prep_fused_kernel<NC, kSharq>, threads, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    c = per_sm * sms > 0 ? per_sm * sms : -1;
  }
  return c > 0 ? c : 0;
}

template <int NC, bool kSharq>
cudaError_t try_fused(const __nv_bfloat16* Xb, const __nv_bfloat16* Gb, float eps, const int* row_index, int T,
                      int Tp, int K, float* inv_rms, unsigned int* sync, float* s_g, QuantPtrs p,
                      cudaStream_t stream, bool* launched) {
  *launched = false;
  const int tpr = (((K >> 3) / NC) + 31) & ~31;
  int rpc = 512 / tpr;
  rpc = rpc < 1 ? 1 : rpc;
  const int threads = rpc * tpr;
  const int ctas = (T + rpc - 1) / rpc;
  if (ctas > fused_max_ctas_t<NC, kSharq>(threads)) return cudaSuccess;
  // A plain launch: the grid fits the GPU at once (checked above), so all
  // CTAs are resident together when the stream reaches this kernel; the
  // GEMM that follows as a programmatic dependent can start only after every
  // CTA of this grid has started (each triggers at entry), so it cannot
  // crowd out a CTA that has not arrived at the grid barrier.  The barrier's
  // spin is bounded all the same.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prep_fused_kernel<NC, kSharq>, Xb, Gb, eps, row_index, T, Tp, K, rpc,
                                     inv_rms, sync, s_g, p);
  if (e == cudaSuccess) *launched = true;
  else cudaGetLastError();  // fall back to the two-launch form
  return cudaSuccess;
}

template <bool kSharq>
cudaError_t try_fused_any(const __nv_bfloat16* Xb, const __nv_bfloat16* Gb, float eps, const int* row_index, int T,
                          int Tp, int K, float* inv_rms, unsigned int* sync, float* s_g, QuantPtrs p,
                          cudaStream_t stream, bool* launched) {
  switch (fused_runs_per_thread(K)) {
    case 1: return try_fused<1, kSharq>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, stream, launched);
    case 2: return try_fused<2, kSharq>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, stream, launched);
    case 4: return try_fused<4, kSharq>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, stream, launched);
    default: *launched = false; return cudaSuccess;
  }
}

}  // namespace

#ifdef SHARQ_TRACE
extern "C" int sharq_debug_set_trace_prep(void* p) {
  return cudaMemcpyToSymbol(g_trace_prep, &p, sizeof(p)) == cudaSuccess ? 0 : -4;
}
#endif

cudaError_t launch_prep(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp,
                        int K, bool sharq_mode, float* inv_rms, float* s_g, unsigned int* gmax_bits,
                        uint8_t* sp_codes, uint8_t* meta, uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf,
                        cudaStream_t stream) {
  // gmax_bits[0..3]: device-wide max, barrier arrivals, departures, error
  // word; zero at rest (the kernels reset them), so no memset is needed
  cudaError_t e = cudaSuccess;
  QuantPtrs p{sp_codes, meta, sp_sf, r_codes, r_sf};
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  const __nv_bfloat16* Gb = static_cast<const __nv_bfloat16*>(gamma);

  if (T > 0) {
    bool launched = false;
    e = sharq_mode ? try_fused_any<true>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, stream,
                                         &launched)
                   : try_fused_any<false>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, stream,
                                          &launched);
    if (e != cudaSuccess) return e;
    if (launched) return cudaSuccess;
  }

  static bool carveout_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev < 64 && !carveout_set[dev]) {
    prefer_max_shared(prep_quant_kernel<true>);
    prefer_max_shared(prep_quant_kernel<false>);
    carveout_set[dev] = true;
  }
  if (T > 0) {
    prep_stats_kernel<<<T, kStatsThreads, 0, stream>>>(Xb, Gb, eps, row_index, K, inv_rms, gmax_bits);
  }
  const long long n = (long long)T * (K >> 5);
  // at least one block so that s_g is published (= 1) even for T == 0
  const unsigned grid = n > 0 ? (unsigned)((n + kQuantThreads - 1) / kQuantThreads) : 1u;
  if (sharq_mode)
    prep_quant_kernel<true><<<grid, kQuantThreads, 0, stream>>>(Xb, Gb, row_index, T, Tp, K, inv_rms, gmax_bits,
                                                                 s_g, p);
  else
    prep_quant_kernel<false><<<grid, kQuantThreads, 0, stream>>>(Xb, Gb, row_index, T, Tp, K, inv_rms,
                                                                  gmax_bits, s_g, p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free form (the sharq_prep_noalloc entry point).  The prep's
// working memory -- the device-wide max, the grid-barrier and departure
// counters, the error word, and the per-row 1/rms -- lives in this
// file-scope device array instead of the caller's buffer.  Every GPU that
// loads the library keeps the array until the process exits, and all calls
// share it: calls whose kernels overlap on the GPU race on it.
constexpr int kNoAllocMaxRows = 16384;
constexpr size_t kNoAllocSyncBytes = 256;
static __device__ __align__(256) unsigned char g_prep_scratch[kNoAllocSyncBytes + 4 * kNoAllocMaxRows];

int noalloc_max_rows() { return kNoAllocMaxRows; }

// Device address of g_prep_scratch for the current device, looked up on the
// first call on that device (host code cannot use the symbol itself).
static cudaError_t noalloc_scratch(unsigned char** out) {
  static unsigned char* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prep_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_prep_noalloc(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp,
                                int K, bool sharq_mode, float* s_g, uint8_t* sp_codes, uint8_t* meta,
                                uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf, unsigned int* err_out,
                                cudaStream_t stream) {
  if (T > kNoAllocMaxRows) return cudaErrorInvalidValue;
  unsigned char* scr = nullptr;
  cudaError_t e = noalloc_scratch(&scr);
  if (e != cudaSuccess) return e;
  unsigned int* sync = reinterpret_cast<unsigned int*>(scr);
  float* inv = reinterpret_cast<float*>(scr + kNoAllocSyncBytes);
  // the array keeps the last call's contents: start every call from zero
  e = cudaMemsetAsync(sync, 0, 4 * sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  e = launch_prep(X, gamma, eps, row_index, T, Tp, K, sharq_mode, inv, s_g, sync, sp_codes, meta, sp_sf, r_codes,
                  r_sf, stream);
  if (e != cudaSuccess) return e;
  // forward the error word to where sharq_linear looks for it
  if (err_out) e = cudaMemcpyAsync(err_out, sync + 3, sizeof(unsigned int), cudaMemcpyDeviceToDevice, stream);
  return e;
}

}  // namespace sharq

// prep.cu - sharq_prep: the fused activation preparation of SharQ.
//
// xllm-io review of SharQ, section 3.5 ("fused activation preparation":
// RMSNorm/PTS + pair-top-k 4:8 in-pairs mask + sparse compression + dense
// residual construction in one preparation step) and sections 3.2-3.3 for
// what is computed; kasblo.com explainer, steps 1-3 of the recipe.
//
// Two launches, because the per-tensor scale (PTS) is a device-wide max that
// every quantization step needs before it can emit a code:
//   prep_stats_kernel  one CTA per row: sum of squares (float64) -> 1/rms,
//                      then max |Xn| of the row -> atomicMax into gmax.
//   prep_quant_kernel  one thread per (row, 32 logical K): reload the row
//                      segment (L2-resident for tensors below ~100 MB), redo
//                      Xn, pick the 2 of 4 pairs in each run of 8, quantize
//                      the 16 kept values (one E4M3 scale per 32 logical K),
//                      form R = Xn - dequant(backbone) in registers, quantize
//                      R in two 16-element blocks, store every output in the
//                      MMA-ready tiled layout of include/sharq.h.
// Loads are 128-bit and coalesced (consecutive threads take consecutive
// 64-byte row segments); the residual never leaves registers.
#include "sharq_device.cuh"

namespace sharq {

namespace {

__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 p = __bfloat1622float2(h[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

// Xn = bf16_rn(f32(f32(x * inv) * g))
__device__ __forceinline__ float norm_one(float x, float inv, float g) {
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(__fmul_rn(x, inv), g)));
}

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

// pick a[sel] for sel in 0..3 without dynamic register indexing
__device__ __forceinline__ float pick4(const float* a, int sel) {
  float r = a[0];
  r = sel == 1 ? a[1] : r;
  r = sel == 2 ? a[2] : r;
  r = sel == 3 ? a[3] : r;
  return r;
}

// 16 values -> 8 bytes of E2M1 codes (value 2i in the low nibble of byte i)
__device__ __forceinline__ uint2 quant16(const float* v, float inv, uint32_t* codes) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = cvt_e2m1x2(__fmul_rn(v[2 * i], inv), __fmul_rn(v[2 * i + 1], inv));
    codes[2 * i] = b[i] & 0xFu;
    codes[2 * i + 1] = b[i] >> 4;
  }
  uint2 out;
  out.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  out.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  return out;
}

__device__ __forceinline__ float amax_n(const float* v, int n) {
  float a = 0.0f;
  for (int i = 0; i < n; ++i) a = fmaxf(a, fabsf(v[i]));
  return a;
}

struct QuantPtrs {
  uint8_t* sp_codes;
  uint8_t* meta;
  uint8_t* sp_sf;
  uint8_t* r_codes;
  uint8_t* r_sf;
};

constexpr int kQuantThreads = 256;

// Quantize one row segment of 32 logical K (row t, 32-block j) held in
// registers: mask, backbone NVFP4, residual, dense NVFP4, tiled stores.
template <bool kSharq>
__device__ __forceinline__ void quant_segment(const float (&x)[32], int t, int j, int K, float s, float six_s,
                                              const QuantPtrs& out) {
  const int KS = K >> 8;
  const int kt = j >> 3, q = j & 7;
  const int r = t & 127;
  const size_t tile = (size_t)(t >> 7) * KS + kt;

  float res[32];
  if (kSharq) {
    // --- 4:8 in-pairs mask: keep the 2 of 4 pairs with the largest max|x| ---
    float v[16];
    int lo[4], hi[4];
    uint32_t meta16 = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float sc[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) sc[p] = fmaxf(fabsf(x[8 * c + 2 * p]), fabsf(x[8 * c + 2 * p + 1]));
      bool keep[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        int beaten = 0;
#pragma unroll
        for (int o = 0; o < 4; ++o)
          if (o != p) beaten += (sc[o] > sc[p]) || (sc[o] == sc[p] && o < p);
        keep[p] = beaten < 2;
      }
      int a = -1, b = -1;
#pragma unroll
      for (int p = 3; p >= 0; --p)
        if (keep[p]) { b = a; a = p; }
      lo[c] = a;
      hi[c] = b;
      meta16 |= (uint32_t)(a | (b << 2)) << (4 * c);
      float ev[4], od[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) { ev[p] = x[8 * c + 2 * p]; od[p] = x[8 * c + 2 * p + 1]; }
      v[4 * c + 0] = pick4(ev, a);
      v[4 * c + 1] = pick4(od, a);
      v[4 * c + 2] = pick4(ev, b);
      v[4 * c + 3] = pick4(od, b);
    }
    // --- backbone NVFP4: one scale for these 32 logical K (16 kept values) ---
    const BlockScale bs = block_scale(amax_n(v, 16), six_s, s);
    uint32_t code[16];
    const uint2 spc = quant16(v, bs.inv, code);
    // --- residual R = Xn - dequant(backbone), exact float32 per element ---
#pragma unroll
    for (int i = 0; i < 32; ++i) res[i] = x[i];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const bool is_lo = (p == lo[c]), is_hi = (p == hi[c]);
        if (is_lo || is_hi) {
          const int slot = is_lo ? 0 : 2;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            uint32_t cd = code[4 * c + e];
            cd = slot ? code[4 * c + 2 + e] : cd;
            const float xt = __fmul_rn(__fmul_rn(e2m1_value(cd), bs.dec), s);
            res[8 * c + 2 * p + e] = __fsub_rn(x[8 * c + 2 * p + e], xt);
          }
        }
      }
    }
    // --- stores: sparse codes, metadata, sparse scale ---
    *reinterpret_cast<uint2*>(out.sp_codes + tile * kSpTile + sp_chunk_off(r, q >> 1) + (q & 1) * 8) = spc;
    *reinterpret_cast<uint16_t*>(out.meta + tile * kMetaTile + r * 16 + q * 2) = (uint16_t)meta16;
    out.sp_sf[tile * kSf32Tile + sf_off(r, q >> 2, q & 3)] = (uint8_t)bs.sb;
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) res[i] = x[i];
  }

  // --- dense NVFP4 of R (or of Xn in NVFP4 mode): two 16-element blocks ---
  const BlockScale b0 = block_scale(amax_n(res, 16), six_s, s);
  const BlockScale b1 = block_scale(amax_n(res + 16, 16), six_s, s);
  uint32_t dummy[16];
  const uint2 c0 = quant16(res, b0.inv, dummy);
  const uint2 c1 = quant16(res + 16, b1.inv, dummy);
  *reinterpret_cast<uint4*>(out.r_codes + tile * kCodesTile + codes_chunk_off(r, q)) =
      make_uint4(c0.x, c0.y, c1.x, c1.y);
  *reinterpret_cast<uint16_t*>(out.r_sf + tile * kSf16Tile + sf_off(r, q >> 1, 2 * (q & 1))) =
      (uint16_t)(b0.sb | (b1.sb << 8));
}


template <bool kSharq>
__global__ void __launch_bounds__(kQuantThreads) prep_quant_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma,
    const int* __restrict__ row_index, int T, int Tp, int K, const float* __restrict__ inv_rms,
    const unsigned int* __restrict__ gmax_bits, float* __restrict__ s_g_out, QuantPtrs out) {
  const int nb32 = K >> 5;
  const long long gid = (long long)blockIdx.x * kQuantThreads + threadIdx.x;
  const float gmax = __uint_as_float(*gmax_bits);
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  if (gid == 0) *s_g_out = s;  // published even when there are no rows
  if (gid >= (long long)Tp * nb32) return;
  const int t = (int)(gid / nb32);
  const int j = (int)(gid - (long long)t * nb32);
  const float six_s = __fmul_rn(6.0f, s);

  // --- load the 32 values of this row segment and normalise them ---
  float x[32];
  int src = -1;
  if (t < T) src = row_index ? row_index[t] : t;
  if (src >= 0) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)src * K + 32 * j);
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = xr[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) bf16x8_to_float(raw[i], x + 8 * i);
    if (gamma) {
      const float inv = inv_rms[t];
      const uint4* gr = reinterpret_cast<const uint4*>(gamma + 32 * j);
      float g[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) bf16x8_to_float(gr[i], g + 8 * i);
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = norm_one(x[i], inv, g[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = 0.0f;
  }

  quant_segment<kSharq>(x, t, j, K, s, six_s, out);
}


// ---------------------------------------------------------------------------
// Single-launch form: one cooperative grid, one thread per (row, 32-K block),
// whole rows inside a CTA (rows_per_cta x K/32 threads).  The row's values
// stay in registers from the load to the stores:
//   1. load + sum of squares (float64, fixed-order tree per row) -> 1/rms,
//      normalise in registers, CTA max |Xn|  -> atomicMax(gmax);
//   2. grid-wide barrier (arrival counter, bounded spin on the global timer);
//   3. quantize from registers (same code as prep_quant_kernel).
// X is read from HBM exactly once.  Used whenever the grid fits on the GPU at
// once (cooperative launch guarantees co-residency); larger tensors take the
// two-launch path above.
constexpr int kFusedMaxThreads = 640;            // K/32 <= 592 threads per row
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

template <bool kSharq>
__global__ void __launch_bounds__(kFusedMaxThreads) prep_fused_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma, float eps,
    const int* __restrict__ row_index, int T, int Tp, int K, int rows_per_cta, float* __restrict__ inv_rms,
    unsigned int* sync, float* __restrict__ s_g_out, QuantPtrs out) {
  __shared__ double part[kFusedMaxThreads];
  __shared__ float wmax[kFusedMaxThreads / 32];
  __shared__ float gmax_sh;
  const int nb32 = K >> 5;
  const int rl = threadIdx.x / nb32;
  const int j = threadIdx.x - rl * nb32;
  const int t = blockIdx.x * rows_per_cta + rl;
  const bool live = t < Tp;

  float x[32];
  int src = -1;
  if (live && t < T) src = row_index ? row_index[t] : t;
  if (src >= 0) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)src * K + 32 * j);
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = xr[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) bf16x8_to_float(raw[i], x + 8 * i);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = 0.0f;
  }

  if (gamma) {
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 32; ++i) ss += (double)x[i] * (double)x[i];
    part[threadIdx.x] = ss;
    __syncthreads();
    int span = 1;
    while (span < nb32) span <<= 1;
    for (int off = span >> 1; off > 0; off >>= 1) {
      if (j < off && j + off < nb32) part[threadIdx.x] += part[threadIdx.x + off];
      __syncthreads();
    }
    const float inv = (float)(1.0 / sqrt(part[rl * nb32] / (double)K + (double)eps));
    if (live && t < T && j == 0) inv_rms[t] = inv;
    const uint4* gr = reinterpret_cast<const uint4*>(gamma + 32 * j);
    float g[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) bf16x8_to_float(gr[i], g + 8 * i);
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = norm_one(x[i], inv, g[i]);
  } else if (live && t < T && j == 0) {
    inv_rms[t] = 1.0f;
  }

  // CTA max |Xn| -> device-wide max
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) m = fmaxf(m, wmax[w]);
    atomicMax(sync, __float_as_uint(m));
    __threadfence();
    atomicAdd(sync + 1, 1u);
    // grid barrier: every CTA has published its max
    const uint64_t deadline = globaltimer_ns() + kBarrierLimitNs;
    unsigned seen = 0;
    do {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(sync + 1) : "memory");
      if (seen >= gridDim.x) break;
      if (globaltimer_ns() > deadline) {
        atomicCAS(reinterpret_cast<int*>(sync + 3), 0, -5);  // SHARQ_ERR_TIMEOUT
        break;
      }
    } while (true);
    unsigned gb;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(gb) : "l"(sync) : "memory");
    gmax_sh = __uint_as_float(gb);
  }
  __syncthreads();
  const float gmax = gmax_sh;
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s;
  if (live) quant_segment<kSharq>(x, t, j, K, s, __fmul_rn(6.0f, s), out);
}


// rows per CTA of the single-launch form for a row length of K
int fused_rows_per_cta(int K) {
  const int nb32 = K >> 5;
  if (nb32 > kFusedMaxThreads) return 0;
  return nb32 >= 256 ? 1 : 256 / nb32;
}

// Largest grid of the single-launch form that can be resident at once.
int fused_max_ctas(bool sharq_mode, int threads) {
  static int cache[2][kFusedMaxThreads + 1][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return 0;
  int& c = cache[sharq_mode ? 1 : 0][threads][dev];
  if (c == 0) {
    int per_sm = 0, sms = 0;
    cudaError_t e = sharq_mode
        ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prep_fused_kernel<true>, threads, 0)
        : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prep_fused_kernel<false>, threads, 0);
    if (e != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    c = per_sm * sms > 0 ? per_sm * sms : -1;
  }
  return c > 0 ? c : 0;
}

}  // namespace

cudaError_t launch_prep(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp,
                        int K, bool sharq_mode, float* inv_rms, float* s_g, unsigned int* gmax_bits,
                        uint8_t* sp_codes, uint8_t* meta, uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf,
                        cudaStream_t stream) {
  // gmax, barrier arrivals, (unused), error word
  cudaError_t e = cudaMemsetAsync(gmax_bits, 0, 4 * sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  QuantPtrs p{sp_codes, meta, sp_sf, r_codes, r_sf};
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  const __nv_bfloat16* Gb = static_cast<const __nv_bfloat16*>(gamma);

  const int rpc = fused_rows_per_cta(K);
  if (Tp > 0 && rpc > 0) {
    const int threads = rpc * (K >> 5);
    const int ctas = (Tp + rpc - 1) / rpc;
    if (ctas <= fused_max_ctas(sharq_mode, threads)) {
      void* args[] = {(void*)&Xb, (void*)&Gb, (void*)&eps, (void*)&row_index, (void*)&T, (void*)&Tp, (void*)&K,
                      (void*)&rpc, (void*)&inv_rms, (void*)&gmax_bits, (void*)&s_g, (void*)&p};
      const void* fn = sharq_mode ? reinterpret_cast<const void*>(prep_fused_kernel<true>)
                                  : reinterpret_cast<const void*>(prep_fused_kernel<false>);
      e = cudaLaunchCooperativeKernel(fn, dim3(ctas), dim3(threads), args, 0, stream);
      if (e == cudaSuccess) return cudaSuccess;
      cudaGetLastError();  // fall back to the two-launch form below
    }
  }

  if (T > 0) {
    prep_stats_kernel<<<T, kStatsThreads, 0, stream>>>(Xb, Gb, eps, row_index, K, inv_rms, gmax_bits);
  }
  const long long n = (long long)Tp * (K >> 5);
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

}  // namespace sharq

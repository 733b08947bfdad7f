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
#include "sharq_device.cuh"

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

struct QuantPtrs {
  uint8_t* sp_codes;
  uint8_t* meta;
  uint8_t* sp_sf;
  uint8_t* r_codes;
  uint8_t* r_sf;
};

// max over the `width` adjacent lanes of an aligned lane group
__device__ __forceinline__ float group_max(float v, int width) {
  for (int o = 1; o < width; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Keep mask of one 4:8 in-pairs run: bit p set = pair p kept.  Pair p is
// kept iff fewer than two pairs beat it, where q beats p if its score is
// larger, or equal with q < p; the six pairwise comparisons give every rank.
__device__ __forceinline__ uint32_t keep_mask4(const float (&sc)[4]) {
  const int c01 = sc[1] > sc[0], c02 = sc[2] > sc[0], c03 = sc[3] > sc[0];
  const int c12 = sc[2] > sc[1], c13 = sc[3] > sc[1], c23 = sc[3] > sc[2];
  const int r0 = c01 + c02 + c03;
  const int r1 = (1 - c01) + c12 + c13;
  const int r2 = (1 - c02) + (1 - c12) + c23;
  const int r3 = (1 - c03) + (1 - c13) + (1 - c23);
  return (uint32_t)(r0 < 2) | ((uint32_t)(r1 < 2) << 1) | ((uint32_t)(r2 < 2) << 2) | ((uint32_t)(r3 < 2) << 3);
}

// one byte of two E2M1 codes -> their values (exact), low nibble first
__device__ __forceinline__ float2 e2m1x2_values(uint32_t byte) {
  uint32_t h2;
  asm("{\n\t.reg .b8 q;\n\tcvt.u8.u32 q, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, q;\n\t}" : "=r"(h2) : "r"(byte));
  return __half22float2(*reinterpret_cast<__half2*>(&h2));
}

// Quantize NC consecutive runs of 8 logical K of row t, held in registers
// (x[8*c + e] = run c, element e), starting at run index c0 of the row.
// NC = 4: every block is inside the thread.  NC = 1, 2: the 32-K block spans
// 4 / NC adjacent lanes and (NC = 1) the 16-K block 2 lanes; all 32 lanes of
// the warp must call it then (warp shuffles).
template <int NC, bool kSharq>
__device__ __forceinline__ void quant_runs(const float (&x)[8 * NC], int t, int c0, int K, float s, float six_s,
                                           const QuantPtrs& out, bool store = true) {
  const int KS = K >> 8;
  const int r = t & 127;
  float res[8 * NC];
#pragma unroll
  for (int i = 0; i < 8 * NC; ++i) res[i] = x[i];

  if (kSharq) {
    // --- 4:8 in-pairs mask per run: keep the 2 of 4 pairs with the largest max|x|
    float v[4 * NC];
    uint32_t km[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float sc[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) sc[p] = fmaxf(fabsf(x[8 * c + 2 * p]), fabsf(x[8 * c + 2 * p + 1]));
      km[c] = keep_mask4(sc);
      const bool k0 = km[c] & 1u, k1 = km[c] & 2u, k3 = km[c] & 8u;
      // lowest kept pair (0..2) and highest kept pair (1..3)
      const float* xc = x + 8 * c;
      v[4 * c + 0] = k0 ? xc[0] : (k1 ? xc[2] : xc[4]);
      v[4 * c + 1] = k0 ? xc[1] : (k1 ? xc[3] : xc[5]);
      v[4 * c + 2] = k3 ? xc[6] : ((km[c] & 4u) ? xc[4] : xc[2]);
      v[4 * c + 3] = k3 ? xc[7] : ((km[c] & 4u) ? xc[5] : xc[3]);
    }
    // --- backbone NVFP4: one scale per 32 logical K (4 runs = 16 kept values)
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 4 * NC; ++i) am = fmaxf(am, fabsf(v[i]));
    if (NC < 4) am = group_max(am, 4 / NC);
    const BlockScale bs = block_scale(am, six_s, s);
    uint32_t cb[2 * NC];  // code bytes: kept values (2i, 2i+1)
#pragma unroll
    for (int i = 0; i < 2 * NC; ++i) cb[i] = cvt_e2m1x2(__fmul_rn(v[2 * i], bs.inv), __fmul_rn(v[2 * i + 1], bs.inv));
    // --- residual R = Xn - dequant(backbone) at kept positions (exact fp32)
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float2 lo2 = e2m1x2_values(cb[2 * c]), hi2 = e2m1x2_values(cb[2 * c + 1]);
      const float t0 = __fmul_rn(__fmul_rn(lo2.x, bs.dec), s), t1 = __fmul_rn(__fmul_rn(lo2.y, bs.dec), s);
      const float t2 = __fmul_rn(__fmul_rn(hi2.x, bs.dec), s), t3 = __fmul_rn(__fmul_rn(hi2.y, bs.dec), s);
      const uint32_t m = km[c];
      const bool k0 = m & 1u, k1 = m & 2u, k2 = m & 4u, k3 = m & 8u;
      // pair p holds (t0,t1) if it is the lowest kept pair, (t2,t3) if the highest
      float* rc = res + 8 * c;
      if (k0) { rc[0] = __fsub_rn(rc[0], t0); rc[1] = __fsub_rn(rc[1], t1); }
      if (k1) { rc[2] = __fsub_rn(rc[2], k0 ? t2 : t0); rc[3] = __fsub_rn(rc[3], k0 ? t3 : t1); }
      if (k2) { rc[4] = __fsub_rn(rc[4], k3 ? t0 : t2); rc[5] = __fsub_rn(rc[5], k3 ? t1 : t3); }
      if (k3) { rc[6] = __fsub_rn(rc[6], t2); rc[7] = __fsub_rn(rc[7], t3); }
    }
    // --- stores: per run 2 bytes of kept codes, one metadata nibble
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int g = c0 + c;               // run index in the row
      const int kt = g >> 5, w = g & 31;  // K tile, run within the 256-K tile
      const size_t tile = (size_t)(t >> 7) * KS + kt;
      if (store)
        *reinterpret_cast<uint16_t*>(out.sp_codes + tile * kSpTile + sp_chunk_off(r, w >> 3) + 2 * (w & 7)) =
            (uint16_t)(cb[2 * c] | (cb[2 * c + 1] << 8));
      const uint32_t m = km[c];
      const uint32_t nib = (uint32_t)((__ffs(m) - 1) | ((31 - __clz(m)) << 2));
      if (NC == 1) {
        const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
        if (store && (w & 1) == 0) out.meta[tile * kMetaTile + r * 16 + (w >> 1)] = (uint8_t)(nib | (other << 4));
      } else if (store && (c & 1) == 0) {
        const uint32_t m2 = km[c + 1 < NC ? c + 1 : c];
        const uint32_t other = (uint32_t)((__ffs(m2) - 1) | ((31 - __clz(m2)) << 2));
        out.meta[tile * kMetaTile + r * 16 + (w >> 1)] = (uint8_t)(nib | (other << 4));
      }
      if (store && (w & 3) == 0) out.sp_sf[tile * kSf32Tile + sf_off(r, w >> 4, (w >> 2) & 3)] = (uint8_t)bs.sb;
    }
  }

  // --- dense NVFP4 of R (or of Xn in NVFP4 mode): 16-element blocks
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    if (NC > 1 && (c & 1)) continue;  // the even run handles its block of two runs
    const int nr = NC == 1 ? 1 : 2;   // runs of this block held by this thread
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8 * nr; ++i) am = fmaxf(am, fabsf(res[8 * c + i]));
    if (NC == 1) am = group_max(am, 2);
    const BlockScale bs = block_scale(am, six_s, s);
#pragma unroll
    for (int h = 0; h < nr; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        word |= cvt_e2m1x2(__fmul_rn(res[8 * (c + h) + 2 * i], bs.inv), __fmul_rn(res[8 * (c + h) + 2 * i + 1], bs.inv))
                << (8 * i);
      const int g = c0 + c + h;
      const int kt = g >> 5, w = g & 31;
      const size_t tile = (size_t)(t >> 7) * KS + kt;
      if (store) {
        *reinterpret_cast<uint32_t*>(out.r_codes + tile * kCodesTile + codes_chunk_off(r, w >> 2) + 4 * (w & 3)) =
            word;
        if ((w & 1) == 0) out.r_sf[tile * kSf16Tile + sf_off(r, w >> 3, (w >> 1) & 3)] = (uint8_t)bs.sb;
      }
    }
  }
}

// load NC runs of 8 (one 16-byte load each) and normalise them
template <int NC>
__device__ __forceinline__ void load_runs(float (&x)[8 * NC], const __nv_bfloat16* X, int src, int K, int c0) {
  if (src >= 0) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)src * K) + c0;
    uint4 raw[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) raw[c] = xr[c];
#pragma unroll
    for (int c = 0; c < NC; ++c) bf16x8_to_float(raw[c], x + 8 * c);
  } else {
#pragma unroll
    for (int i = 0; i < 8 * NC; ++i) x[i] = 0.0f;
  }
}

template <int NC>
__device__ __forceinline__ void normalise_runs(float (&x)[8 * NC], const __nv_bfloat16* gamma, int c0, float inv) {
  const uint4* gr = reinterpret_cast<const uint4*>(gamma) + c0;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    float g[8];
    bf16x8_to_float(gr[c], g);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[8 * c + e] = norm_one(x[8 * c + e], inv, g[e]);
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

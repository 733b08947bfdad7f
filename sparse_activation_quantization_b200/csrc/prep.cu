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
#include "strip.cuh"

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

constexpr int kRowThreads = 256;
constexpr int kRowChunk = 8;  // 16-byte loads in flight per lane

// bf16 (upper / lower half of a word) -> its value times 2^128 as a double,
// by moving the exponent and mantissa fields (no conversion unit): exact for
// normal numbers.  Zeros and subnormals come out as (1 + m/128) * 2^-127
// (times 2^128) instead; see prep_rowstats_kernel for why that is harmless.
__device__ __forceinline__ double bf16_hi_x2p128(uint32_t w) {
  return __hiloint2double((int)(((w >> 3) & 0x0FFFE000u) | 0x40000000u), 0);
}
__device__ __forceinline__ double bf16_lo_x2p128(uint32_t w) {
  return __hiloint2double((int)(((w << 13) & 0x0FFFE000u) | 0x40000000u), 0);
}

// v[u] (vector c0 + 32 u of a row, zeros past its end) <- h, and h stored to
// hr (the same vectors of the output) when hr is given
template <int N>
__device__ __forceinline__ void row_epi(uint4 (&v)[N], const uint4* rr, uint4* hr, int c0, int nv, int kind) {
  uint4 r[N];
#pragma unroll
  for (int u = 0; u < N; ++u) r[u] = c0 + 32 * u < nv ? rr[c0 + 32 * u] : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int u = 0; u < N; ++u) v[u] = epi8(v[u], r[u], kind);
  if (hr) {
#pragma unroll
    for (int u = 0; u < N; ++u)
      if (c0 + 32 * u < nv) hr[c0 + 32 * u] = v[u];
  }
}

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Wide form, first launch: one warp per row (rows strided over a grid that
// fits the GPU), 8 loads of 16 bytes in flight per lane.
//   RMSNorm rows: float64 sum of squares -> 1/rms, then max |Xn| (Xn
//   recomputed from L1/L2 as in the quantizer: bf16(f32(f32(x/rms) g))).
//   Rows without RMSNorm: max |x| on packed bf16 bits.
// With an epilogue (kEpi: the residual add or the SwiGLU product) the rows
// are h: the first pass forms h (4 vectors of X and 4 of B in flight per
// lane) and, when an output is given, stores it there; the second pass and
// the quantizer launch then read h alone.  Each element of h is stored and
// re-read by the lane that formed it.
// The device-wide max goes to gmax_bits[0] with one atomicMax per CTA.
// Sum of squares: each square of a bf16 value is exact in float64, and the
// values enter scaled by 2^128 (bf16_*_x2p128, squares scaled by 2^256,
// undone exactly at the end).  A zero or subnormal element then adds at most
// 2^-252 (unscaled) instead of its true square, i.e. at most K 2^-252 per
// row -- far below one ulp of mean(x^2) + eps for any eps >= 2^-60, where
// the result is that of an exact-input float64 sum in this lane order.  For
// eps < 2^-60 (`exact`) the elements are converted exactly instead.
template <bool kGamma, bool kEpi>
__global__ void __launch_bounds__(kRowThreads) prep_rowstats_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma, float eps,
    const int* __restrict__ row_index, int T, int K, int exact, float* __restrict__ inv_rms,
    unsigned int* __restrict__ gmax_bits, Epi rs) {
  constexpr int kC = kEpi ? kRowChunk / 2 : kRowChunk;  // vectors of the row in flight per lane
  __shared__ uint32_t wmax[kRowThreads / 32];
  // the strip quantizer, launched as this grid's programmatic dependent, may
  // start its set-up now; it waits for this grid before reading its results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = gridDim.x * (kRowThreads / 32);
  const int nv = K >> 3;  // 16-byte vectors per row
  uint32_t mx = 0;        // max |Xn| so far: bf16 bit patterns, one per half
  for (int t = blockIdx.x * (kRowThreads / 32) + warp; t < T; t += nw) {
    const int src = row_index ? row_index[t] : t;  // warp-uniform
    if (src < 0) {  // zero padding row of the grouped form: Xn = 0
      if (lane == 0) inv_rms[t] = kGamma ? (float)(1.0 / sqrt((double)eps)) : 1.0f;
      continue;
    }
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)src * K);
    const uint4* rr = kEpi ? reinterpret_cast<const uint4*>(rs.B + (size_t)src * K) : nullptr;
    uint4* hr = kEpi && rs.H ? reinterpret_cast<uint4*>(rs.H + (size_t)src * K) : nullptr;
    if (kGamma) {
      double acc0 = 0.0, acc1 = 0.0;
      for (int c0 = lane; c0 < nv; c0 += 32 * kC) {
        uint4 v[kC];
#pragma unroll
        for (int u = 0; u < kC; ++u) v[u] = c0 + 32 * u < nv ? xr[c0 + 32 * u] : make_uint4(0, 0, 0, 0);
        if (kEpi) row_epi<kC>(v, rr, hr, c0, nv, rs.kind);
        if (!exact) {
#pragma unroll
          for (int u = 0; u < kC; ++u) {
            if (c0 + 32 * u < nv) {
              const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const double dl = bf16_lo_x2p128(w[i]), dh = bf16_hi_x2p128(w[i]);
                acc0 = fma(dl, dl, acc0);
                acc1 = fma(dh, dh, acc1);
              }
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < kC; ++u) {
            float f[8];
            bf16x8_to_float(v[u], f);  // zero-filled beyond the row: adds 0
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              acc0 = fma((double)f[e], (double)f[e], acc0);
              acc1 = fma((double)f[e + 1], (double)f[e + 1], acc1);
            }
          }
        }
      }
      double acc = acc0 + acc1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const double ss = exact ? acc : acc * 0x1p-256;
      const float inv = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
      if (lane == 0) inv_rms[t] = inv;
      const f2_t inv2 = f2_make(inv, inv);
      const uint4* gr = reinterpret_cast<const uint4*>(gamma);
      const uint4* sr = hr ? hr : xr;  // h, once stored
      for (int c0 = lane; c0 < nv; c0 += 32 * kC) {
        uint4 v[kC], g[kC];
#pragma unroll
        for (int u = 0; u < kC; ++u) {
          const bool in = c0 + 32 * u < nv;
          v[u] = in ? sr[c0 + 32 * u] : make_uint4(0, 0, 0, 0);
          g[u] = in ? gr[c0 + 32 * u] : make_uint4(0, 0, 0, 0);
        }
        if (kEpi && !hr) row_epi<kC>(v, rr, nullptr, c0, nv, rs.kind);
#pragma unroll
        for (int u = 0; u < kC; ++u) {
          const uint32_t xw[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          const uint32_t gw[4] = {g[u].x, g[u].y, g[u].z, g[u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t n =
                bf16x2_from_f2(f2_mul(f2_mul(f2_from_bf16x2(xw[i]), inv2), f2_from_bf16x2(gw[i])));
            mx = vmax_u16x2(mx, n & 0x7FFF7FFFu);
          }
        }
      }
    } else {
      for (int c0 = lane; c0 < nv; c0 += 32 * kC) {
        uint4 v[kC];
#pragma unroll
        for (int u = 0; u < kC; ++u) v[u] = c0 + 32 * u < nv ? xr[c0 + 32 * u] : make_uint4(0, 0, 0, 0);
        if (kEpi) row_epi<kC>(v, rr, hr, c0, nv, rs.kind);
#pragma unroll
        for (int u = 0; u < kC; ++u) {
          mx = vmax_u16x2(mx, v[u].x & 0x7FFF7FFFu);
          mx = vmax_u16x2(mx, v[u].y & 0x7FFF7FFFu);
          mx = vmax_u16x2(mx, v[u].z & 0x7FFF7FFFu);
          mx = vmax_u16x2(mx, v[u].w & 0x7FFF7FFFu);
        }
      }
      if (lane == 0) inv_rms[t] = 1.0f;
    }
  }
  // CTA max -> device-wide max (non-negative floats order as their bits)
  uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t cm = 0;
#pragma unroll
    for (int w = 0; w < kRowThreads / 32; ++w) cm = max(cm, wmax[w]);
    if (cm) atomicMax(gmax_bits, cm << 16);
  }
}

// Wide form of the SwiGLU prep without RMSNorm when h is written out: one
// elementwise pass over the whole tensor forms h = bf16(silu_bf16(gate) * up),
// stores it and takes the device-wide max |h|; the strip quantizer then reads
// h alone (from L2 when it fits).  Every thread works on independent 16-byte
// vectors, two in flight, where the statistics kernel's row loop keeps too few
// loads in flight to cover the SiLU's extra work.  h may alias up: each
// element is read and then written by the same thread.
constexpr int kEwThreads = 256;
__global__ void __launch_bounds__(kEwThreads) prep_swiglu_h_kernel(
    const __nv_bfloat16* __restrict__ G, const __nv_bfloat16* U, __nv_bfloat16* H, size_t n_vec, int T,
    float* __restrict__ inv_rms, unsigned int* __restrict__ gmax_bits, int stats) {
  __shared__ uint32_t wmax[kEwThreads / 32];
  const uint4* g = reinterpret_cast<const uint4*>(G);
  const uint4* u = reinterpret_cast<const uint4*>(U);
  uint4* h = reinterpret_cast<uint4*>(H);
  const size_t stride = (size_t)gridDim.x * kEwThreads;
  size_t i = (size_t)blockIdx.x * kEwThreads + threadIdx.x;
  uint32_t mx = 0;  // max |h| so far: bf16 bit patterns, one per half
  auto fold = [&](const uint4& v) {
    mx = vmax_u16x2(mx, v.x & 0x7FFF7FFFu);
    mx = vmax_u16x2(mx, v.y & 0x7FFF7FFFu);
    mx = vmax_u16x2(mx, v.z & 0x7FFF7FFFu);
    mx = vmax_u16x2(mx, v.w & 0x7FFF7FFFu);
  };
  for (; i + stride < n_vec; i += 2 * stride) {
    const uint4 a0 = g[i], b0 = u[i], a1 = g[i + stride], b1 = u[i + stride];
    const uint4 h0 = epi8(a0, b0, kEpiSiluMul), h1 = epi8(a1, b1, kEpiSiluMul);
    h[i] = h0;
    h[i + stride] = h1;
    fold(h0);
    fold(h1);
  }
  if (i < n_vec) {
    const uint4 h0 = epi8(g[i], u[i], kEpiSiluMul);
    h[i] = h0;
    fold(h0);
  }
  if (!stats) return;  // h only: the prep that follows takes its own statistics
  for (size_t t = (size_t)blockIdx.x * kEwThreads + threadIdx.x; t < (size_t)T; t += stride) inv_rms[t] = 1.0f;
  // CTA max -> device-wide max (non-negative floats order as their bits)
  uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t cm = 0;
#pragma unroll
    for (int w = 0; w < kEwThreads / 32; ++w) cm = max(cm, wmax[w]);
    if (cm) atomicMax(gmax_bits, cm << 16);
  }
}

// Allow the next kernel in the stream (the GEMM, launched as a programmatic
// dependent) to start its set-up and weight loads now; it waits for this
// grid's completion (griddepcontrol.wait) before reading our outputs.
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Words of the act scalar block (gmax_bits) that the prep kernels use:
//   0  device-wide max |Xn| (float bits)    1  grid-barrier arrivals
//   2  departures                           3  error word of the last call
//                                              (read by sharq_linear)
//   4  error of the call in flight          5  fault-injection word (tests)
// Words 0..2 and 4 are zero at rest.  A CTA whose bounded barrier wait runs
// out records into word 4; only the last CTA out moves word 4 into word 3,
// so a CTA that starts late can neither erase nor miss this call's error.
enum : int { kSyncMax = 0, kSyncArrive = 1, kSyncDepart = 2, kSyncErr = 3, kSyncPending = 4, kSyncInject = 5 };

// Last CTA out publishes this call's error word and resets the device-wide
// max and the counters, so the next sharq_prep on this buffer starts from
// zero without a memset.  Called by thread 0 of every CTA at its end, after
// the CTA has read the max (so the reset cannot race a reader) and after any
// error it recorded (atomics, complete before the departure is counted).
__device__ __forceinline__ void depart_and_reset(unsigned int* sync) {
  if (atomicAdd(sync + kSyncDepart, 1u) == gridDim.x - 1) {
    sync[kSyncErr] = atomicExch(sync + kSyncPending, 0u);
    sync[kSyncMax] = 0u;
    sync[kSyncArrive] = 0u;
    sync[kSyncDepart] = 0u;
    __threadfence();
  }
}

constexpr int kStripThreads = 256;

// Wide form, second launch: one thread per 32-K strip of a row.  Warp w of
// the grid owns strip group w % G (32 adjacent strips = 2 KB of a row, G
// groups per row) and walks the rows T - 1 - w / G, T - 1 - w / G - nw / G,
// ... (nw, the warps used, is a multiple of G), so its lanes load and unpack
// gamma once
// and prefetch the next row's 64 bytes while quantizing the current one.
template <bool kSharq, bool kGamma>
__global__ void __launch_bounds__(kStripThreads) prep_strip_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma,
    const int* __restrict__ row_index, int T, int K, int nw, const float* __restrict__ inv_rms,
    unsigned int* __restrict__ gmax_bits, float* __restrict__ s_g_out, QuantPtrs out, Epi rs) {
  __shared__ float2 tab[128];
  __shared__ uint32_t msel[16];
  allow_dependents();
  // launched as a programmatic dependent of the statistics grid: the max,
  // 1/rms and (with an epilogue) h are read only once it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float gmax = __uint_as_float(*(volatile const unsigned int*)gmax_bits);
  const float s = gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s;  // published even when there are no rows
  strip_tables_init(s, tab, msel);
  __syncthreads();
  const StripCtx ctx = strip_ctx(s, tab, msel);
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kStripThreads / 32) + (threadIdx.x >> 5);
  const int nstrips = K >> 5, G = (nstrips + 31) >> 5, KS = K >> 8;
  if (gw < nw && T > 0) {
    const int j = (gw % G) * 32 + lane;
    const bool active = j < nstrips;
    const int rstride = nw / G;
    f2_t gm[16];
    if (kGamma && active) {
      const uint4* gp = reinterpret_cast<const uint4*>(gamma + 32 * (size_t)j);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 v = gp[u];
        gm[4 * u] = f2_from_bf16x2(v.x);
        gm[4 * u + 1] = f2_from_bf16x2(v.y);
        gm[4 * u + 2] = f2_from_bf16x2(v.z);
        gm[4 * u + 3] = f2_from_bf16x2(v.w);
      }
    }
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    // Rows are walked from the last one back: the statistics launch read the
    // last rows most recently, so when X is larger than L2 the first rows
    // this launch reads are still there.  t counts walked rows, T - 1 - t is
    // the row.
    int t = gw / G;  // < T: the host uses at most T warps per strip group
    int src = row_index ? row_index[T - 1 - t] : T - 1 - t;
    uint4 cur[4];
    float inv = 1.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      cur[u] = (active && src >= 0) ? reinterpret_cast<const uint4*>(X + (size_t)src * K + 32 * (size_t)j)[u] : z4;
    if (rs.kind && active && src >= 0) apply_epi<4>(cur, (size_t)src * K + 32 * (size_t)j, rs);
    if (kGamma) inv = inv_rms[T - 1 - t];
    while (t < T) {
      // prefetch the next row of this warp
      const int tn = t + rstride;
      int srcn = -1;
      uint4 nxt[4] = {z4, z4, z4, z4};
      float invn = 1.0f;
      if (tn < T) {
        srcn = row_index ? row_index[T - 1 - tn] : T - 1 - tn;
        if (active && srcn >= 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) nxt[u] = reinterpret_cast<const uint4*>(X + (size_t)srcn * K + 32 * (size_t)j)[u];
          if (rs.kind) apply_epi<4>(nxt, (size_t)srcn * K + 32 * (size_t)j, rs);
        }
        if (kGamma) invn = inv_rms[T - 1 - tn];
      }
      if (active) {
        f2_t P[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          P[4 * u] = f2_from_bf16x2(cur[u].x);
          P[4 * u + 1] = f2_from_bf16x2(cur[u].y);
          P[4 * u + 2] = f2_from_bf16x2(cur[u].z);
          P[4 * u + 3] = f2_from_bf16x2(cur[u].w);
        }
        if (kGamma && src >= 0) {
          const f2_t inv2 = f2_make(inv, inv);
#pragma unroll
          for (int i = 0; i < 16; ++i) P[i] = f2_norm(P[i], inv2, gm[i]);
        }
        quant_strip<kSharq>(P, T - 1 - t, j, KS, ctx, out);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
      src = srcn;
      inv = invn;
      t = tn;
    }
  }
  if (threadIdx.x == 0) depart_and_reset(gmax_bits);
}

// Two-launch form of the Table-5 operand kinds (Dense+Dense, Sparse+Sparse):
// after prep_rowstats_kernel, one thread per 32 consecutive K (four runs,
// every block inside the thread), flat over rows.
constexpr int kRunsThreads = 256;
template <int kKind>
__global__ void __launch_bounds__(kRunsThreads) prep_runs_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma,
    const int* __restrict__ row_index, int T, int K, const float* __restrict__ inv_rms,
    unsigned int* __restrict__ gmax_bits, float* __restrict__ s_g_out, QuantPtrs out, Epi rs) {
  __shared__ float gmax_sh;
  allow_dependents();
  const int segs = K >> 5;
  const long long gid = (long long)blockIdx.x * kRunsThreads + threadIdx.x;
  if (threadIdx.x == 0) gmax_sh = __uint_as_float(*(volatile const unsigned int*)gmax_bits);
  __syncthreads();
  const float gmax = gmax_sh;
  // MX formats have no tensor scale
  const float s = kind_is_mx(kKind) ? 1.0f : (gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f);
  if (gid == 0) *s_g_out = s;
  // Every lane of the warp runs the quantizer (an MXFP4 backbone block spans
  // two lanes, reduced with warp shuffles); lanes past the end work on zeros
  // and store nothing.  Active lanes come in groups of 8 (K / 32 is a
  // multiple of 8), so a block never mixes active and idle lanes.
  const bool active = gid < (long long)T * segs;
  const long long g = active ? gid : 0;
  const int t = (int)(g / segs);
  const int c0 = (int)(g - (long long)t * segs) * 4;
  const int src = active ? (row_index ? row_index[t] : t) : -1;
  float x[32];
  load_runs<4>(x, X, src, K, c0, rs);
  if (gamma && src >= 0) normalise_runs<4>(x, gamma, c0, inv_rms[t]);
  quant_runs<4, kKind>(x, t, c0, K, s, __fmul_rn(6.0f, s), out, active);
  if (threadIdx.x == 0) depart_and_reset(gmax_bits);
}

// ---------------------------------------------------------------------------
// Single-launch form (cooperative grid; whole rows inside a CTA).
constexpr int kFusedMaxThreads = 1024;
constexpr int kMaxClusterCtas = 16;  // cluster form: at most 16 CTAs (non-portable size above 8)
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

template <int NC>
constexpr int fused_max_threads() { return NC == 4 ? 640 : kFusedMaxThreads; }

template <int NC, int kKind, bool kPerToken = false>
__global__ void __launch_bounds__(fused_max_threads<NC>()) prep_fused_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ gamma, float eps,
    const int* __restrict__ row_index, int T, int Tp, int K, int rows_per_cta, float* __restrict__ inv_rms,
    unsigned int* sync, float* __restrict__ s_g_out, QuantPtrs out, Epi rs, int cluster) {
  __shared__ double wsum[kFusedMaxThreads / 32];
  __shared__ float cmax[kMaxClusterCtas];  // cluster form: every CTA's max
  __shared__ float wmax[kFusedMaxThreads / 32];
  __shared__ float gmax_sh;
  PREP_TRACE(0);
  allow_dependents();
  // cluster form: announce this CTA (its shared memory exists) before any
  // peer stores into it; the matching wait comes just before those stores
  if (cluster) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // forms without a grid barrier cannot time out: this call's error word is 0
  if ((kPerToken || cluster || gridDim.x == 1) && blockIdx.x == 0 && threadIdx.x == 0) sync[kSyncErr] = 0u;
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
  load_runs<NC>(x, X, src, K, c0, rs);
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

  // CTA max |Xn| -> device-wide max (per-token: the row max)
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8 * NC; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) wmax[warp] = a;
  __syncthreads();
  if (kPerToken) {
    // every row is its own tensor: s_t from the row's warps, no grid barrier
    float m = 0.0f;
    for (int w = 0; w < wpr; ++w) m = fmaxf(m, wmax[rl * wpr + w]);
    const float s = m > 0.0f ? __fdiv_rn(m, kGlobalDiv) : 1.0f;
    if (live && li == 0) s_g_out[t] = s;
    if (live) quant_runs<NC, kKind>(x, t, c0, K, s, __fmul_rn(6.0f, s), out, has);
    return;
  }
  if (cluster) {
    // The grid is one thread-block cluster: every CTA writes its max into
    // every CTA's shared memory, and one hardware cluster barrier (release /
    // acquire) replaces the global-memory grid barrier.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every peer has started
    if (threadIdx.x == 0) {
      float m = 0.0f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
      const uint32_t dst = smem_u32(&cmax[blockIdx.x]);
      for (uint32_t r = 0; r < gridDim.x; ++r) {
        const uint32_t a = mapa_shared(dst, r);
        asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(m) : "memory");
      }
    }
    cluster_sync_all();
    if (threadIdx.x == 0) {
      float m = 0.0f;
      for (int r = 0; r < (int)gridDim.x; ++r) m = fmaxf(m, cmax[r]);
      gmax_sh = m;
      PREP_TRACE(2);
    }
  } else if (threadIdx.x == 0) {
    float m = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
    if (gridDim.x == 1) {
      gmax_sh = m;  // one CTA holds the whole tensor: no grid barrier
    } else {
      // a test can name one CTA (index + 1) that never arrives, so that every
      // CTA's bounded wait runs out; zero in normal use
      const unsigned skip = *(volatile unsigned int*)(sync + kSyncInject);
      if (skip != blockIdx.x + 1u) {
        atomicMax(sync + kSyncMax, __float_as_uint(m));
        // arrival with release semantics: our max is visible before the count
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(sync + kSyncArrive) : "memory");
      }
      PREP_TRACE(1);
      // grid barrier: every CTA has published its max (bounded spin)
      const uint64_t deadline = globaltimer_ns() + kBarrierLimitNs;
      unsigned seen = 0;
      do {
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(sync + kSyncArrive) : "memory");
        if (seen >= gridDim.x) break;
        if (globaltimer_ns() > deadline) {
          atomicCAS(reinterpret_cast<int*>(sync + kSyncPending), 0, -5);  // SHARQ_ERR_TIMEOUT
          break;
        }
      } while (true);
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      gmax_sh = __uint_as_float(*(volatile unsigned int*)(sync + kSyncMax));
    }
    PREP_TRACE(2);
  }
  __syncthreads();
  const float gmax = gmax_sh;
  // MX formats have no tensor scale
  const float s = kind_is_mx(kKind) ? 1.0f : (gmax > 0.0f ? __fdiv_rn(gmax, kGlobalDiv) : 1.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s;
  // rows past T: whole warps (rows span whole warps), so they can skip
  if (live) quant_runs<NC, kKind>(x, t, c0, K, s, __fmul_rn(6.0f, s), out, has);
  if (threadIdx.x == 0 && gridDim.x > 1 && !cluster) depart_and_reset(sync);
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

template <int NC, int kKind>
int fused_max_ctas_t(int threads) {
  static int cache[kFusedMaxThreads + 1][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return 0;
  int& c = cache[threads][dev];
  if (c == 0) {
    prefer_max_shared(prep_fused_kernel<NC, kKind>);
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prep_fused_kernel<NC, kKind>, threads, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    c = per_sm * sms > 0 ? per_sm * sms : -1;
  }
  return c > 0 ? c : 0;
}

template <int NC, int kKind>
cudaError_t try_fused(const __nv_bfloat16* Xb, const __nv_bfloat16* Gb, float eps, const int* row_index, int T,
                      int Tp, int K, float* inv_rms, unsigned int* sync, float* s_g, QuantPtrs p, Epi rs,
                      cudaStream_t stream, bool* launched) {
  *launched = false;
  const int tpr = (((K >> 3) / NC) + 31) & ~31;
  // Small tensors: CTAs of about 512 threads (larger ones would keep the
  // GEMM launched as this grid's programmatic dependent off their SMs); a
  // single CTA needs no barrier at all, and 2-16 CTAs run as one thread-block
  // cluster whose hardware barrier replaces the global-memory grid barrier.
  {
    const int rpc = 512 / tpr > 0 ? 512 / tpr : 1;
    const int ctas = rpc > 0 ? (T + rpc - 1) / rpc : 0;
    if (ctas >= 1 && ctas <= kMaxClusterCtas) {
      const int threads = (ctas == 1 ? T : rpc) * tpr;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(ctas);
      cfg.blockDim = dim3(threads);
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      if (ctas > 1) {
        static bool nonportable[64] = {};
        int dev = 0;
        if (ctas > 8 && cudaGetDevice(&dev) == cudaSuccess && dev < 64 && !nonportable[dev]) {
          cudaFuncSetAttribute(prep_fused_kernel<NC, kKind>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
          cudaGetLastError();
          nonportable[dev] = true;
        }
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)ctas;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
      }
      cudaError_t e = cudaLaunchKernelEx(&cfg, prep_fused_kernel<NC, kKind>, Xb, Gb, eps, row_index, T, Tp, K,
                                         ctas == 1 ? T : rpc, inv_rms, sync, s_g, p, rs, ctas > 1 ? 1 : 0);
      if (e == cudaSuccess) {
        *launched = true;
        return cudaSuccess;
      }
      cudaGetLastError();  // e.g. no GPC can host the cluster: the grid-barrier form below
    }
  }
  int rpc = 512 / tpr;
  rpc = rpc < 1 ? 1 : rpc;
  const int threads = rpc * tpr;
  const int ctas = (T + rpc - 1) / rpc;
  if (ctas > fused_max_ctas_t<NC, kKind>(threads)) return cudaSuccess;
  // A cooperative launch: the CTAs wait for one another at the grid barrier,
  // so they must all be resident at once, which a cooperative launch
  // guarantees (or refuses, and the two-launch form below runs instead).  The
  // GEMM that follows as a programmatic dependent can start only after every
  // CTA of this grid has started (each triggers at entry), so it cannot crowd
  // out a CTA that has not arrived at the barrier.  The barrier's spin is
  // bounded all the same.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute coop[1];
  coop[0].id = cudaLaunchAttributeCooperative;
  coop[0].val.cooperative = 1;
  cfg.attrs = coop;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prep_fused_kernel<NC, kKind>, Xb, Gb, eps, row_index, T, Tp, K, rpc,
                                     inv_rms, sync, s_g, p, rs, 0);
  if (e == cudaSuccess) *launched = true;
  else cudaGetLastError();  // fall back to the two-launch form
  return cudaSuccess;
}

// Per-token scales need no device-wide max: the single-launch kernel serves
// every T (CTAs are independent, so the grid need not fit the GPU).
template <int NC>
cudaError_t launch_per_token_nc(const __nv_bfloat16* Xb, const __nv_bfloat16* Gb, float eps, const int* row_index,
                                int T, int Tp, int K, float* inv_rms, unsigned int* sync, float* s_t, QuantPtrs p,
                                Epi rs, cudaStream_t stream) {
  const int tpr = (((K >> 3) / NC) + 31) & ~31;
  int rpc = 512 / tpr;
  rpc = rpc < 1 ? 1 : rpc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((T + rpc - 1) / rpc);
  cfg.blockDim = dim3(rpc * tpr);
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, prep_fused_kernel<NC, kKindSharq, true>, Xb, Gb, eps, row_index, T, Tp, K, rpc, inv_rms,
                            sync, s_t, p, rs, 0);
}

template <int kKind>
cudaError_t try_fused_any(const __nv_bfloat16* Xb, const __nv_bfloat16* Gb, float eps, const int* row_index, int T,
                          int Tp, int K, float* inv_rms, unsigned int* sync, float* s_g, QuantPtrs p, Epi rs,
                          cudaStream_t stream, bool* launched) {
  switch (fused_runs_per_thread(K)) {
    case 1: return try_fused<1, kKind>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, rs, stream,
                                          launched);
    case 2: return try_fused<2, kKind>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, rs, stream,
                                          launched);
    case 4: return try_fused<4, kKind>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, sync, s_g, p, rs, stream,
                                          launched);
    default: *launched = false; return cudaSuccess;
  }
}

// CTAs of `fn` resident per SM at `threads` threads (cached per device and
// kernel); the maximum shared-memory carveout is requested first so that an
// SM running them keeps room for a GEMM CTA launched as their dependent.
template <class F>
int resident_ctas(F* fn, int threads, int dev) {
  static F* fns[16] = {};
  static int cache[16][64] = {};
  int slot = 0;
  while (slot < 16 && fns[slot] && fns[slot] != fn) ++slot;
  if (slot == 16) return 1;
  if (!fns[slot]) fns[slot] = fn;
  if (cache[slot][dev] == 0) {
    prefer_max_shared(fn);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, 0) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 1;
    }
    cache[slot][dev] = n;
  }
  return cache[slot][dev];
}

}  // namespace

#ifdef SHARQ_TRACE
extern "C" int sharq_debug_set_trace_prep(void* p) {
  return cudaMemcpyToSymbol(g_trace_prep, &p, sizeof(p)) == cudaSuccess ? 0 : -4;
}
#endif

bool prep_per_token_supported(int K) { return fused_runs_per_thread(K) != 0; }

cudaError_t launch_prep(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp,
                        int K, int kind, bool per_token, float* inv_rms, float* s_g, unsigned int* gmax_bits,
                        uint8_t* sp_codes, uint8_t* meta, uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf,
                        uint8_t* r_meta, int epi_kind, const void* epi_b, void* epi_h, cudaStream_t stream) {
  // gmax_bits[0..3]: device-wide max, barrier arrivals, departures, error
  // word; zero at rest (the kernels reset them), so no memset is needed
  cudaError_t e = cudaSuccess;
  QuantPtrs p{sp_codes, meta, sp_sf, r_codes, r_sf, r_meta};
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  const __nv_bfloat16* Gb = static_cast<const __nv_bfloat16*>(gamma);
  const Epi rs{static_cast<const __nv_bfloat16*>(epi_b), static_cast<__nv_bfloat16*>(epi_h), epi_b ? epi_kind : kEpiNone};
  if (per_token) {  // s_g: Tp floats, one per row (SharQ mode only)
    if (T == 0) return cudaSuccess;
    switch (fused_runs_per_thread(K)) {
      case 1: return launch_per_token_nc<1>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs,
                                                stream);
      case 2: return launch_per_token_nc<2>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs,
                                                stream);
      case 4: return launch_per_token_nc<4>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs,
                                                stream);
      default: return cudaErrorInvalidValue;
    }
  }

  // SwiGLU without RMSNorm, h written out, and a tensor that one cluster of
  // the single-launch form holds (T <= 16 at K = 14336): h first, by the
  // elementwise pass spread over many CTAs, then the prep of h alone -- each
  // CTA of the single-launch form would otherwise evaluate its rows' SiLUs on
  // one SM.
  if (T > 0 && rs.kind == kEpiSiluMul && !Gb && rs.H && fused_runs_per_thread(K) != 0) {
    const int tpr = (((K >> 3) / fused_runs_per_thread(K)) + 31) & ~31;
    const int rpc = 512 / tpr > 0 ? 512 / tpr : 1;
    if ((T + rpc - 1) / rpc <= kMaxClusterCtas) {
      const size_t n_vec = (size_t)T * (size_t)(K >> 3);
      const unsigned grid = (unsigned)((n_vec + kEwThreads - 1) / kEwThreads);
      prep_swiglu_h_kernel<<<grid, kEwThreads, 0, stream>>>(Xb, rs.B, rs.H, n_vec, T, inv_rms, gmax_bits, 0);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      return launch_prep(rs.H, nullptr, eps, nullptr, T, Tp, K, kind, false, inv_rms, s_g, gmax_bits, sp_codes, meta,
                         sp_sf, r_codes, r_sf, r_meta, kEpiNone, nullptr, nullptr, stream);
    }
  }

  if (T > 0) {
    bool launched = false;
    switch (kind) {
      case kKindNvfp4:
        e = try_fused_any<kKindNvfp4>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                               &launched);
        break;
      case kKindSharq:
        e = try_fused_any<kKindSharq>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                               &launched);
        break;
      case kKindDenseDense:
        e = try_fused_any<kKindDenseDense>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                                           &launched);
        break;
      case kKindSparseSparse:
        e = try_fused_any<kKindSparseSparse>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                                             &launched);
        break;
      case kKindSharqMx:
        e = try_fused_any<kKindSharqMx>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                                        &launched);
        break;
      case kKindMxfp4:
        e = try_fused_any<kKindMxfp4>(Xb, Gb, eps, row_index, T, Tp, K, inv_rms, gmax_bits, s_g, p, rs, stream,
                                      &launched);
        break;
      default:
        return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (launched) return cudaSuccess;
  }

  // wide form: row statistics, then the strip quantizer
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const bool g = Gb != nullptr;
  const int exact = eps < 0x1p-60f ? 1 : 0;
  if (T > 0 && rs.kind == kEpiSiluMul && !g && rs.H) {
    // SwiGLU without RMSNorm, h written out: the elementwise first pass
    const size_t n_vec = (size_t)T * (size_t)(K >> 3);
    const int per_sm = resident_ctas(prep_swiglu_h_kernel, kEwThreads, dev);
    long long grid = (long long)((n_vec + kEwThreads - 1) / kEwThreads);
    if (grid > (long long)sms * per_sm) grid = (long long)sms * per_sm;
    prep_swiglu_h_kernel<<<(unsigned)grid, kEwThreads, 0, stream>>>(Xb, rs.B, rs.H, n_vec, T, inv_rms, gmax_bits, 1);
  } else if (T > 0) {
    auto rowstats_fn = g ? (rs.kind ? prep_rowstats_kernel<true, true> : prep_rowstats_kernel<true, false>)
                         : (rs.kind ? prep_rowstats_kernel<false, true> : prep_rowstats_kernel<false, false>);
    const int per_sm = resident_ctas(rowstats_fn, kRowThreads, dev);
    const int rows_per_cta = kRowThreads / 32;
    int grid = (T + rows_per_cta - 1) / rows_per_cta;
    if (grid > sms * per_sm) grid = sms * per_sm;
    rowstats_fn<<<grid, kRowThreads, 0, stream>>>(Xb, Gb, eps, row_index, T, K, exact, inv_rms, gmax_bits, rs);
  }
  // once the statistics launch has stored h, the quantizer reads h alone
  const __nv_bfloat16* Xq = rs.H ? rs.H : Xb;
  const Epi rq = rs.H ? Epi{} : rs;
  if (kind != kKindSharq && kind != kKindNvfp4) {
    const long long n = (long long)T * (K >> 5);
    const unsigned grid = n > 0 ? (unsigned)((n + kRunsThreads - 1) / kRunsThreads) : 1u;
#define SHARQ_RUNS(KIND) prep_runs_kernel<KIND><<<grid, kRunsThreads, 0, stream>>>(Xq, Gb, row_index, T, K, \
                                                                                inv_rms, gmax_bits, s_g, p, rq)
    switch (kind) {
      case kKindDenseDense: SHARQ_RUNS(kKindDenseDense); break;
      case kKindSparseSparse: SHARQ_RUNS(kKindSparseSparse); break;
      case kKindSharqMx: SHARQ_RUNS(kKindSharqMx); break;
      default: SHARQ_RUNS(kKindMxfp4); break;
    }
#undef SHARQ_RUNS
    return cudaGetLastError();
  }
  const bool sharq_mode = kind == kKindSharq;
  auto strip_fn = sharq_mode ? (g ? prep_strip_kernel<true, true> : prep_strip_kernel<true, false>)
                             : (g ? prep_strip_kernel<false, true> : prep_strip_kernel<false, false>);
  const int G = ((K >> 5) + 31) >> 5;  // strip groups (warps) per row
  const int max_warps = sms * resident_ctas(strip_fn, kStripThreads, dev) * (kStripThreads / 32);
  long long rows = max_warps / G;
  if (rows < 1) rows = 1;
  if (rows > T) rows = T;
  const int nw = (int)(rows * G);  // 0 when T == 0: one CTA still publishes s_g
  const int grid = nw > 0 ? (nw + kStripThreads / 32 - 1) / (kStripThreads / 32) : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kStripThreads);
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = T > 0 ? 1 : 0;  // T == 0: no statistics launch precedes it
  return cudaLaunchKernelEx(&cfg, strip_fn, Xq, Gb, row_index, T, K, nw, (const float*)inv_rms, gmax_bits, s_g, p, rq);
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
                                int K, int kind, bool per_token, float* s_g, uint8_t* sp_codes, uint8_t* meta,
                                uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf, uint8_t* r_meta,
                                unsigned int* err_out, cudaStream_t stream) {
  if (T > kNoAllocMaxRows) return cudaErrorInvalidValue;
  unsigned char* scr = nullptr;
  cudaError_t e = noalloc_scratch(&scr);
  if (e != cudaSuccess) return e;
  unsigned int* sync = reinterpret_cast<unsigned int*>(scr);
  float* inv = reinterpret_cast<float*>(scr + kNoAllocSyncBytes);
  // the array keeps the last call's contents: start every call from zero
  // (the max, the counters, both error words and the injection word)
  e = cudaMemsetAsync(sync, 0, 8 * sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  e = launch_prep(X, gamma, eps, row_index, T, Tp, K, kind, per_token, inv, s_g, sync, sp_codes, meta, sp_sf,
                  r_codes, r_sf, r_meta, 0, nullptr, nullptr, stream);
  if (e != cudaSuccess) return e;
  // forward the error word to where sharq_linear looks for it
  if (err_out) e = cudaMemcpyAsync(err_out, sync + 3, sizeof(unsigned int), cudaMemcpyDeviceToDevice, stream);
  return e;
}

}  // namespace sharq

// quant.cuh - the per-element SharQ quantization steps, shared by the prep
// kernels (prep.cu) and the fused decode GEMM (gemm.cu).
//
// xllm-io review of SharQ, sections 3.2-3.3 (4:8 in-pairs backbone, residual
// w.r.t. the quantized backbone) and 3.5 (one fused preparation step);
// kasblo.com explainer, steps 1-3.  The float32 operation order is the one
// include/sharq.h documents for sharq_prep.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sharq_device.cuh"

namespace sharq {

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

struct QuantPtrs {
  uint8_t* sp_codes;
  uint8_t* meta;
  uint8_t* sp_sf;
  uint8_t* r_codes;
  uint8_t* r_sf;
  uint8_t* r_meta;  // Sparse+Sparse only: the residual's metadata
};

// How the activation is split into its two FP4 operands (xllm-io review,
// section 3 for SharQ; section 5.3, Table 5, for the others; plain NVFP4 is
// the comparator of Table 1).
enum : int {
  kKindNvfp4 = 0,        // one dense operand: NVFP4 of Xn
  kKindSharq = 1,        // sparse backbone + dense residual (also Sparse only: the GEMM drops the residual)
  kKindDenseDense = 2,   // dense NVFP4 of Xn + dense NVFP4 of its residual
  kKindSparseSparse = 3,  // sparse backbone + sparse (4:8 in-pairs) residual
  kKindSharqMx = 4,       // SharQ in MXFP4: E8M0 scales, backbone per 64 logical K, residual per 32 K
  kKindMxfp4 = 5          // plain MXFP4 of Xn (32-element blocks)
};
__host__ __device__ constexpr bool kind_is_mx(int kind) { return kind == kKindSharqMx || kind == kKindMxfp4; }

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

// Sparse operand of NC consecutive runs of 8 logical K of row t, held in
// registers (v[8*c + e] = run c, element e), starting at run c0 of the row:
// the 4:8 in-pairs mask (keep the 2 of 4 pairs with the largest max|v|, ties
// to the lower pair), the kept values' NVFP4 codes with one scale per 32
// logical K, the metadata; out[] = v - f32(val * dec * s) at kept positions
// and v elsewhere (exact).  Tiles: codes 8 KB (64-byte swizzle), metadata
// 2 KB, scales 1 KB.  NC = 1, 2: the 32-K block spans 4 / NC adjacent lanes
// (all 32 lanes of the warp must call it).  kMx: one E8M0 scale per 64
// logical K (8 runs; 512-byte scale tiles), s must be 1.
template <int NC, bool kMx = false>
__device__ __forceinline__ void sparse_operand(const float (&x)[8 * NC], float (&res)[8 * NC], int t, int c0, int K,
                                               float s, float six_s, uint8_t* codes_out, uint8_t* meta_out,
                                               uint8_t* sf_out, bool store) {
  const int KS = K >> 8;
  const int r = t & 127;
#pragma unroll
  for (int i = 0; i < 8 * NC; ++i) res[i] = x[i];
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
  // one scale per 32 logical K (4 runs = 16 kept values); MX: per 64 (8 runs)
  constexpr int kBlockRuns = kMx ? 8 : 4;
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < 4 * NC; ++i) am = fmaxf(am, fabsf(v[i]));
  if (NC < kBlockRuns) am = group_max(am, kBlockRuns / NC);
  const BlockScale bs = kMx ? mx_block_scale(am) : block_scale(am, six_s, s);
  uint32_t cb[2 * NC];  // code bytes: kept values (2i, 2i+1)
#pragma unroll
  for (int i = 0; i < 2 * NC; ++i) cb[i] = cvt_e2m1x2(__fmul_rn(v[2 * i], bs.inv), __fmul_rn(v[2 * i + 1], bs.inv));
  // residual w.r.t. the quantized operand at kept positions (exact fp32)
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
  // stores: per run 2 bytes of kept codes, one metadata nibble
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int g = c0 + c;               // run index in the row
    const int kt = g >> 5, w = g & 31;  // K tile, run within the 256-K tile
    const size_t tile = (size_t)(t >> 7) * KS + kt;
    if (store)
      *reinterpret_cast<uint16_t*>(codes_out + tile * kSpTile + sp_chunk_off(r, w >> 3) + 2 * (w & 7)) =
          (uint16_t)(cb[2 * c] | (cb[2 * c + 1] << 8));
    const uint32_t m = km[c];
    const uint32_t nib = (uint32_t)((__ffs(m) - 1) | ((31 - __clz(m)) << 2));
    if (NC == 1) {
      const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
      if (store && (w & 1) == 0) meta_out[tile * kMetaTile + r * 16 + (w >> 1)] = (uint8_t)(nib | (other << 4));
    } else if (store && (c & 1) == 0) {
      const uint32_t m2 = km[c + 1 < NC ? c + 1 : c];
      const uint32_t other = (uint32_t)((__ffs(m2) - 1) | ((31 - __clz(m2)) << 2));
      meta_out[tile * kMetaTile + r * 16 + (w >> 1)] = (uint8_t)(nib | (other << 4));
    }
    if (kMx) {
      if (store && (w & 7) == 0) sf_out[tile * kSf64Tile + sf_off(r, 0, w >> 3)] = (uint8_t)bs.sb;
    } else if (store && (w & 3) == 0) {
      sf_out[tile * kSf32Tile + sf_off(r, w >> 4, (w >> 2) & 3)] = (uint8_t)bs.sb;
    }
  }
}

// Dense operand: NVFP4 of v in 16-element blocks; with kDeq, deq[] receives
// f32(val * dec * s) of every element.  Tiles: codes 16 KB (128-byte
// swizzle), scales 2 KB.  kMx: MXFP4, one E8M0 scale per 32 K (1 KB scale
// tiles), s must be 1.  A block spans 2 (MX: 4) runs; when a thread holds
// fewer, it spans adjacent lanes (all 32 lanes of the warp must call it).
template <int NC, bool kDeq, bool kMx = false>
__device__ __forceinline__ void dense_operand(const float (&res)[8 * NC], float (&deq)[8 * NC], int t, int c0, int K,
                                              float s, float six_s, uint8_t* codes_out, uint8_t* sf_out, bool store) {
  const int KS = K >> 8;
  const int r = t & 127;
  constexpr int kBlockRuns = kMx ? 4 : 2;
  constexpr int nr = NC < kBlockRuns ? NC : kBlockRuns;  // runs of a block held by this thread
  constexpr int lanes = kBlockRuns / nr;                  // lanes a block spans
#pragma unroll
  for (int c = 0; c < NC; c += nr) {
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8 * nr; ++i) am = fmaxf(am, fabsf(res[8 * c + i]));
    if (lanes > 1) am = group_max(am, lanes);
    const BlockScale bs = kMx ? mx_block_scale(am) : block_scale(am, six_s, s);
#pragma unroll
    for (int h = 0; h < nr; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t b = cvt_e2m1x2(__fmul_rn(res[8 * (c + h) + 2 * i], bs.inv),
                                      __fmul_rn(res[8 * (c + h) + 2 * i + 1], bs.inv));
        word |= b << (8 * i);
        if (kDeq) {
          const float2 q = e2m1x2_values(b);
          deq[8 * (c + h) + 2 * i] = __fmul_rn(__fmul_rn(q.x, bs.dec), s);
          deq[8 * (c + h) + 2 * i + 1] = __fmul_rn(__fmul_rn(q.y, bs.dec), s);
        }
      }
      const int g = c0 + c + h;
      const int kt = g >> 5, w = g & 31;
      const size_t tile = (size_t)(t >> 7) * KS + kt;
      if (store) {
        *reinterpret_cast<uint32_t*>(codes_out + tile * kCodesTile + codes_chunk_off(r, w >> 2) + 4 * (w & 3)) =
            word;
        if (kMx) {
          if ((w & 3) == 0) sf_out[tile * kSf32Tile + sf_off(r, w >> 4, (w >> 2) & 3)] = (uint8_t)bs.sb;
        } else if ((w & 1) == 0) {
          sf_out[tile * kSf16Tile + sf_off(r, w >> 3, (w >> 1) & 3)] = (uint8_t)bs.sb;
        }
      }
    }
  }
}

// Quantize NC consecutive runs of 8 logical K of row t into the two operands
// of kKind (see the enum).  NC = 4: every block is inside the thread; NC = 1,
// 2: blocks span adjacent lanes and all 32 lanes of the warp must call it.
template <int NC, int kKind>
__device__ __forceinline__ void quant_runs(const float (&x)[8 * NC], int t, int c0, int K, float s, float six_s,
                                           const QuantPtrs& out, bool store = true) {
  float res[8 * NC];
  if (kKind == kKindNvfp4) {
    dense_operand<NC, false>(x, res, t, c0, K, s, six_s, out.r_codes, out.r_sf, store);
  } else if (kKind == kKindSharq) {
    sparse_operand<NC>(x, res, t, c0, K, s, six_s, out.sp_codes, out.meta, out.sp_sf, store);
    dense_operand<NC, false>(res, res, t, c0, K, s, six_s, out.r_codes, out.r_sf, store);
  } else if (kKind == kKindDenseDense) {
    float deq[8 * NC];
    dense_operand<NC, true>(x, deq, t, c0, K, s, six_s, out.sp_codes, out.sp_sf, store);
#pragma unroll
    for (int i = 0; i < 8 * NC; ++i) res[i] = __fsub_rn(x[i], deq[i]);
    dense_operand<NC, false>(res, deq, t, c0, K, s, six_s, out.r_codes, out.r_sf, store);
  } else if (kKind == kKindSparseSparse) {
    float res2[8 * NC];
    sparse_operand<NC>(x, res, t, c0, K, s, six_s, out.sp_codes, out.meta, out.sp_sf, store);
    sparse_operand<NC>(res, res2, t, c0, K, s, six_s, out.r_codes, out.r_meta, out.r_sf, store);
  } else if (kKind == kKindSharqMx) {
    sparse_operand<NC, true>(x, res, t, c0, K, 1.0f, 6.0f, out.sp_codes, out.meta, out.sp_sf, store);
    dense_operand<NC, false, true>(res, res, t, c0, K, 1.0f, 6.0f, out.r_codes, out.r_sf, store);
  } else {  // kKindMxfp4
    dense_operand<NC, false, true>(x, res, t, c0, K, 1.0f, 6.0f, out.r_codes, out.r_sf, store);
  }
}

// Epilogues of the preceding operation, fused into the preparation
// (kasblo.com explainer, section 4 on fusing the preparation: RMSNorm and the
// epilogues before it join the prep kernel).  The prep input becomes h, formed
// element by element from two bf16 tensors A (the prep's X) and B:
//   kEpiAdd:     h = bf16_rn(f32(a) + f32(b))  -- the residual-stream update
//                before a pre-norm layer's RMSNorm (a = sublayer output, b =
//                residual stream);
//   kEpiSiluMul: h = bf16_rn(silu_bf16(a) * f32(b))  -- the SwiGLU product a
//                down projection takes (a = gate, b = up), with silu_bf16 the
//                correctly rounded bf16 of silu(a) = a / (1 + e^-a).
// h is optionally written out (H may alias B: each element is read and
// written by the same thread).
enum : int { kEpiNone = 0, kEpiAdd = 1, kEpiSiluMul = 2 };
struct Epi {
  const __nv_bfloat16* B = nullptr;  // second input, [T][K], or nullptr
  __nv_bfloat16* H = nullptr;        // h out (may alias B), or nullptr
  int kind = kEpiNone;
};

// silu(g) rounded to bf16 by way of float64 and round-to-odd (the slow path
// of silu_bf16; out of line so that its registers stay out of the callers').
//   |g| < 1:   g/2 + d with d = (g/2) tanh(g/2) >= 0, kept as the pair hi + lo
//              (Knuth's two-sum), so that hi on a bf16 midpoint -- g/2 for
//              tiny g -- rounds the way lo points;
//   g >= 1:    g / (1 + e^-g);   g <= -1:  g e^g / (1 + e^g).
// hi + lo goes to float32 rounded to odd (truncate, then set the last bit
// when inexact), then to bf16 to nearest even: float32 keeps more than two
// extra bits, so the two roundings give the correctly rounded bf16.
static __device__ __noinline__ float silu_bf16_f64(float g) {
  if (isinf(g)) return g > 0.0f ? g : -0.0f;  // silu(+inf) = +inf, silu(-inf) = -0
  const double gd = g;
  double hi, lo = 0.0;
  if (fabs(gd) < 1.0) {
    const double a = 0.5 * gd, d = a * tanh(a);
    hi = a + d;
    const double bb = hi - a;
    lo = (a - (hi - bb)) + (d - bb);
  } else if (gd >= 1.0) {
    hi = gd / (1.0 + exp(-gd));
  } else {
    const double e = exp(gd);
    hi = gd * e / (1.0 + e);
  }
  const double mag = fabs(hi);
  const double b = hi < 0.0 ? -lo : lo;  // lo along the magnitude
  uint32_t fb = __float_as_uint(__double2float_rz(mag));
  if ((double)__uint_as_float(fb) != mag) fb |= 1u;  // strictly between two floats
  else if (b > 0.0) fb |= 1u;
  else if (b < 0.0 && fb != 0u) fb = (fb - 1u) | 1u;
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(__uint_as_float(fb)));
  // silu(g) has the sign of g (silu(g) / g = sigmoid(g) > 0), zeros included
  return __uint_as_float(((uint32_t)r << 16) | (__float_as_uint(g) & 0x80000000u));
}

// silu(g) correctly rounded to bf16, returned as a float32 holding it.  Fast
// path in float32, branch-free: e = expf(-|g|) in (0, 1] (CUDA's expf, max
// error 2 ulp), numerator g (g >= 0) or g e (g < 0), one __fdividef by 1 + e
// (max error 2 ulp for divisors in [1, 2]): the result is within about 7
// float32 ulps of silu(g), which fixes its bf16 rounding unless it lies within
// 16 ulps of a bf16 rounding midpoint (low 16 bits near 0x8000).  Those
// inputs, g < -80 (e near float32's subnormals), the infinities and NaN take
// the float64 path.
__device__ __forceinline__ float silu_bf16(float g) {
  const float e = expf(-fabsf(g));
  const float num = g >= 0.0f ? g : __fmul_rn(g, e);
  const float s = __fdividef(num, __fadd_rn(1.0f, e));
  const uint32_t low = __float_as_uint(s) & 0xFFFFu;
  if (low + 16u - 0x8000u > 32u && g > -80.0f && g < INFINITY) {  // |low - 0x8000| > 16
    // s is not near a midpoint, so rounding half up in magnitude is rounding
    // to nearest
    return __uint_as_float((__float_as_uint(s) + 0x8000u) & 0xFFFF0000u);
  }
  return silu_bf16_f64(g);
}

__device__ __forceinline__ uint32_t silu_mul_bf16x2(uint32_t g2, uint32_t u2) {
  const float h_lo = __fmul_rn(silu_bf16(__uint_as_float(g2 << 16)), __uint_as_float(u2 << 16));
  const float h_hi = __fmul_rn(silu_bf16(__uint_as_float(g2 & 0xFFFF0000u)), __uint_as_float(u2 & 0xFFFF0000u));
  uint32_t o;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o) : "f"(h_hi), "f"(h_lo));
  return o;
}

__device__ __forceinline__ uint4 add_bf16x8(const uint4& a, const uint4& b) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fadd_rn(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16));
    const float hi = __fadd_rn(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wb[i] & 0xFFFF0000u));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[i]) : "f"(hi), "f"(lo));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// h for 8 consecutive elements (a from X, b from B)
__device__ __forceinline__ uint4 epi8(const uint4& a, const uint4& b, int kind) {
  if (kind == kEpiAdd) return add_bf16x8(a, b);
  return make_uint4(silu_mul_bf16x2(a.x, b.x), silu_mul_bf16x2(a.y, b.y), silu_mul_bf16x2(a.z, b.z),
                    silu_mul_bf16x2(a.w, b.w));
}

// N consecutive vectors of 8 bf16 from element offset off, whose X values
// are already in v: v <- h, and h written out when an output is given (by the
// thread that read B there, so H may alias B).
template <int N>
__device__ __forceinline__ void apply_epi(uint4 (&v)[N], size_t off, const Epi& ep) {
  const uint4* bp = reinterpret_cast<const uint4*>(ep.B + off);
  uint4 r[N];
#pragma unroll
  for (int c = 0; c < N; ++c) r[c] = bp[c];
#pragma unroll
  for (int c = 0; c < N; ++c) v[c] = epi8(v[c], r[c], ep.kind);
  if (ep.H) {
    uint4* hh = reinterpret_cast<uint4*>(ep.H + off);
#pragma unroll
    for (int c = 0; c < N; ++c) hh[c] = v[c];
  }
}

// load NC runs of 8 (one 16-byte load each) of row src (zeros when src < 0);
// with an epilogue the runs are h (and h is stored when an output is given)
template <int NC>
__device__ __forceinline__ void load_runs(float (&x)[8 * NC], const __nv_bfloat16* X, int src, int K, int c0,
                                          const Epi& ep = Epi{}) {
  if (src >= 0) {
    const size_t off = (size_t)src * K + 8 * (size_t)c0;
    const uint4* xr = reinterpret_cast<const uint4*>(X + off);
    uint4 raw[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) raw[c] = xr[c];
    if (ep.kind) apply_epi<NC>(raw, off, ep);
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

}  // namespace sharq

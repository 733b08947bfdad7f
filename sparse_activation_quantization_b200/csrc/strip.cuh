// strip.cuh - the 32-K strip quantizer of sharq_prep's wide (prefill) form.
//
// xllm-io review of SharQ, sections 3.2-3.3 (4:8 in-pairs mask, sparse
// backbone quantization, residual R = Xn - dequant(backbone)) and 3.5 (the
// dense residual in 16-element blocks); kasblo.com explainer, steps 1-3.
//
// One thread quantizes 32 consecutive K of one row -- four 4:8 runs, the
// whole 32-K backbone block and both 16-K residual blocks -- so no value
// crosses a lane.  The arithmetic is the same as quant_runs<4> (quant.cuh),
// step for step and rounding for rounding, with fewer instructions:
//  - pairs of fp32 values use the packed f32x2 multiply of sm_100 (never a
//    packed multiply feeding a packed add or subtract: ptxas fuses those into
//    one rounding whatever the rounding modifiers say);
//  - the four pair scores become integer-ordered keys (score bits | 3 - p)
//    and the 4:8 selection is a 7-op top-2 network; the backbone block's
//    amax is the largest run score (the run maximum is always kept);
//  - every code of a run is converted, and byte permutes pick the two kept
//    pairs (one permute for two runs) and zero the codes of the dropped
//    pairs for the residual;
//  - amax/(6 s) uses Markstein's correction step (see quot_six_s) and the
//    block-scale decode and reciprocal come from a per-CTA table indexed by
//    the E4M3 byte;
//  - each output goes out in one vector store per strip.
#pragma once
#include "quant.cuh"

namespace sharq {

// ------------------------------------------------- packed fp32 pairs ----
typedef unsigned long long f2_t;  // {low: element 2i, high: element 2i+1}

__device__ __forceinline__ f2_t f2_make(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(f2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
  f2_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// two bf16 (one 32-bit word, lower K in the low half) -> exact fp32 pair
__device__ __forceinline__ f2_t f2_from_bf16x2(uint32_t w) {
  return f2_make(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// fp32 pair -> two bf16 (round to nearest even), low element in the low half
__device__ __forceinline__ uint32_t bf16x2_from_f2(f2_t v) {
  float lo, hi;
  f2_split(v, lo, hi);
  uint32_t w;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(hi), "f"(lo));
  return w;
}
// Xn = bf16_rn(f32(f32(x * inv) * g)) for a pair, returned as exact fp32
__device__ __forceinline__ f2_t f2_norm(f2_t x, f2_t inv2, f2_t g) {
  return f2_from_bf16x2(bf16x2_from_f2(f2_mul(f2_mul(x, inv2), g)));
}

// eight fp32 values (four pairs) -> eight E2M1 codes in one word, element
// 2p in the low nibble of byte p
__device__ __forceinline__ uint32_t e2m1x8(f2_t p0, f2_t p1, f2_t p2, f2_t p3) {
  float a0, a1, b0, b1, c0, c1, d0, d1;
  f2_split(p0, a0, a1);
  f2_split(p1, b0, b1);
  f2_split(p2, c0, c1);
  f2_split(p3, d0, d1);
  uint32_t w;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(w)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1), "f"(d0), "f"(d1));
  return w;
}

// byte p of a word of E2M1 codes -> the two values as exact f16x2, each
// multiplied by the block's E4M3 scale value (exact: at most 6 significant
// bits, within the f16 normal range)
__device__ __forceinline__ void e2m1x8_times(uint32_t w, uint32_t dec_h2, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      ".reg .b32 v0, v1, v2, v3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 v0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 v1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 v2, q2;\n\t"
      "cvt.rn.f16x2.e2m1x2 v3, q3;\n\t"
      "mul.rn.f16x2 %0, v0, %5;\n\t"
      "mul.rn.f16x2 %1, v1, %5;\n\t"
      "mul.rn.f16x2 %2, v2, %5;\n\t"
      "mul.rn.f16x2 %3, v3, %5;\n\t}"
      : "=&r"(h[0]), "=&r"(h[1]), "=&r"(h[2]), "=&r"(h[3])  // written before dec_h2 is last read
      : "r"(w), "r"(dec_h2));
}
__device__ __forceinline__ f2_t f2_from_f16x2(uint32_t h) {
  float lo, hi;
  asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return f2_make(lo, hi);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// ------------------------------------------------- per-tensor context ----
struct StripCtx {
  float s;       // per-tensor scale s_g
  float six_s;   // f32(6 * s)
  float y6;      // f32(1 / six_s), correctly rounded
  bool mark;     // six_s within the range where quot_six_s is exact
  const float2* tab;     // [128] by E4M3 byte: {1/S (0 if S == 0), dec}, S = f32(dec * s)
  const uint32_t* msel;  // [16] by metadata nibble: byte-permute keeping the two kept pairs' codes
};

// f32(a / six_s), correctly rounded, for a >= 0.  Markstein's theorem
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990; also Muller et al., Handbook
// of Floating-Point Arithmetic, section 5.3): with y the correctly rounded
// 1/b and q0 = RN(a y) (within one ulp of a/b), the remainder r = a - q0 b
// is exact in one fma and RN(q0 + r y) is the correctly rounded a/b, as long
// as nothing under- or overflows.  With 2^-60 <= b <= 2^60 that holds for
// every quotient that can round to a nonzero E4M3 value (>= 2^-10), and
// smaller quotients encode to 0 either way; quotients stay below ~2^10 here
// (a block amax never exceeds twice the tensor max).  Outside that range of
// b the correctly rounded division is used directly.
__device__ __forceinline__ float quot_six_s(float a, const StripCtx& c) {
  if (!c.mark) return __fdiv_rn(a, c.six_s);
  const float q0 = __fmul_rn(a, c.y6);
  const float r = __fmaf_rn(-q0, c.six_s, a);
  return __fmaf_rn(r, c.y6, q0);
}

// the tables of StripCtx, filled by the first 128 threads of the CTA
__device__ __forceinline__ void strip_tables_init(float s, float2* tab, uint32_t* msel) {
  const int c = threadIdx.x;
  if (c < 128) {
    const float dec = e4m3_value((uint32_t)c);
    const float S = __fmul_rn(dec, s);
    tab[c] = make_float2(S > 0.0f ? __frcp_rn(S) : 0.0f, dec);
  }
  if (c < 16) {
    // kept pairs lo = c & 3, hi = c >> 2: their bytes stay, the others come
    // from byte 4 (the zero operand)
    const uint32_t lo = c & 3, hi = c >> 2;
    uint32_t m = 0;
#pragma unroll
    for (uint32_t p = 0; p < 4; ++p) m |= ((p == lo || p == hi) ? p : 4u) << (4 * p);
    msel[c] = m;
  }
}

__device__ __forceinline__ StripCtx strip_ctx(float s, const float2* tab, const uint32_t* msel) {
  StripCtx c;
  c.s = s;
  c.six_s = __fmul_rn(6.0f, s);
  c.y6 = __frcp_rn(c.six_s);
  c.mark = c.six_s >= 0x1p-60f && c.six_s <= 0x1p60f;
  c.tab = tab;
  c.msel = msel;
  return c;
}

// Quantize strip j (K = 32j .. 32j+31) of row t.  P[i] holds Xn at K = 32j +
// 2i, 2i + 1 (bf16-exact fp32).  KS = K / 256.
template <bool kSharq>
__device__ __forceinline__ void quant_strip(const f2_t (&P)[16], int t, int j, int KS, const StripCtx& c,
                                            const QuantPtrs& out) {
  const uint32_t r = (uint32_t)t & 127u;
  const uint32_t jj = (uint32_t)j & 7u;
  const size_t tile = (size_t)(t >> 7) * KS + (j >> 3);
  f2_t R[16];

  if (kSharq) {
    // --- 4:8 in-pairs mask per run: keys = score bits | (3 - p); scores are
    // bf16-exact, so the two low bits are free and equal scores order by
    // the lower pair first
    uint32_t nib[4], sel[4];
    float rmax[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t k[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float lo, hi;
        f2_split(P[4 * q + p], lo, hi);
        k[p] = __float_as_uint(fmaxf(fabsf(lo), fabsf(hi))) | (3u - p);
      }
      const uint32_t a = max(k[0], k[1]), b = min(k[0], k[1]);
      const uint32_t d = max(k[2], k[3]), e = min(k[2], k[3]);
      const uint32_t t1 = max(a, d);
      const uint32_t t2 = max(max(min(a, d), b), e);
      const uint32_t i1 = ~t1 & 3u, i2 = ~t2 & 3u;
      const uint32_t lo = min(i1, i2), hi = max(i1, i2);
      nib[q] = lo | (hi << 2);
      sel[q] = lo | (hi << 4);
      rmax[q] = __uint_as_float(t1 & ~3u);
    }
    // --- backbone block (the whole strip: 32 logical K, 16 kept values)
    const float am = fmaxf(fmaxf(rmax[0], rmax[1]), fmaxf(rmax[2], rmax[3]));
    const uint32_t sb = cvt_e4m3(quot_six_s(am, c));
    const float2 td = c.tab[sb];
    const f2_t inv2 = f2_make(td.x, td.x);
    uint32_t word[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      word[q] = e2m1x8(f2_mul(P[4 * q], inv2), f2_mul(P[4 * q + 1], inv2), f2_mul(P[4 * q + 2], inv2),
                       f2_mul(P[4 * q + 3], inv2));
    // kept codes: bytes lo and hi of each run, two runs per permute
    const uint32_t kept01 = prmt(word[0], word[1], sel[0] | ((sel[1] + 0x44u) << 8));
    const uint32_t kept23 = prmt(word[2], word[3], sel[2] | ((sel[3] + 0x44u) << 8));
    // --- residual: R = Xn - f32(val * dec * s) at kept positions, Xn - 0 elsewhere
    uint32_t dec_h2;
    asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(dec_h2) : "f"(td.y));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t h[4];
      e2m1x8_times(prmt(word[q], 0u, c.msel[nib[q]]), dec_h2, h);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        // scalar: ptxas contracts a packed multiply followed by a packed
        // subtract into one fused (singly rounded) op, even with an explicit
        // rounding mode; the method rounds t = f32(val dec s) first
        float x0, x1, v0, v1;
        f2_split(P[4 * q + p], x0, x1);
        f2_split(f2_from_f16x2(h[p]), v0, v1);
        R[4 * q + p] = f2_make(__fsub_rn(x0, __fmul_rn(v0, c.s)), __fsub_rn(x1, __fmul_rn(v1, c.s)));
      }
    }
    // --- stores
    *reinterpret_cast<uint2*>(out.sp_codes + tile * kSpTile + sp_chunk_off(r, jj >> 1) + 8u * (jj & 1u)) =
        make_uint2(kept01, kept23);
    *reinterpret_cast<uint16_t*>(out.meta + tile * kMetaTile + r * 16u + 2u * jj) =
        (uint16_t)(nib[0] | (nib[1] << 4) | (nib[2] << 8) | (nib[3] << 12));
    out.sp_sf[tile * kSf32Tile + sf_off(r, jj >> 2, jj & 3u)] = (uint8_t)sb;
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) R[i] = P[i];
  }

  // --- dense NVFP4 of R (of Xn in NVFP4 mode): blocks of 16 = runs 0-1, 2-3
  float qb[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float lo, hi;
      f2_split(R[8 * b + i], lo, hi);
      am = fmaxf(am, fmaxf(fabsf(lo), fabsf(hi)));
    }
    qb[b] = quot_six_s(am, c);
  }
  uint32_t sbs;
  asm("{\n\t.reg .b16 q;\n\tcvt.rn.satfinite.e4m3x2.f32 q, %1, %2;\n\tcvt.u32.u16 %0, q;\n\t}"
      : "=r"(sbs)
      : "f"(qb[1]), "f"(qb[0]));
  uint32_t wd[4];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const float inv = c.tab[(sbs >> (8 * b)) & 0xFFu].x;
    const f2_t inv2 = f2_make(inv, inv);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int q = 2 * b + h;
      wd[q] = e2m1x8(f2_mul(R[4 * q], inv2), f2_mul(R[4 * q + 1], inv2), f2_mul(R[4 * q + 2], inv2),
                     f2_mul(R[4 * q + 3], inv2));
    }
  }
  *reinterpret_cast<uint4*>(out.r_codes + tile * kCodesTile + codes_chunk_off(r, jj)) =
      make_uint4(wd[0], wd[1], wd[2], wd[3]);
  *reinterpret_cast<uint16_t*>(out.r_sf + tile * kSf16Tile + sf_off(r, jj >> 1, 2u * (jj & 1u))) = (uint16_t)sbs;
}

}  // namespace sharq

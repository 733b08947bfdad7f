// pack_weight.cu - sharq_pack_weight: the shared FP4 weight payload.
//
// xllm-io review of SharQ, section 3.5 ("shared FP4 weight payload": both
// paths use one FP4 weight body and differ only in the scale view -- sparse
// group-32 scales, dense group-16 scales duplicated), section 3.4 for the
// operators Q_w,sp(W) and Q_w,dn(W); kasblo.com explainer, step 3.
//
// W in R^{K x D} (bf16, row-major, per expert) is quantized per output column
// d along K: one E4M3 scale per 32 K and an FP32 global scale
// s_w = amax(W) / (6 * 448).  The kernel writes the K-major FP4 codes in the
// 128-byte-swizzled tile layout the MMA reads, the per-32 scale view and the
// per-16 view in which every per-32 byte appears twice (identical dequantized
// values, the layout the dense block16 MMA wants).
//
// Runs once per weight; two launches (device-wide amax, then quantization).
// The MXFP4 payload (launch_pack_weight_mx) is one launch.
#include "sharq_device.cuh"

namespace sharq {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) weight_amax_kernel(const __nv_bfloat16* __restrict__ W,
                                                                long long per_expert,
                                                                unsigned int* __restrict__ amax_bits) {
  const int e = blockIdx.y;
  const __nv_bfloat16* w = W + (size_t)e * per_expert;
  float a = 0.0f;
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < per_expert;
       i += (long long)gridDim.x * kThreads)
    a = fmaxf(a, fabsf(__bfloat162float(w[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + e, __float_as_uint(a));
}

// one thread per (expert, 32-K block, column d); consecutive threads take
// consecutive d so each of the 32 row loads is coalesced across the warp
__global__ void __launch_bounds__(kThreads) weight_quant_kernel(
    const __nv_bfloat16* __restrict__ W, int K, int D, const unsigned int* __restrict__ amax_bits,
    float* __restrict__ s_w, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf32,
    uint8_t* __restrict__ sf16) {
  const int e = blockIdx.z;
  const int kb = blockIdx.y;                       // 32-K block
  const int d = blockIdx.x * kThreads + threadIdx.x;
  if (d >= D) return;
  const float amax = __uint_as_float(amax_bits[e]);
  const float s = amax > 0.0f ? __fdiv_rn(amax, kGlobalDiv) : 1.0f;
  if (kb == 0 && d == 0) s_w[e] = s;
  const __nv_bfloat16* w = W + (size_t)e * K * D + (size_t)(32 * kb) * D + d;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(w[(size_t)i * D]);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(v[i]));
  const BlockScale bs = block_scale(a, __fmul_rn(6.0f, s), s);
  uint32_t word[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t wv = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = 8 * k + 2 * b;
      wv |= cvt_e2m1x2(__fmul_rn(v[i], bs.inv), __fmul_rn(v[i + 1], bs.inv)) << (8 * b);
    }
    word[k] = wv;
  }
  const int KS = K >> 8, NB = D >> 7;
  const int kt = kb >> 3, q = kb & 7, nb = d >> 7, r = d & 127;
  const size_t tile = ((size_t)e * NB + nb) * KS + kt;
  *reinterpret_cast<uint4*>(codes + tile * kCodesTile + codes_chunk_off(r, q)) =
      make_uint4(word[0], word[1], word[2], word[3]);
  sf32[tile * kSf32Tile + sf_off(r, q >> 2, q & 3)] = (uint8_t)bs.sb;
  *reinterpret_cast<uint16_t*>(sf16 + tile * kSf16Tile + sf_off(r, q >> 1, 2 * (q & 1))) =
      (uint16_t)(bs.sb | (bs.sb << 8));
}

// MXFP4 payload (OCP Microscaling: E8M0 power-of-two scales, no tensor
// scale): one thread per (expert, 64-K block, column d) -- 64 K is the scale
// granularity of the sparse kind::mxf4 MMA, so the sparse view holds one byte
// per 64 K and the dense view (32-K blocks) repeats it twice.  s_w = 1.
__global__ void __launch_bounds__(kThreads) weight_quant_mx_kernel(
    const __nv_bfloat16* __restrict__ W, int K, int D, float* __restrict__ s_w, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf64, uint8_t* __restrict__ sf32) {
  const int e = blockIdx.z;
  const int kb = blockIdx.y;  // 64-K block
  const int d = blockIdx.x * kThreads + threadIdx.x;
  if (d >= D) return;
  if (kb == 0 && d == 0) s_w[e] = 1.0f;
  const __nv_bfloat16* w = W + (size_t)e * K * D + (size_t)(64 * kb) * D + d;
  float v[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __bfloat162float(w[(size_t)i * D]);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 64; ++i) a = fmaxf(a, fabsf(v[i]));
  const BlockScale bs = mx_block_scale(a);
  uint32_t word[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t wv = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = 8 * k + 2 * b;
      wv |= cvt_e2m1x2(__fmul_rn(v[i], bs.inv), __fmul_rn(v[i + 1], bs.inv)) << (8 * b);
    }
    word[k] = wv;
  }
  const int KS = K >> 8, NB = D >> 7;
  const int kt = kb >> 2, j = kb & 3, nb = d >> 7, r = d & 127;
  const size_t tile = ((size_t)e * NB + nb) * KS + kt;
  *reinterpret_cast<uint4*>(codes + tile * kCodesTile + codes_chunk_off(r, 2 * j)) =
      make_uint4(word[0], word[1], word[2], word[3]);
  *reinterpret_cast<uint4*>(codes + tile * kCodesTile + codes_chunk_off(r, 2 * j + 1)) =
      make_uint4(word[4], word[5], word[6], word[7]);
  sf64[tile * kSf64Tile + sf_off(r, 0, j)] = (uint8_t)bs.sb;
  *reinterpret_cast<uint16_t*>(sf32 + tile * kSf32Tile + sf_off(r, j >> 1, (2 * j) & 3)) =
      (uint16_t)(bs.sb | (bs.sb << 8));
}

}  // namespace

cudaError_t launch_pack_weight_mx(const void* W, int K, int D, int E, uint8_t* codes, uint8_t* sf64, uint8_t* sf32,
                                  float* s_w, cudaStream_t stream) {
  weight_quant_mx_kernel<<<dim3((D + kThreads - 1) / kThreads, K / 64, E), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(W), K, D, s_w, codes, sf64, sf32);
  return cudaGetLastError();
}

cudaError_t launch_pack_weight(const void* W, int K, int D, int E, uint8_t* codes, uint8_t* sf32,
                               uint8_t* sf16, float* s_w, unsigned int* amax_bits, cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(amax_bits, 0, sizeof(unsigned int) * E, stream);
  if (err != cudaSuccess) return err;
  const long long per = (long long)K * D;
  int gx = (int)((per + kThreads * 8 - 1) / (kThreads * 8));
  gx = gx < 1 ? 1 : (gx > 1184 ? 1184 : gx);
  weight_amax_kernel<<<dim3(gx, E), kThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(W), per, amax_bits);
  weight_quant_kernel<<<dim3((D + kThreads - 1) / kThreads, K / 32, E), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(W), K, D, amax_bits, s_w, codes, sf32, sf16);
  return cudaGetLastError();
}

}  // namespace sharq

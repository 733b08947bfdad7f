// api.cu - the extern "C" boundary declared in include/sharq.h.
//
// Host-side only: size queries, carving caller-owned buffers into views,
// argument / shape / architecture checks, and the kernel launches of
// prep.cu, pack_weight.cu and gemm.cu.  Nothing here allocates device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sharq.h"
#include "sharq_device.cuh"

namespace sharq {
cudaError_t launch_prep(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp, int K,
                        int kind, bool per_token, float* inv_rms, float* s_g, unsigned int* gmax_bits,
                        uint8_t* sp_codes, uint8_t* meta, uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf,
                        uint8_t* r_meta, int epi_kind, const void* epi_b, void* epi_h, cudaStream_t stream);
cudaError_t launch_pack_weight(const void* W, int K, int D, int E, uint8_t* codes, uint8_t* sf32, uint8_t* sf16,
                               float* s_w, unsigned int* amax_bits, cudaStream_t stream);
cudaError_t launch_pack_weight_mx(const void* W, int K, int D, int E, uint8_t* codes, uint8_t* sf64, uint8_t* sf32,
                                  float* s_w, cudaStream_t stream);
cudaError_t launch_linear(const uint8_t* a_sp, const uint8_t* a_meta, const uint8_t* a_spsf, const uint8_t* a_r,
                          const uint8_t* a_rsf, const uint8_t* a_rmeta, const float* s_g, int T, int Tp, int K,
                          int gmode,
                          const uint8_t* w_codes, const uint8_t* w_sf32, const uint8_t* w_sf16, const float* s_w,
                          int D, int E, const int* group_offsets, void* Y, int out_f32, int bn, int splits,
                          int* err, const int* act_err, cudaStream_t stream, const void* X_fused,
                          const void* gamma_fused, float eps_fused, bool per_token);
int noalloc_max_rows();
int split_max_clusters(int splits, bool fused);
bool prep_per_token_supported(int K);
cudaError_t launch_prep_noalloc(const void* X, const void* gamma, float eps, const int* row_index, int T, int Tp,
                                int K, int kind, bool per_token, float* s_g, uint8_t* sp_codes, uint8_t* meta,
                                uint8_t* sp_sf, uint8_t* r_codes, uint8_t* r_sf, uint8_t* r_meta,
                                unsigned int* err_out, cudaStream_t stream);
}  // namespace sharq

namespace {

constexpr int kMaxT = 1 << 22;
constexpr int kMaxK = 1 << 17;
constexpr int kMaxD = 1 << 18;
constexpr int kMaxE = 4096;
constexpr size_t kAlign = 256;
constexpr size_t kWsHeader = 256;  // error word + reserved
constexpr int kTargetCtas = 148;   // B200 SM count: one GEMM CTA per SM

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool shape_ok_k(int K) { return K > 0 && K <= kMaxK && K % 256 == 0; }
bool shape_ok_d(int D) { return D > 0 && D <= kMaxD && D % 128 == 0; }
bool shape_ok_t(int T) { return T >= 0 && T <= kMaxT; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool mode_ok(int mode) { return mode >= SHARQ_MODE_SHARQ && mode <= SHARQ_MODE_MXFP4_PLAIN; }
bool mode_is_mx(int mode) { return mode == SHARQ_MODE_MXFP4 || mode == SHARQ_MODE_MXFP4_PLAIN; }
// operand sets per mode: first operand (sp_codes/meta/sp_sf) sparse or dense,
// second operand (r_codes/r_sf, r_meta) dense or sparse
bool has_first(int mode) { return mode != SHARQ_MODE_NVFP4 && mode != SHARQ_MODE_MXFP4_PLAIN; }
bool first_sparse(int mode) { return has_first(mode) && mode != SHARQ_MODE_DENSE_DENSE; }
bool second_sparse(int mode) { return mode == SHARQ_MODE_SPARSE_SPARSE; }
// prep operand kind (csrc/quant.cuh) and GEMM operand set (csrc/gemm.cu)
int prep_kind(int mode) {
  switch (mode) {
    case SHARQ_MODE_NVFP4: return 0;
    case SHARQ_MODE_DENSE_DENSE: return 2;
    case SHARQ_MODE_SPARSE_SPARSE: return 3;
    case SHARQ_MODE_MXFP4: return 4;
    case SHARQ_MODE_MXFP4_PLAIN: return 5;
    default: return 1;  // SHARQ, SHARQ_TOKEN, SPARSE_ONLY
  }
}
int gemm_mode(int mode) {
  switch (mode) {
    case SHARQ_MODE_NVFP4: return 1;
    case SHARQ_MODE_SPARSE_ONLY: return 2;
    case SHARQ_MODE_DENSE_DENSE: return 3;
    case SHARQ_MODE_SPARSE_SPARSE: return 4;
    case SHARQ_MODE_MXFP4: return 5;
    case SHARQ_MODE_MXFP4_PLAIN: return 6;
    default: return 0;  // SHARQ, SHARQ_TOKEN
  }
}

// layout sizes, shared by the *_bytes and *_view functions
struct ActLayout {
  size_t r_codes, r_sf, sp_codes, meta, sp_sf, r_meta, inv, s_tok, scal, total;
};
ActLayout act_layout(int T, int K, int mode) {
  ActLayout L{};
  const size_t Tp = round_up((size_t)T, 128);
  const size_t tiles = (Tp / 128) * (size_t)(K / 256);
  size_t off = 0;
  const bool s2 = second_sparse(mode);
  // scale tiles: NVFP4 sparse operand 1 KB (per 32 logical K), dense 2 KB
  // (per 16); MXFP4 sparse 512 B (per 64 logical K), dense 1 KB (per 32)
  const size_t sf_sp = mode_is_mx(mode) ? sharq::kSf64Tile : sharq::kSf32Tile;
  const size_t sf_dn = mode_is_mx(mode) ? sharq::kSf32Tile : sharq::kSf16Tile;
  L.r_codes = off; off += tiles * (s2 ? sharq::kSpTile : sharq::kCodesTile);
  L.r_sf = off;    off += tiles * (s2 ? sf_sp : sf_dn);
  L.sp_codes = off;
  if (has_first(mode)) off += tiles * (first_sparse(mode) ? sharq::kSpTile : sharq::kCodesTile);
  L.meta = off;
  if (first_sparse(mode)) off += tiles * sharq::kMetaTile;
  L.sp_sf = off;
  if (has_first(mode)) off += round_up(tiles * (first_sparse(mode) ? sf_sp : sf_dn), 16);
  L.r_meta = off;
  if (s2) off += tiles * sharq::kMetaTile;
  L.inv = off;     off = round_up(off + Tp * sizeof(float), kAlign);
  L.s_tok = off;   // per-token scales (SHARQ_TOKEN only)
  if (mode == SHARQ_MODE_SHARQ_TOKEN) off = round_up(off + Tp * sizeof(float), kAlign);
  L.scal = off;    off += kAlign;  // s_g, gmax_bits
  L.total = off;
  return L;
}

struct WeightLayout {
  size_t codes, sf32, sf16, s_w, scratch, total;
};
// fmt: SHARQ_FMT_NVFP4 (sparse view per 32 K, dense view per 16) or
// SHARQ_FMT_MXFP4 (sparse view per 64 K, dense view per 32)
WeightLayout weight_layout(int K, int D, int E, int fmt = SHARQ_FMT_NVFP4) {
  WeightLayout L{};
  const size_t tiles = (size_t)E * (D / 128) * (K / 256);
  const bool mx = fmt == SHARQ_FMT_MXFP4;
  size_t off = 0;
  L.codes = off; off += tiles * sharq::kCodesTile;
  L.sf32 = off;  off += tiles * (mx ? sharq::kSf64Tile : sharq::kSf32Tile);
  L.sf16 = off;  off += tiles * (mx ? sharq::kSf32Tile : sharq::kSf16Tile);
  L.s_w = off;   off = round_up(off + (size_t)E * sizeof(float), kAlign);
  L.scratch = off; off = round_up(off + (size_t)E * sizeof(unsigned), kAlign);
  L.total = off;
  return L;
}

// GEMM launch shape for a problem: tile width BN and the number of K splits.
// Prefill shapes have enough output tiles to fill the GPU (no split).  Decode
// shapes split K over a cluster of up to 8 CTAs per output tile so that about
// one CTA per SM streams a slice of the weight; the partial tiles are reduced
// over distributed shared memory, so no workspace is needed for them.
struct GemmShape {
  int bn, splits, m_tiles, n_tiles;
};
GemmShape gemm_shape(int T, int K, int D, int E, bool fused = false) {
  GemmShape g{};
  const int Tp = (int)round_up((size_t)T, 128);
  g.m_tiles = Tp / 128;
  const int KS = K / 256;
  g.bn = (D % 256 == 0) ? 256 : 128;
  g.n_tiles = D / g.bn;
  g.splits = 1;
  if (E == 1 && (long long)g.m_tiles * g.n_tiles < kTargetCtas / 2) {
    // split: 128-wide tiles (the partial and the received slices must fit the
    // shared-memory ring) and clusters of at most 4, which the GPCs can host
    // all at once with one CTA per SM
    g.bn = 128;
    g.n_tiles = D / 128;
    const long long mn = (long long)g.m_tiles * g.n_tiles;
    int s = (int)(kTargetCtas / mn);
    s = s < 4 ? s : 4;
    s = s < KS ? s : KS;
    // no second wave: as many clusters as the GPCs hold at once (36 clusters
    // of 4 do not fit; 36 of 3 do)
    while (s > 1) {
      const int mc = sharq::split_max_clusters(s, fused);
      if (mc == 0 || mn <= mc) break;
      --s;
    }
    g.splits = s > 1 ? s : 1;
  }
  return g;
}

int check_device() {
  static int cached[64] = {};  // 0 unknown, 1 ok, -1 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SHARQ_ERR_CUDA;
  if (dev < 64 && cached[dev]) return cached[dev] > 0 ? SHARQ_OK : SHARQ_ERR_ARCH;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SHARQ_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev < 64) cached[dev] = ok ? 1 : -1;
  return ok ? SHARQ_OK : SHARQ_ERR_ARCH;
}

// for_prep: sharq_prep writes inv_rms and uses gmax_bits; sharq_linear reads
// neither (a NULL gmax_bits only means no prep error word to forward)
int act_ok(const sharq_act* a, bool for_prep = true) {
  if (!a) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_t(a->T) || !shape_ok_k(a->K)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (!mode_ok(a->mode)) return SHARQ_ERR_INVALID_ARG;
  if (a->Tp != (int)round_up((size_t)a->T, 128)) return SHARQ_ERR_INVALID_ARG;
  if (!a->r_codes || !a->r_sf || !a->s_g) return SHARQ_ERR_INVALID_ARG;
  if (for_prep && (!a->inv_rms || !a->gmax_bits)) return SHARQ_ERR_INVALID_ARG;
  if (has_first(a->mode) && (!a->sp_codes || !a->sp_sf)) return SHARQ_ERR_INVALID_ARG;
  if (first_sparse(a->mode) && !a->meta) return SHARQ_ERR_INVALID_ARG;
  if (second_sparse(a->mode) && !a->r_meta) return SHARQ_ERR_INVALID_ARG;
  const void* p[] = {a->r_codes, a->r_sf, a->sp_codes, a->meta, a->sp_sf, a->r_meta};
  for (const void* q : p)
    if (q && !aligned(q, 16)) return SHARQ_ERR_INVALID_ARG;
  return SHARQ_OK;
}

int weight_ok(const sharq_weight* w) {
  if (!w) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_k(w->K) || !shape_ok_d(w->D) || w->E < 1 || w->E > kMaxE) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (!w->codes || !w->sf32 || !w->sf16 || !w->s_w) return SHARQ_ERR_INVALID_ARG;
  if (!aligned(w->codes, 16) || !aligned(w->sf32, 16) || !aligned(w->sf16, 16)) return SHARQ_ERR_INVALID_ARG;
  if (w->fmt != SHARQ_FMT_NVFP4 && w->fmt != SHARQ_FMT_MXFP4) return SHARQ_ERR_INVALID_ARG;
  return SHARQ_OK;
}

int linear_common(const sharq_act* a, const int* d_offsets, const sharq_weight* w, void* d_Y, int out_dtype,
                  void* d_ws, size_t ws_bytes, sharq_stream_t stream, bool grouped) {
  int st = act_ok(a, false);
  if (st) return st;
  if ((st = weight_ok(w))) return st;
  if (a->K != w->K) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (mode_is_mx(a->mode) != (w->fmt == SHARQ_FMT_MXFP4)) return SHARQ_ERR_INVALID_ARG;  // formats must match
  if (!grouped && w->E != 1) return SHARQ_ERR_INVALID_ARG;
  if (grouped && !d_offsets) return SHARQ_ERR_INVALID_ARG;
  if (out_dtype != SHARQ_OUT_BF16 && out_dtype != SHARQ_OUT_F32) return SHARQ_ERR_INVALID_ARG;
  if (a->T > 0 && (!d_Y || !aligned(d_Y, 16))) return SHARQ_ERR_INVALID_ARG;
  if (!d_ws || ws_bytes < sharq_workspace_bytes(a->T, a->K, w->D, grouped ? w->E : 1) || !aligned(d_ws, 16))
    return SHARQ_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  const GemmShape g = gemm_shape(a->T, a->K, w->D, grouped ? w->E : 1);
  cudaError_t e = sharq::launch_linear(
      static_cast<const uint8_t*>(a->sp_codes), static_cast<const uint8_t*>(a->meta),
      static_cast<const uint8_t*>(a->sp_sf), static_cast<const uint8_t*>(a->r_codes),
      static_cast<const uint8_t*>(a->r_sf), static_cast<const uint8_t*>(a->r_meta), a->s_g, a->T, a->Tp, a->K,
      gemm_mode(a->mode),
      static_cast<const uint8_t*>(w->codes), static_cast<const uint8_t*>(w->sf32),
      static_cast<const uint8_t*>(w->sf16), w->s_w, w->D, w->E, grouped ? d_offsets : nullptr, d_Y,
      out_dtype == SHARQ_OUT_F32 ? 1 : 0, g.bn, g.splits, static_cast<int*>(d_ws),
      a->gmax_bits ? reinterpret_cast<const int*>(a->gmax_bits + 3) : nullptr, reinterpret_cast<cudaStream_t>(stream),
      nullptr, nullptr,
      0.0f, a->mode == SHARQ_MODE_SHARQ_TOKEN);
  return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}

}  // namespace

extern "C" {

int sharq_abi_version(void) { return SHARQ_ABI_VERSION; }

const char* sharq_status_string(int status) {
  switch (status) {
    case SHARQ_OK: return "SHARQ_OK";
    case SHARQ_ERR_INVALID_ARG: return "SHARQ_ERR_INVALID_ARG";
    case SHARQ_ERR_UNSUPPORTED_SHAPE: return "SHARQ_ERR_UNSUPPORTED_SHAPE";
    case SHARQ_ERR_ARCH: return "SHARQ_ERR_ARCH";
    case SHARQ_ERR_CUDA: return "SHARQ_ERR_CUDA";
    case SHARQ_ERR_TIMEOUT: return "SHARQ_ERR_TIMEOUT";
    case SHARQ_ERR_WORKSPACE: return "SHARQ_ERR_WORKSPACE";
    default: return "SHARQ_ERR_UNKNOWN";
  }
}

size_t sharq_weight_bytes_fmt(int K, int D, int E, int fmt) {
  if (!shape_ok_k(K) || !shape_ok_d(D) || E < 1 || E > kMaxE) return 0;
  if (fmt != SHARQ_FMT_NVFP4 && fmt != SHARQ_FMT_MXFP4) return 0;
  return weight_layout(K, D, E, fmt).total;
}

size_t sharq_weight_bytes(int K, int D, int E) { return sharq_weight_bytes_fmt(K, D, E, SHARQ_FMT_NVFP4); }

size_t sharq_act_bytes(int T, int K, int mode) {
  if (!shape_ok_t(T) || !shape_ok_k(K)) return 0;
  if (!mode_ok(mode)) return 0;
  return act_layout(T, K, mode).total;
}

size_t sharq_workspace_bytes(int T, int K, int D, int E) {
  if (!shape_ok_t(T) || !shape_ok_k(K) || !shape_ok_d(D) || E < 1 || E > kMaxE) return 0;
  return kWsHeader;
}

int sharq_weight_view_fmt(void* d_buf, int K, int D, int E, int fmt, sharq_weight* out) {
  if (!d_buf || !out) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_k(K) || !shape_ok_d(D) || E < 1 || E > kMaxE) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt != SHARQ_FMT_NVFP4 && fmt != SHARQ_FMT_MXFP4) return SHARQ_ERR_INVALID_ARG;
  if (!aligned(d_buf, kAlign)) return SHARQ_ERR_INVALID_ARG;
  const WeightLayout L = weight_layout(K, D, E, fmt);
  uint8_t* b = static_cast<uint8_t*>(d_buf);
  out->codes = b + L.codes;
  out->sf32 = b + L.sf32;
  out->sf16 = b + L.sf16;
  out->s_w = reinterpret_cast<float*>(b + L.s_w);
  out->K = K;
  out->D = D;
  out->E = E;
  out->fmt = fmt;
  return SHARQ_OK;
}

int sharq_weight_view(void* d_buf, int K, int D, int E, sharq_weight* out) {
  return sharq_weight_view_fmt(d_buf, K, D, E, SHARQ_FMT_NVFP4, out);
}

int sharq_act_view(void* d_buf, int T, int K, int mode, sharq_act* out) {
  if (!d_buf || !out) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_t(T) || !shape_ok_k(K)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (!mode_ok(mode)) return SHARQ_ERR_INVALID_ARG;
  if (!aligned(d_buf, kAlign)) return SHARQ_ERR_INVALID_ARG;
  const ActLayout L = act_layout(T, K, mode);
  uint8_t* b = static_cast<uint8_t*>(d_buf);
  out->r_codes = b + L.r_codes;
  out->r_sf = b + L.r_sf;
  out->sp_codes = has_first(mode) ? b + L.sp_codes : nullptr;
  out->meta = first_sparse(mode) ? b + L.meta : nullptr;
  out->sp_sf = has_first(mode) ? b + L.sp_sf : nullptr;
  out->r_meta = second_sparse(mode) ? b + L.r_meta : nullptr;
  out->inv_rms = reinterpret_cast<float*>(b + L.inv);
  out->s_g = reinterpret_cast<float*>(b + (mode == SHARQ_MODE_SHARQ_TOKEN ? L.s_tok : L.scal));
  out->gmax_bits = reinterpret_cast<unsigned int*>(b + L.scal + 16);
  out->T = T;
  out->Tp = (int)round_up((size_t)T, 128);
  out->K = K;
  out->mode = mode;
  return SHARQ_OK;
}

int sharq_pack_weight(const void* d_W, const sharq_weight* w, sharq_stream_t stream) {
  int st = weight_ok(w);
  if (st) return st;
  if (!d_W || !aligned(d_W, 2)) return SHARQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  if (w->fmt == SHARQ_FMT_MXFP4) {
    cudaError_t e = sharq::launch_pack_weight_mx(d_W, w->K, w->D, w->E, static_cast<uint8_t*>(w->codes),
                                                 static_cast<uint8_t*>(w->sf32), static_cast<uint8_t*>(w->sf16),
                                                 w->s_w, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
  }
  const WeightLayout L = weight_layout(w->K, w->D, w->E);
  unsigned int* scratch = reinterpret_cast<unsigned int*>(reinterpret_cast<uint8_t*>(w->s_w) + (L.scratch - L.s_w));
  cudaError_t e = sharq::launch_pack_weight(d_W, w->K, w->D, w->E, static_cast<uint8_t*>(w->codes),
                                            static_cast<uint8_t*>(w->sf32), static_cast<uint8_t*>(w->sf16), w->s_w,
                                            scratch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}

namespace {
// epi_kind: 0 none, 1 residual add (h = x + b), 2 SwiGLU product (h = silu(x) * b)
int prep_common(const void* d_X, const void* d_gamma, float eps, const int* d_row_index, const sharq_act* a,
                int epi_kind, const void* d_b, void* d_h, sharq_stream_t stream) {
  int st = act_ok(a);
  if (st) return st;
  if (a->T > 0 && (!d_X || !aligned(d_X, 16))) return SHARQ_ERR_INVALID_ARG;
  if (d_gamma && !aligned(d_gamma, 16)) return SHARQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return SHARQ_ERR_INVALID_ARG;
  const bool per_token = a->mode == SHARQ_MODE_SHARQ_TOKEN;
  if (per_token && !sharq::prep_per_token_supported(a->K)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if ((st = check_device())) return st;
  cudaError_t e = sharq::launch_prep(
      d_X, d_gamma, eps, d_row_index, a->T, a->Tp, a->K, prep_kind(a->mode), per_token, a->inv_rms, a->s_g,
      a->gmax_bits, static_cast<uint8_t*>(a->sp_codes), static_cast<uint8_t*>(a->meta),
      static_cast<uint8_t*>(a->sp_sf), static_cast<uint8_t*>(a->r_codes), static_cast<uint8_t*>(a->r_sf),
      static_cast<uint8_t*>(a->r_meta), epi_kind, d_b, d_h, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}
}  // namespace

int sharq_prep(const void* d_X, const void* d_gamma, float eps, const int* d_row_index, const sharq_act* a,
               sharq_stream_t stream) {
  return prep_common(d_X, d_gamma, eps, d_row_index, a, 0, nullptr, nullptr, stream);
}

namespace {
int prep_epilogue(int kind, const void* d_A, const void* d_B, void* d_H, const void* d_gamma, float eps,
                  const sharq_act* a, sharq_stream_t stream) {
  if (!a) return SHARQ_ERR_INVALID_ARG;
  if (a->T > 0 && (!d_B || !aligned(d_B, 16))) return SHARQ_ERR_INVALID_ARG;
  if (d_H && !aligned(d_H, 16)) return SHARQ_ERR_INVALID_ARG;
  if (a->T > 0 && d_H == d_A) return SHARQ_ERR_INVALID_ARG;  // may alias d_B, not d_A
  if (a->T == 0) return prep_common(d_A, d_gamma, eps, nullptr, a, 0, nullptr, nullptr, stream);
  return prep_common(d_A, d_gamma, eps, nullptr, a, kind, d_B, d_H, stream);
}
}  // namespace

int sharq_prep_residual(const void* d_X, const void* d_res, void* d_res_out, const void* d_gamma, float eps,
                        const sharq_act* a, sharq_stream_t stream) {
  return prep_epilogue(1, d_X, d_res, d_res_out, d_gamma, eps, a, stream);
}

int sharq_prep_silu_mul(const void* d_gate, const void* d_up, void* d_h, const void* d_gamma, float eps,
                        const sharq_act* a, sharq_stream_t stream) {
  return prep_epilogue(2, d_gate, d_up, d_h, d_gamma, eps, a, stream);
}

int sharq_prep_noalloc(const void* d_X, const void* d_gamma, float eps, const int* d_row_index,
                       const sharq_act* a, sharq_stream_t stream) {
  if (!a) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_t(a->T) || !shape_ok_k(a->K)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (a->T > sharq::noalloc_max_rows()) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (!mode_ok(a->mode)) return SHARQ_ERR_INVALID_ARG;
  if (a->Tp != (int)round_up((size_t)a->T, 128)) return SHARQ_ERR_INVALID_ARG;
  if (!a->r_codes || !a->r_sf || !a->s_g) return SHARQ_ERR_INVALID_ARG;
  if (has_first(a->mode) && (!a->sp_codes || !a->sp_sf)) return SHARQ_ERR_INVALID_ARG;
  if (first_sparse(a->mode) && !a->meta) return SHARQ_ERR_INVALID_ARG;
  if (second_sparse(a->mode) && !a->r_meta) return SHARQ_ERR_INVALID_ARG;
  if (a->mode == SHARQ_MODE_SHARQ_TOKEN && !sharq::prep_per_token_supported(a->K)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  const void* p[] = {a->r_codes, a->r_sf, a->sp_codes, a->meta, a->sp_sf, a->r_meta};
  for (const void* q : p)
    if (q && !aligned(q, 16)) return SHARQ_ERR_INVALID_ARG;
  if (a->T > 0 && (!d_X || !aligned(d_X, 16))) return SHARQ_ERR_INVALID_ARG;
  if (d_gamma && !aligned(d_gamma, 16)) return SHARQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return SHARQ_ERR_INVALID_ARG;
  int st = check_device();
  if (st) return st;
  cudaError_t e = sharq::launch_prep_noalloc(
      d_X, d_gamma, eps, d_row_index, a->T, a->Tp, a->K, prep_kind(a->mode), a->mode == SHARQ_MODE_SHARQ_TOKEN,
      a->s_g, static_cast<uint8_t*>(a->sp_codes), static_cast<uint8_t*>(a->meta), static_cast<uint8_t*>(a->sp_sf),
      static_cast<uint8_t*>(a->r_codes), static_cast<uint8_t*>(a->r_sf), static_cast<uint8_t*>(a->r_meta),
      a->gmax_bits ? a->gmax_bits + 3 : nullptr,
      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}

int sharq_prep_linear(const void* d_X, const void* d_gamma, float eps, int T, const sharq_act* a,
                      const sharq_weight* w, void* d_Y, int out_dtype, void* d_ws, size_t ws_bytes,
                      sharq_stream_t stream) {
  int st = weight_ok(w);
  if (st) return st;
  if (w->E != 1 || w->fmt != SHARQ_FMT_NVFP4) return SHARQ_ERR_INVALID_ARG;
  if (!shape_ok_t(T)) return SHARQ_ERR_UNSUPPORTED_SHAPE;
  if (T > SHARQ_FUSED_MAX_T) {  // larger batches: the two-call path through `a`
    if (!a || a->T != T || a->K != w->K || (a->mode != SHARQ_MODE_SHARQ && a->mode != SHARQ_MODE_SHARQ_TOKEN))
      return SHARQ_ERR_INVALID_ARG;
    if ((st = sharq_prep(d_X, d_gamma, eps, nullptr, a, stream))) return st;
    return sharq_linear(a, w, d_Y, out_dtype, d_ws, ws_bytes, stream);
  }
  if (out_dtype != SHARQ_OUT_BF16 && out_dtype != SHARQ_OUT_F32) return SHARQ_ERR_INVALID_ARG;
  if (T > 0 && (!d_X || !aligned(d_X, 16) || !d_Y || !aligned(d_Y, 16))) return SHARQ_ERR_INVALID_ARG;
  if (d_gamma && !aligned(d_gamma, 16)) return SHARQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return SHARQ_ERR_INVALID_ARG;
  if (!d_ws || ws_bytes < sharq_workspace_bytes(T, w->K, w->D, 1) || !aligned(d_ws, 16)) return SHARQ_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  if (T == 0) return SHARQ_OK;
  const GemmShape g = gemm_shape(T, w->K, w->D, 1, true);
  cudaError_t e = sharq::launch_linear(
      nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, T, (int)round_up((size_t)T, 128), w->K,
      0 /* SharQ operands */,
      static_cast<const uint8_t*>(w->codes), static_cast<const uint8_t*>(w->sf32),
      static_cast<const uint8_t*>(w->sf16), w->s_w, w->D, 1, nullptr, d_Y, out_dtype == SHARQ_OUT_F32 ? 1 : 0,
      g.bn, g.splits, static_cast<int*>(d_ws), nullptr, reinterpret_cast<cudaStream_t>(stream), d_X, d_gamma, eps,
      false);
  return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}

int sharq_linear(const sharq_act* a, const sharq_weight* w, void* d_Y, int out_dtype, void* d_ws, size_t ws_bytes,
                 sharq_stream_t stream) {
  return linear_common(a, nullptr, w, d_Y, out_dtype, d_ws, ws_bytes, stream, false);
}

int sharq_linear_grouped(const sharq_act* a, const int* d_group_offsets, const sharq_weight* w, void* d_Y,
                         int out_dtype, void* d_ws, size_t ws_bytes, sharq_stream_t stream) {
  return linear_common(a, d_group_offsets, w, d_Y, out_dtype, d_ws, ws_bytes, stream, true);
}

int sharq_check_status(void* d_ws, sharq_stream_t stream) {
  if (!d_ws) return SHARQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, d_ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SHARQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SHARQ_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(d_ws, 0, sizeof(int), s) != cudaSuccess) return SHARQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SHARQ_ERR_CUDA;
  }
  return word;
}

}  // extern "C"

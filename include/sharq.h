/*
 * sharq.h - C ABI of the SharQ hot path for NVIDIA B200 (sm_100a).
 *
 * SharQ ("SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
 * Inference", arXiv 2606.26587) replaces one linear layer Y = X W
 * (X in R^{T x K}, W in R^{K x D}; xllm-io review, section 3.1) by
 *
 *   Y = GEMM_sp(Q_sp(X_sp), Q_w,sp(W)) + GEMM_dn(Q_dn(R), Q_w,dn(W))
 *
 * (section 3.4), where X_sp = M(X) . X is an input-adaptive 4:8 in-pairs
 * sparse backbone (section 3.2) and R = X - D_sp(Q_sp(X_sp)) is the residual
 * w.r.t. the *quantized* backbone (section 3.3).  Both paths are NVFP4
 * (E2M1 values, E4M3 block scales, FP32 global scale) and share one FP4 weight
 * payload through two scale views (section 3.5).
 *
 * Three calls make up the path:
 *   sharq_pack_weight  once per weight: FP4 payload + per-32 and per-16 scales
 *   sharq_prep         per activation tensor: RMSNorm, per-tensor scale (PTS),
 *                      4:8 in-pairs mask, NVFP4 backbone, NVFP4 residual
 *   sharq_linear       sparse FP4 MMA + dense FP4 MMA into one accumulator
 *
 * Conventions (all entry points):
 *  - Pointers named d_* / inside sharq_act / sharq_weight are DEVICE pointers.
 *    The caller allocates and owns every buffer; the library never allocates,
 *    keeps no state between calls, and is safe to call from several threads
 *    on different streams with different buffers.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument, shape and architecture checks happen
 *    before anything is enqueued and return a negative sharq_status; nothing
 *    is enqueued in that case.
 *  - A kernel that waits on an on-chip barrier gives up after a bounded time
 *    and records SHARQ_ERR_TIMEOUT in the caller's workspace instead of
 *    hanging; sharq_check_status() reads it back.
 *  - Shapes: K % 256 == 0 (one tile of sparse metadata spans 256 logical K),
 *    D % 128 == 0, 0 <= T, T <= 1<<22.  Non-finite inputs are undefined.
 *  - Buffers carved by the *_view calls must start on a 256-byte boundary.
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SHARQ_ABI_VERSION 2

typedef struct CUstream_st *sharq_stream_t; /* same type as cudaStream_t */

typedef enum {
  SHARQ_OK = 0,
  SHARQ_ERR_INVALID_ARG = -1,      /* NULL pointer, bad enum, misaligned buffer */
  SHARQ_ERR_UNSUPPORTED_SHAPE = -2, /* K % 256, D % 128, T or E out of range */
  SHARQ_ERR_ARCH = -3,             /* current device is not sm_100 */
  SHARQ_ERR_CUDA = -4,             /* a CUDA runtime call failed */
  SHARQ_ERR_TIMEOUT = -5,          /* a device-side bounded wait gave up */
  SHARQ_ERR_WORKSPACE = -6         /* workspace missing or too small */
} sharq_status;

/* Output element type of sharq_linear. */
enum { SHARQ_OUT_BF16 = 0, SHARQ_OUT_F32 = 1 };

/* Activation path.  SHARQ: sparse backbone + dense residual (the method).
 * NVFP4: plain NVFP4 of Xn (16-element blocks, same PTS scale) and a dense
 * FP4 GEMM only -- the "NVFP4" comparator of the xllm-io review's Table 1 and
 * the official repository's NVFP4 mode (kasblo.com explainer).
 * SHARQ_TOKEN: the SharQ path with the global activation scale read as
 * per-TOKEN rather than per-tensor (the pages never expand "PTS", xllm-io
 * review, sections 3.1 and 3.5): row t gets s_t = max|Xn[t]| / (6*448) and is
 * prepared exactly as a one-row tensor; no device-wide reduction.  Its codes
 * are not those of the per-tensor mode.  Supported for K <= 20480. */
enum { SHARQ_MODE_SHARQ = 0, SHARQ_MODE_NVFP4 = 1, SHARQ_MODE_SHARQ_TOKEN = 2 };

/* The other operand splits of the xllm-io review's ablation (section 5.3,
 * Table 5), under the plainest reading of their names; every other step
 * (RMSNorm, the per-tensor scale, the block quantizer, the 4:8 in-pairs rule)
 * is the method's:
 *   SPARSE_ONLY    the SharQ backbone alone: sharq_prep writes the SharQ
 *                  operands, sharq_linear multiplies only the backbone.
 *   DENSE_DENSE    first operand: dense NVFP4 of Xn (16-element blocks) in
 *                  sp_codes / sp_sf (laid out as r_codes / r_sf); second:
 *                  dense NVFP4 of Xn minus its dequantized value.
 *   SPARSE_SPARSE  the SharQ backbone, and the residual pruned by the same
 *                  4:8 in-pairs rule (scores max|R|) and quantized as a
 *                  sparse operand: r_codes laid out as sp_codes, r_sf as
 *                  sp_sf, its metadata in r_meta.
 * These modes always run the persistent GEMM (no split-K decode form) and
 * are not accepted by sharq_prep_linear. */
enum { SHARQ_MODE_SPARSE_ONLY = 3, SHARQ_MODE_DENSE_DENSE = 4, SHARQ_MODE_SPARSE_SPARSE = 5 };

/* MXFP4 (xllm-io review, section 5.3: SharQ on the NVFP4, HiF4 and MXFP4
 * formats).  MXFP4 is the OCP Microscaling format: E2M1 elements and one E8M0
 * (power-of-two) scale X = 2^(floor(log2 amax) - 2) per block, no tensor
 * scale (s_g = 1, s_w = 1).  The pages pair MXFP4 with 2:4 sparsity; the
 * sparse FP4 MMA of sm_100 takes the 4:8 in-pairs pattern, so:
 *   MXFP4        the SharQ decomposition in MXFP4: 4:8 in-pairs backbone with
 *                one E8M0 scale per 64 logical K (sp_sf: 512-byte tiles, one
 *                atom), dense MXFP4 residual with one per 32 K (r_sf: 1024-
 *                byte tiles).
 *   MXFP4_PLAIN  plain MXFP4 of Xn (r_codes, r_sf as above), the comparator.
 * Both need a weight packed in SHARQ_FMT_MXFP4. */
enum { SHARQ_MODE_MXFP4 = 6, SHARQ_MODE_MXFP4_PLAIN = 7 };

/* Weight payload format.  NVFP4: E4M3 scales, sparse view per 32 K, dense
 * view per 16 K, FP32 s_w.  MXFP4: E8M0 scales per 64 K (the sparse MXFP4
 * MMA's granularity) in sf32 (512-byte tiles), the dense view per 32 K in sf16
 * (1024-byte tiles, each byte twice), s_w = 1. */
enum { SHARQ_FMT_NVFP4 = 0, SHARQ_FMT_MXFP4 = 1 };

/* Tile geometry of every packed operand: 128 rows x 256 logical K. */
#define SHARQ_TILE_ROWS 128
#define SHARQ_TILE_K 256

/*
 * Packed weight (xllm-io review, section 3.5: one FP4 weight body, sparse
 * path group-32 scales, dense path group-16 scales duplicated).
 * W in R^{K x D} is quantized per output column d along K, one E4M3 scale per
 * 32 K, FP32 global scale s_w = amax(W) / (6 * 448) (1 if W == 0).
 * Layout, for expert e, column tile nb = d / 128, K tile kt = k / 256,
 * tile index i = (e * D/128 + nb) * K/256 + kt,  r = d % 128, c = k % 256:
 *   codes: 16384-byte tiles; row r is the 128-byte line at r*128, E2M1 codes
 *          of K c..c+1 in byte c/2 (low nibble = lower K), with the 16-byte
 *          chunks of a line permuted by chunk ^= (r % 8) (128-byte swizzle).
 *   sf32:  1024-byte tiles = 2 scale atoms of 512 bytes; the scale of 32-block
 *          b = c/32 is at atom b/4, byte (r%32)*16 + (r/32)*4 + b%4.
 *   sf16:  2048-byte tiles = 4 atoms; block b = c/16 at atom b/4, same byte
 *          formula; each sf32 byte appears twice (b = 2j, 2j+1).
 *   s_w:   E floats.
 */
typedef struct {
  void *codes;
  void *sf32;
  void *sf16;
  float *s_w;
  int K, D, E;
  int fmt; /* SHARQ_FMT_NVFP4 (set by sharq_weight_view) or SHARQ_FMT_MXFP4 */
} sharq_weight;

/*
 * Prepared activation (output of sharq_prep, operand A of sharq_linear).
 * The tiles cover Tp = ceil(T/128)*128 rows; rows T..Tp-1 are not written by
 * sharq_prep and never read as operands by sharq_linear (their contents are
 * unspecified).
 * Tile index i = (t/128) * K/256 + k/256, r = t % 128, c = k % 256:
 *   r_codes: 16384-byte tiles, 128-byte lines, 128-byte swizzle (as weight
 *            codes).  SHARQ: residual codes.  NVFP4: codes of Xn.
 *   r_sf:    2048-byte tiles, one scale per 16 K (as weight sf16).
 *   sp_codes (SHARQ, SHARQ_TOKEN): 8192-byte tiles; row r is the 64-byte line at
 *            r*64 holding the 128 kept values of its 256 logical K in
 *            ascending K order, byte j/2 for kept value j; 16-byte chunks
 *            permuted by chunk ^= (r/2) % 4 (64-byte swizzle).
 *   meta (SHARQ, SHARQ_TOKEN): 2048-byte tiles, row r at r*16; chunk of 8 logical K
 *            g = c/8 in byte g/2 (low nibble = lower chunk); nibble =
 *            p_lo | p_hi << 2, the kept pair indices, p_lo < p_hi.
 *   sp_sf (SHARQ, SHARQ_TOKEN): 1024-byte tiles, one scale per 32 logical K (16 kept
 *            values), atom layout as weight sf32.
 *   inv_rms: Tp floats (1/rms per row; 1 when RMSNorm is off).
 *   s_g:     the per-tensor global scale gmax / (6*448) (1 if gmax == 0);
 *            SHARQ_TOKEN: Tp floats, s_t of row t (rows >= T unused).
 *   gmax_bits: 24 bytes of scratch, six 32-bit words: device-wide amax,
 *            grid-barrier count, departure count, the error word of the last
 *            sharq_prep (SHARQ_ERR_TIMEOUT when its grid barrier timed out;
 *            sharq_linear forwards it to its workspace), the error of the
 *            prep in flight, and a fault-injection word that must stay zero
 *            (a test writes k + 1 there to make CTA k of the grid-barrier form
 *            skip its arrival, so that the bounded wait runs out).
 *   The 256-byte scalar block that holds gmax_bits (and s_g outside
 *   SHARQ_TOKEN)
 *   must be zero before the first sharq_prep on a buffer (zero the whole
 *   buffer once after allocation); sharq_prep leaves gmax_bits[0..2] and
 *   gmax_bits[4] zero again, so no per-call memset is needed.
 *   sharq_linear reads only the operands, s_g and (when it is not NULL)
 *   gmax_bits[3]; it does not need inv_rms.
 */
typedef struct {
  void *sp_codes;
  void *meta;
  void *sp_sf;
  void *r_codes;
  void *r_sf;
  float *inv_rms;
  float *s_g;
  unsigned int *gmax_bits;
  int T, Tp, K, mode;
  void *r_meta; /* SPARSE_SPARSE only: the residual's metadata (layout as meta) */
} sharq_act;

/* Host-only size queries (pure functions; 0 on invalid shape). */
size_t sharq_weight_bytes(int K, int D, int E); /* SHARQ_FMT_NVFP4 */
/* Bytes of a packed weight in format fmt (SHARQ_FMT_*); 0 on an invalid shape or format. */
size_t sharq_weight_bytes_fmt(int K, int D, int E, int fmt);
size_t sharq_act_bytes(int T, int K, int mode);
/* Workspace of sharq_linear (E = 1) / sharq_linear_grouped (E experts):
 * the device-side error word (256 bytes reserved).  The caller zeroes it
 * once after allocation; sharq_check_status clears it after reading. */
size_t sharq_workspace_bytes(int T, int K, int D, int E);

/* Carve the views of a caller-owned device buffer of at least the size
 * returned above (no device access). */
int sharq_weight_view(void *d_buf, int K, int D, int E, sharq_weight *out); /* SHARQ_FMT_NVFP4 */
/* Views of a weight buffer in format fmt; sharq_pack_weight packs in w->fmt.
 * Errors: SHARQ_ERR_INVALID_ARG (null, misaligned, unknown fmt),
 * SHARQ_ERR_UNSUPPORTED_SHAPE. */
int sharq_weight_view_fmt(void *d_buf, int K, int D, int E, int fmt, sharq_weight *out);
int sharq_act_view(void *d_buf, int T, int K, int mode, sharq_act *out);

/*
 * sharq_pack_weight - quantize W once into the shared FP4 payload.
 * d_W: bf16 [E][K][D] row-major (W in R^{K x D} per expert).
 * Fills w->codes, w->sf32, w->sf16, w->s_w (buffers from sharq_weight_view).
 */
int sharq_pack_weight(const void *d_W, const sharq_weight *w, sharq_stream_t stream);

/*
 * sharq_prep - the fused preparation step (xllm-io review, section 3.5:
 * RMSNorm/PTS + pair-top-k 4:8 in-pairs mask + sparse compression + dense
 * residual construction; kasblo.com explainer, steps 1-3).
 * d_X:      bf16 [rows][K] row-major.
 * d_gamma:  bf16 [K] RMSNorm weight, or NULL for an input that is not
 *           normalised (Xn = X).
 * eps:      RMSNorm epsilon.
 * d_row_index: NULL (row t of the output is row t of X) or int32 [a->T]
 *           (row t of the output is row d_row_index[t] of X, or a row of
 *           zeros where d_row_index[t] < 0; MoE gather with padding).
 * a:        view from sharq_act_view(T, K, mode).
 * Arithmetic (bit-exact contract):
 *   inv = f32(1/sqrt(sum(x^2)/K + eps)) with the sum, division and sqrt in
 *   float64; Xn = bf16_rn(f32(f32(x*inv)*gamma)).  s_g = f32(max|Xn| / 2688).
 *   Pair score max(|x_2p|,|x_2p+1|) per 8 consecutive K; keep the 2 largest,
 *   ties to the lower pair index.  Per block: sb = e4m3_rn_satfinite(
 *   f32(amax / f32(6*s_g))), S = f32(dec(sb)*s_g), inv = S>0 ? f32(1/S) : 0,
 *   code = e2m1_rn_satfinite(f32(v*inv)).  Backbone blocks are 32 logical K
 *   (16 kept values); residual R = f32(Xn - f32(val*dec(sb)*s_g)) at kept
 *   positions and Xn elsewhere, in 16-element blocks.
 */
int sharq_prep(const void *d_X, const void *d_gamma, float eps, const int *d_row_index,
               const sharq_act *a, sharq_stream_t stream);

/*
 * sharq_prep_residual - sharq_prep of the updated residual stream.
 * A pre-norm decoder layer adds a sublayer's output to the residual stream
 * and normalises the sum before the next linear layer; the kasblo.com
 * explainer (section 4, on fusing the preparation) counts that epilogue
 * among what the prep kernel takes in.  This call does both in the same
 * kernels: the prep input is h = bf16_rn(f32(x) + f32(res)), element by
 * element (a bf16 framework's x + res), and h is written out as the new
 * residual stream.  Outputs in `a` are those of sharq_prep on h, bit for bit.
 * d_X:       bf16 [a->T][K] row-major, the sublayer output.
 * d_res:     bf16 [a->T][K] row-major, the residual stream.
 * d_res_out: bf16 [a->T][K] that receives h, or NULL (h not stored).  It may
 *            be d_res itself (in-place update: each element is read and then
 *            written by the same thread); it must not overlap d_X, nor
 *            overlap d_res other than exactly.
 * d_gamma, eps, a: as for sharq_prep.  Row gathering is not offered.
 * Errors: as sharq_prep; SHARQ_ERR_INVALID_ARG for a NULL or misaligned
 * (16-byte) d_res or d_res_out, or d_res_out == d_X.  a->T == 0 touches
 * none of the three arrays.
 */
int sharq_prep_residual(const void *d_X, const void *d_res, void *d_res_out, const void *d_gamma, float eps,
                        const sharq_act *a, sharq_stream_t stream);

/*
 * sharq_prep_silu_mul - sharq_prep of the SwiGLU product a down projection
 * takes.  In a Llama-style MLP the down projection's input is SiLU(gate) * up;
 * the kasblo.com explainer (section 4, on fusing the preparation) counts the
 * epilogues before the preparation among what the prep kernel takes in.  The
 * prep input here is, element by element,
 *     h = bf16_rn(f32(silu_bf16(gate)) * f32(up))
 * where silu_bf16(g) is silu(g) = g / (1 + e^-g) correctly rounded to bf16
 * (silu(+-0) = +-0, silu(+inf) = +inf, silu(-inf) = -0), as a bf16 framework
 * stores SiLU(gate) before multiplying by up.  Outputs in `a` are those of
 * sharq_prep on h, bit for bit.
 * d_gate, d_up: bf16 [a->T][K] row-major.
 * d_h:      bf16 [a->T][K] that receives h, or NULL.  It may be d_up itself;
 *           it must not overlap d_gate, nor overlap d_up other than exactly.
 * d_gamma, eps, a: as for sharq_prep (the down projection's input is not
 *           normalised: pass NULL).  Row gathering is not offered.
 * Errors: as sharq_prep_residual.
 */
int sharq_prep_silu_mul(const void *d_gate, const void *d_up, void *d_h, const void *d_gamma, float eps,
                        const sharq_act *a, sharq_stream_t stream);

/*
 * sharq_prep_noalloc - sharq_prep for callers that cannot allocate device
 * memory: a host framework whose memory planner owns all device memory and
 * hands out only the tensors it planned, or a serving loop that must not
 * call cudaMalloc (it can synchronise the device and stall every stream).
 * The paper has no counterpart; this is a deployment variant of the same
 * computation, with results identical to sharq_prep's.
 * Differences from sharq_prep:
 *  - The prep's working memory (device-wide max, grid-barrier counters,
 *    error word, per-row 1/rms) lives in a fixed array inside the library
 *    (256 bytes + 4 bytes per row, up to 16384 rows, about 64 KB, held by
 *    every GPU that loads the library until the process exits).  a->inv_rms
 *    is not written (it may be NULL) and a->gmax_bits[0..2] are not used;
 *    a->gmax_bits may be NULL.  If it is not, the error word is copied to
 *    a->gmax_bits[3], where sharq_linear looks for it; if it is, sharq_linear
 *    on that view has no prep error word to forward.
 *  - a->T > 16384 returns SHARQ_ERR_UNSUPPORTED_SHAPE.
 *  - The first call on each device looks the array's address up
 *    (cudaGetSymbolAddress, a host-side query that allocates nothing).
 *  - Each call clears the array's counters and error words with a 32-byte
 *    cudaMemsetAsync (no allocation).  All calls share the array: calls whose
 *    work overlaps on the GPU (different streams without ordering) race on it.
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
int sharq_prep_noalloc(const void *d_X, const void *d_gamma, float eps, const int *d_row_index,
                       const sharq_act *a, sharq_stream_t stream);

/*
 * sharq_linear - dual-path FP4 GEMM (xllm-io review, sections 3.4-3.5).
 * A 4:8 sparse block-scaled FP4 MMA on the backbone and a dense block-scaled
 * FP4 MMA on the residual accumulate into one TMEM accumulator per output
 * tile; neither branch output is materialised.  Both read the same weight
 * codes, through sf32 (sparse) and sf16 (dense).
 * Launched as a programmatic dependent of the preceding kernel in the
 * stream: set-up and the first weight tiles overlap the tail of sharq_prep,
 * and the activation is read only after that kernel has completed.
 * Y = round(f32(acc * f32(s_g * s_w))) written to d_Y [T][D] row-major,
 * bf16 or float32 per out_dtype.  Mode NVFP4 runs the dense MMA only.
 * d_ws: workspace of at least sharq_workspace_bytes(T, K, D, 1) bytes, zeroed
 * once by the caller after allocation; it receives device-side error codes.
 */
int sharq_linear(const sharq_act *a, const sharq_weight *w, void *d_Y, int out_dtype,
                 void *d_ws, size_t ws_bytes, sharq_stream_t stream);

/*
 * sharq_prep_linear - sharq_prep followed by sharq_linear, as one call
 * (xllm-io review, sections 3.4-3.5).  For decode batches (T <= 32) it runs
 * as ONE kernel: every GEMM CTA reads the T rows of X, computes the row
 * 1/rms and the tensor max itself (identical values in every CTA), and
 * quantizes its own K-slice straight into shared memory in the MMA layout
 * while its weight tiles stream in, so no prepared activation goes through
 * HBM and no separate prep kernel runs.  Codes, scales and Y are the same
 * as sharq_prep + sharq_linear (same arithmetic and order).
 * T > 32 runs sharq_prep into `a` (a view for T rows, SHARQ mode) and then
 * sharq_linear; for T <= 32 `a` is not used and may be NULL.
 * d_X: bf16 [T][K]; d_gamma: bf16 [K] or NULL; w: E == 1; d_Y: [T][D];
 * d_ws: workspace of at least sharq_workspace_bytes(T, K, D, 1) bytes.
 */
#define SHARQ_FUSED_MAX_T 32
int sharq_prep_linear(const void *d_X, const void *d_gamma, float eps, int T, const sharq_act *a,
                      const sharq_weight *w, void *d_Y, int out_dtype, void *d_ws, size_t ws_bytes,
                      sharq_stream_t stream);

/*
 * sharq_linear_grouped - the same GEMM over E experts (xllm-io review,
 * section 5.1: SharQ on the expert linears of Qwen3-30B-A3B).
 * a: one prepared, expert-sorted activation tensor (one PTS scale), usually
 *   gathered by sharq_prep's d_row_index with -1 entries as zero padding
 *   rows so that every expert's group starts on a 128-row tile.
 * d_group_offsets: DEVICE int32 [E+1]; rows offsets[e] .. offsets[e+1]-1 of a
 *   belong to expert e; offsets[0] == 0, non-decreasing, every offset a
 *   multiple of 128, offsets[E] == a->T.  A tile whose expert cannot be found
 *   is skipped and SHARQ_ERR_INVALID_ARG is recorded in d_ws.
 * w: packed weights of all E experts (w->E == E).
 */
int sharq_linear_grouped(const sharq_act *a, const int *d_group_offsets, const sharq_weight *w,
                         void *d_Y, int out_dtype, void *d_ws, size_t ws_bytes,
                         sharq_stream_t stream);

/* Synchronises `stream`, returns the device-side error word of d_ws
 * (SHARQ_OK if none) and clears it. */
int sharq_check_status(void *d_ws, sharq_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *sharq_status_string(int status);

/* SHARQ_ABI_VERSION of the loaded library. */
int sharq_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SHARQ_H */

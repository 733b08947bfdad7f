"""SharQ's sparse-dense decomposition of one linear layer, step by step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows the xllm-io paper review of "SharQ: Bridging Activation Sparsity and
FP4 Quantization for LLM Inference", section 3 (3.1 problem and group
quantization, 3.2 sparse backbone, 3.3 dense residual, 3.4 dual-path GEMM,
3.5 kernel design, 3.6 analysis), and the kasblo.com explainer (4:8 in-pairs,
the residual w.r.t. the quantized backbone, one shared FP4 weight payload).

Floating-point order.  Every float32 step is one IEEE float32 operation done
in numpy float32 (round to nearest even); float64 is used where stated.  The
pages fix none of these orders; the ones below are this library's reading and
the GPU kernels follow the same order, which is what makes codes and scale
bytes comparable bit for bit:

  rmsnorm    ss = sum(x^2) in float64; inv = f32(1/sqrt(ss/K + eps)) in
             float64 rounded once; xn = bf16(f32(f32(x*inv)*gamma)).
  pts        s = f32(gmax / 2688) with 2688 = 6 (E2M1 max) * 448 (E4M3 max);
             s = 1 when gmax = 0.
  quantizer  per block: a = max|v|; sb = E4M3(f32(a / f32(6*s)));
             S = f32(dec(sb)*s); inv = f32(1/S) or 0; code = E2M1(f32(v*inv)).
  dequant    x~ = f32(val(code)*dec(sb)*s)   (val*dec is exact in float32).
  residual   R = f32(xn - x~) at kept positions, R = xn elsewhere.
"""
import numpy as np

from .formats import (bf16_round, e2m1_decode, e2m1_encode, e4m3_decode,
                      e4m3_encode_nonneg, f32, e8m0_decode, mx_scale_exponent)

E2M1_MAX = 6.0
E4M3_MAX = 448.0
GLOBAL_DIV = np.float32(E2M1_MAX * E4M3_MAX)   # 2688


def rmsnorm(x, gamma, eps):
    """RMSNorm fused into the preparation step (xllm-io review, section 3.5:
    "RMSNorm/PTS + pair-topk mask + ... in one preparation kernel").

    x: float32 [T, K] holding bf16 values.  gamma: float32 [K] (bf16 values) or
    None for inputs that are not normalised (then xn = x).  Returns
    (xn float32 [T, K] holding bf16 values, inv float32 [T] or None).
    """
    x = np.asarray(x, dtype=np.float32)
    if gamma is None:
        return x.copy(), None
    T, K = x.shape
    ss = np.sum(x.astype(np.float64) ** 2, axis=1)
    inv = (1.0 / np.sqrt(ss / K + np.float64(np.float32(eps)))).astype(np.float32)
    t1 = (x * inv[:, None]).astype(np.float32)
    t2 = (t1 * np.asarray(gamma, dtype=np.float32)[None, :]).astype(np.float32)
    return bf16_round(t2), inv


def pts_scale(xn):
    """Per-tensor FP32 global scale computed online from the current tensor
    (xllm-io review, sections 3.1 and 3.5, "PTS"; the kasblo.com explainer
    notes SharQ needs no calibration data for it).

    s = gmax / (6 * 448): maps the tensor amax onto the largest E2M1 value
    times the largest E4M3 block scale.
    """
    gmax = np.float32(np.max(np.abs(xn))) if xn.size else np.float32(0)
    if gmax == 0:
        return np.float32(1.0), gmax
    return np.float32(gmax / GLOBAL_DIV), gmax


def pair_mask(xn):
    """4:8 in-pairs mask (xllm-io review, section 3.2; kasblo.com explainer:
    8 consecutive values form 4 pairs, keep 2 pairs = 4 values).

    Pair score = max(|x_2p|, |x_2p+1|).  Keep the 2 highest scores; on equal
    scores the lower pair index wins.  Pair p is kept iff fewer than 2 pairs q
    beat it, where q beats p if s_q > s_p, or s_q == s_p and q < p.

    Returns keep bool [T, K/8, 4] and meta uint8 [T, K/8] = p_lo | p_hi << 2.
    """
    T, K = xn.shape
    a = np.abs(xn.reshape(T, K // 8, 4, 2))
    s = np.max(a, axis=-1)                                     # [T, C, 4]
    beats = np.zeros(s.shape + (4,), dtype=bool)               # [.., p, q]
    for p in range(4):
        for q in range(4):
            if q == p:
                continue
            beats[..., p, q] = (s[..., q] > s[..., p]) | ((s[..., q] == s[..., p]) & (q < p))
    keep = beats.sum(axis=-1) < 2
    idx = np.argsort(~keep, axis=-1, kind="stable")[..., :2]   # kept, ascending
    meta = (idx[..., 0] | (idx[..., 1] << 2)).astype(np.uint8)
    return keep, meta


def nvfp4_quant(v, s):
    """Group-symmetric NVFP4 quantization of blocks (xllm-io review, section
    3.1: s_G = max|x| / alpha_B, plus the second-level FP32 global scale s).

    v: float32 [..., n] (one block per last axis).  s: float32 global scale.
    Returns (codes uint8 [..., n], sb uint8 [...] E4M3 bytes, deq float32
    [..., n] = f32(val * dec(sb) * s)).
    """
    v = np.asarray(v, dtype=np.float32)
    s = np.float32(s)
    a = np.max(np.abs(v), axis=-1)
    denom = np.float32(np.float32(6.0) * s)
    t = (a / denom).astype(np.float32)
    sb = e4m3_encode_nonneg(t)
    dec = e4m3_decode(sb).astype(np.float32)
    S = (dec * s).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(S > 0, (np.float32(1.0) / S).astype(np.float32), np.float32(0.0))
    y = (v * inv[..., None]).astype(np.float32)
    codes = e2m1_encode(y)
    vd = (e2m1_decode(codes) * dec[..., None].astype(np.float64))   # exact
    deq = f32(vd * np.float64(s))
    return codes, sb, deq


def prep(x, gamma=None, eps=1e-5, s_g=None):
    """The fused preparation step (xllm-io review, sections 3.2-3.5;
    kasblo.com explainer, steps 1-3).

    x: float32 [T, K] holding bf16 values, K a multiple of 32.
    s_g: None (the per-tensor scale of x itself, section 3.5 "PTS"), or the
    scale of a larger tensor that these rows are a subset of.
    Returns a dict of logical (untiled) arrays:
      xn [T,K], inv [T] or None, s_g, gmax,
      keep [T,K/8,4], meta [T,K/8]           4:8 in-pairs mask
      sp_vals [T,K/2]                         kept values, ascending K
      sp_codes [T,K/2], sp_sf [T,K/32]        backbone NVFP4 (32 logical K/scale)
      xsp [T,K], xsp_t [T,K]                  X_sp and dequantized X~_sp
      r [T,K]                                 R = Xn - X~_sp (float32)
      r_codes [T,K], r_sf [T,K/16], r_t [T,K] residual NVFP4 (16 K/scale)
    """
    xn, inv = rmsnorm(x, gamma, eps)
    T, K = xn.shape
    if s_g is None:
        s_g, gmax = pts_scale(xn)
    else:
        s_g, gmax = np.float32(s_g), None
    keep, meta = pair_mask(xn)
    keep_el = np.repeat(keep, 2, axis=-1).reshape(T, K)               # [T,K]
    xsp = np.where(keep_el, xn, np.float32(0)).astype(np.float32)
    # compress: kept values of each chunk in ascending K order
    sp_vals = xn[keep_el].reshape(T, K // 2)
    # backbone: one scale per 32 logical K = 16 kept values
    codes, sb, deq = nvfp4_quant(sp_vals.reshape(T, K // 32, 16), s_g)
    sp_codes = codes.reshape(T, K // 2)
    xsp_t = np.zeros((T, K), dtype=np.float32)
    xsp_t[keep_el] = deq.reshape(-1)
    # residual w.r.t. the quantized backbone (section 3.3)
    r = np.where(keep_el, (xn - xsp_t).astype(np.float32), xn).astype(np.float32)
    rc, rsb, rdeq = nvfp4_quant(r.reshape(T, K // 16, 16), s_g)
    return dict(xn=xn, inv=inv, s_g=s_g, gmax=gmax, keep=keep, meta=meta,
                sp_vals=sp_vals, sp_codes=sp_codes, sp_sf=sb, xsp=xsp,
                xsp_t=xsp_t, r=r, r_codes=rc.reshape(T, K), r_sf=rsb,
                r_t=rdeq.reshape(T, K))


def pack_weight(w):
    """Shared FP4 weight payload with two scale views (xllm-io review,
    section 3.5: one FP4 weight body, sparse path group-32 scales, dense path
    group-16 scales duplicated; kasblo.com explainer, step 3).

    w: float32 [K, D] holding bf16 values (W in R^{K x D}, section 3.1).
    Quantized per output column d along K with one scale per 32 K.
    Returns dict: codes [D,K] (E2M1 codes), sf32 [D,K/32], sf16 [D,K/16]
    (each sf32 byte twice), s_w, w_t [K,D] dequantized float64 without s_w,
    i.e. val*dec(sb).
    """
    w = np.asarray(w, dtype=np.float32)
    K, D = w.shape
    amax = np.float32(np.max(np.abs(w))) if w.size else np.float32(0)
    s_w = np.float32(1.0) if amax == 0 else np.float32(amax / GLOBAL_DIV)
    wt = np.ascontiguousarray(w.T)                                     # [D,K]
    codes, sb, _ = nvfp4_quant(wt.reshape(D, K // 32, 32), s_w)
    codes = codes.reshape(D, K)
    sf16 = np.repeat(sb, 2, axis=-1)
    w_t = (e2m1_decode(codes).reshape(D, K // 32, 32)
           * e4m3_decode(sb)[..., None]).reshape(D, K).T
    return dict(codes=codes, sf32=sb, sf16=sf16, s_w=s_w, w_t=np.ascontiguousarray(w_t))


def dequant_sparse(p):
    """val(code)*dec(sb) of the backbone, scattered to [T,K], float64."""
    T, K = p["xn"].shape
    vals = (e2m1_decode(p["sp_codes"]).reshape(T, K // 32, 16)
            * e4m3_decode(p["sp_sf"])[..., None]).reshape(T, K // 2)
    keep_el = np.repeat(p["keep"], 2, axis=-1).reshape(T, K)
    out = np.zeros((T, K), dtype=np.float64)
    out[keep_el] = vals.reshape(-1)
    return out


def dequant_residual(p):
    """val(code)*dec(sb) of the residual, [T,K], float64."""
    T, K = p["xn"].shape
    return (e2m1_decode(p["r_codes"]).reshape(T, K // 16, 16)
            * e4m3_decode(p["r_sf"])[..., None]).reshape(T, K)


def linear(p, wq):
    """Dual-path GEMM of section 3.4 in float64 from the dequantized operands:

        Y = GEMM_sp(Q_sp(X_sp), Q_w,sp(W)) + GEMM_dn(Q_dn(R), Q_w,dn(W))

    Both GEMMs read the same weight codes; the sparse one through the
    per-32 scales and the dense one through the per-16 view (equal values).
    The global scales s_g * s_w multiply the sum (one accumulator).
    Returns float64 [T, D].
    """
    a_sp = dequant_sparse(p)
    a_dn = dequant_residual(p)
    w32 = wq["w_t"]
    K, D = w32.shape
    w16 = (e2m1_decode(wq["codes"]).reshape(D, K // 16, 16)
           * e4m3_decode(wq["sf16"])[..., None]).reshape(D, K).T
    y = a_sp @ w32 + a_dn @ w16
    return y * (_row_scale(p["s_g"], y.shape[0]) * np.float64(wq["s_w"]))


def _row_scale(s_g, T):
    """The global activation scale as a float64 column: one value for the
    per-tensor scale, one per row for the per-token reading."""
    s = np.asarray(s_g, dtype=np.float64)
    return s if s.ndim == 0 else s.reshape(T, 1)


def prep_per_token(x, gamma=None, eps=1e-5):
    """SharQ preparation with the global scale read as per-TOKEN (the
    alternative expansion of "PTS", xllm-io review, sections 3.1 and 3.5): every
    row gets its own s_t = max|Xn[t]| / (6*448) (1 for an all-zero row), and
    each row is prepared exactly as the per-tensor prep() of that row alone
    with s_g = s_t.  Both activation paths of a row share s_t, so the two
    MMAs still add into one accumulator row.  Returns the prep() dict with
    s_g (and gmax) as float32 arrays [T]."""
    x = np.asarray(x, dtype=np.float32)
    T = x.shape[0]
    xn, _ = rmsnorm(x, gamma, eps)
    scales = [pts_scale(xn[t:t + 1]) for t in range(T)]
    rows = [prep(x[t:t + 1], gamma, eps, s_g=scales[t][0]) for t in range(T)]
    out = {}
    for k, v in prep(x[:1] if T else x, gamma, eps).items():
        if k == "s_g":
            out[k] = np.array([sc[0] for sc in scales], np.float32)
        elif k == "gmax":
            out[k] = np.array([sc[1] for sc in scales], np.float32)
        elif v is None or not T:
            out[k] = v
        else:
            out[k] = np.concatenate([r[k] for r in rows], axis=0)
    return out


def epilogue_f32(y64, s_g, s_w):
    """Output rounding for the float32 output mode: the scaled float64
    product rounded to float32 (the reference the float32 output is compared
    against)."""
    return f32(y64)


def linear_grouped(p, wqs, offsets):
    """Grouped form for MoE expert linears (xllm-io review, section 5.1: SharQ
    applies to the expert linear layers of Qwen3-30B-A3B).

    p: prep() of the whole expert-sorted activation tensor (one PTS scale for
    the tensor).  wqs: pack_weight() per expert.  offsets: int [E+1], rows
    offsets[e]:offsets[e+1] belong to expert e.  Returns float64 [rows, D].
    """
    T = p["xn"].shape[0]
    D = wqs[0]["w_t"].shape[1]
    y = np.zeros((T, D), dtype=np.float64)
    for e, wq in enumerate(wqs):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi <= lo:
            continue
        sub = {k: (v[lo:hi] if isinstance(v, np.ndarray) and v.ndim >= 1
                   and v.shape[0] == T else v) for k, v in p.items()}
        y[lo:hi] = linear(sub, wq)
    return y


# ------------------------------------------------- Table-5 path modes ----
# The xllm-io review's ablation (section 5.3, Table 5) compares the SharQ
# decomposition with three other ways of splitting the activation into two
# FP4 operands.  The page names them only; the plainest reading, used here,
# keeps every other step of the method (RMSNorm, the per-tensor scale, the
# block quantizer, the 4:8 in-pairs rule):
#   Sparse only    the backbone alone (no residual operand);
#   Dense+Dense    dense NVFP4 of Xn (16-element blocks), then dense NVFP4 of
#                  its residual Xn - dequant;
#   Sparse+Sparse  the SharQ backbone, then the residual R pruned by the same
#                  4:8 in-pairs rule (scores max|R|) and quantized as a
#                  sparse operand (one scale per 32 logical K).

def prep_dense_dense(x, gamma=None, eps=1e-5):
    """Dense+Dense mode.  Returns dict xn, inv, s_g, gmax, b_codes [T,K],
    b_sf [T,K/16], b_t (dequantized first level), r [T,K] = Xn - b_t
    (float32), r_codes [T,K], r_sf [T,K/16], r_t."""
    xn, inv = rmsnorm(x, gamma, eps)
    T, K = xn.shape
    s_g, gmax = pts_scale(xn)
    bc, bsb, bdeq = nvfp4_quant(xn.reshape(T, K // 16, 16), s_g)
    b_t = bdeq.reshape(T, K)
    r = (xn - b_t).astype(np.float32)
    rc, rsb, rdeq = nvfp4_quant(r.reshape(T, K // 16, 16), s_g)
    return dict(xn=xn, inv=inv, s_g=s_g, gmax=gmax, b_codes=bc.reshape(T, K), b_sf=bsb, b_t=b_t, r=r,
                r_codes=rc.reshape(T, K), r_sf=rsb, r_t=rdeq.reshape(T, K))


def prep_sparse_sparse(x, gamma=None, eps=1e-5):
    """Sparse+Sparse mode: prep() for the backbone and R, then R pruned and
    quantized like the backbone.  Adds r_keep [T,K/8,4], r_meta [T,K/8],
    r_sp_vals [T,K/2], r_sp_codes [T,K/2], r_sp_sf [T,K/32], r_sp_t [T,K]
    (dequantized residual scattered to its kept positions)."""
    p = prep(x, gamma, eps)
    r = p["r"]
    T, K = r.shape
    keep, meta = pair_mask(r)
    keep_el = np.repeat(keep, 2, axis=-1).reshape(T, K)
    vals = r[keep_el].reshape(T, K // 2)
    codes, sb, deq = nvfp4_quant(vals.reshape(T, K // 32, 16), p["s_g"])
    r_sp_t = np.zeros((T, K), dtype=np.float32)
    r_sp_t[keep_el] = deq.reshape(-1)
    out = {k: v for k, v in p.items() if k not in ("r_codes", "r_sf", "r_t")}
    out.update(r_keep=keep, r_meta=meta, r_sp_vals=vals, r_sp_codes=codes.reshape(T, K // 2), r_sp_sf=sb,
               r_sp_t=r_sp_t)
    return out


def approx_activation(x, gamma=None, eps=1e-5, mode="sharq"):
    """The activation each mode hands to the GEMMs, dequantized, float64
    without the global scale folded out: X~ with Y~ = X~ W.  Modes: "nvfp4",
    "sharq", "sparse_only", "dense_dense", "sparse_sparse"."""
    if mode == "nvfp4":
        return prep_nvfp4(x, gamma, eps)["x_t"].astype(np.float64)
    if mode == "dense_dense":
        p = prep_dense_dense(x, gamma, eps)
        return p["b_t"].astype(np.float64) + p["r_t"].astype(np.float64)
    if mode == "sparse_sparse":
        p = prep_sparse_sparse(x, gamma, eps)
        return p["xsp_t"].astype(np.float64) + p["r_sp_t"].astype(np.float64)
    p = prep(x, gamma, eps)
    if mode == "sparse_only":
        return p["xsp_t"].astype(np.float64)
    return p["xsp_t"].astype(np.float64) + p["r_t"].astype(np.float64)


def linear_mode(p, wq, mode):
    """Float64 GEMM of a Table-5 mode from its prep dict: the operands the
    GPU multiplies (dequantized codes times scale values) times the weight
    view each operand is paired with, times s_g * s_w."""
    K, D = wq["w_t"].shape
    w32 = wq["w_t"]
    w16 = (e2m1_decode(wq["codes"]).reshape(D, K // 16, 16)
           * e4m3_decode(wq["sf16"])[..., None]).reshape(D, K).T
    if mode == "sparse_only":
        y = dequant_sparse(p) @ w32
    elif mode == "dense_dense":
        T = p["xn"].shape[0]
        dq = lambda c, sf: (e2m1_decode(c).reshape(T, K // 16, 16) * e4m3_decode(sf)[..., None]).reshape(T, K)
        y = dq(p["b_codes"], p["b_sf"]) @ w16 + dq(p["r_codes"], p["r_sf"]) @ w16
    elif mode == "sparse_sparse":
        T = p["xn"].shape[0]
        r = {"xn": p["xn"], "keep": p["r_keep"], "sp_codes": p["r_sp_codes"], "sp_sf": p["r_sp_sf"]}
        y = dequant_sparse(p) @ w32 + dequant_sparse(r) @ w32
    else:
        raise ValueError(mode)
    return y * (_row_scale(p["s_g"], y.shape[0]) * np.float64(wq["s_w"]))


# ------------------------------------------------------------- MXFP4 -----
# The xllm-io review (section 5.3, "FP4 format generalisation") runs SharQ on
# NVFP4, HiF4 and MXFP4.  MXFP4 is the OCP Microscaling format: E2M1 elements,
# one E8M0 (power-of-two) scale per 32 elements, no second-level scale.  The
# pages pair MXFP4 with 2:4 sparsity; the sparse FP4 MMA of sm_100 takes only
# the 4:8 in-pairs pattern, so the backbone keeps the 4:8 in-pairs mask, and
# its scale covers 64 logical K (32 kept values), the granularity of that
# MMA for E8M0 scales; the dense residual uses the MXFP4 32-element blocks.

def mx_quant(v):
    """MXFP4 quantization of blocks (last axis): X = 2^e, e = floor(log2
    amax) - 2 (E8M0 byte e + 127), codes = E2M1(v / X) with round to nearest
    even and saturation, deq = f32(val * X) (exact).  Returns (codes, sb,
    deq)."""
    v = np.asarray(v, dtype=np.float32)
    e = mx_scale_exponent(np.max(np.abs(v), axis=-1))
    y = (v.astype(np.float64) * np.ldexp(1.0, -e)[..., None]).astype(np.float32)
    codes = e2m1_encode(y)
    deq = f32(e2m1_decode(codes) * np.ldexp(1.0, e)[..., None])
    return codes, (e + 127).astype(np.uint8), deq


def prep_mxfp4(x, gamma=None, eps=1e-5):
    """SharQ with MXFP4 operands: RMSNorm, the 4:8 in-pairs mask, the kept
    values quantized with one E8M0 scale per 64 logical K, the residual
    R = Xn - X~_sp (exact) in MXFP4 32-element blocks.  s_g = 1 (MX formats
    have no tensor scale).  Same keys as prep()."""
    xn, inv = rmsnorm(x, gamma, eps)
    T, K = xn.shape
    keep, meta = pair_mask(xn)
    keep_el = np.repeat(keep, 2, axis=-1).reshape(T, K)
    xsp = np.where(keep_el, xn, np.float32(0)).astype(np.float32)
    sp_vals = xn[keep_el].reshape(T, K // 2)
    codes, sb, deq = mx_quant(sp_vals.reshape(T, K // 64, 32))
    xsp_t = np.zeros((T, K), dtype=np.float32)
    xsp_t[keep_el] = deq.reshape(-1)
    r = np.where(keep_el, (xn - xsp_t).astype(np.float32), xn).astype(np.float32)
    rc, rsb, rdeq = mx_quant(r.reshape(T, K // 32, 32))
    return dict(xn=xn, inv=inv, s_g=np.float32(1.0), gmax=None, keep=keep, meta=meta, sp_vals=sp_vals,
                sp_codes=codes.reshape(T, K // 2), sp_sf=sb, xsp=xsp, xsp_t=xsp_t, r=r, r_codes=rc.reshape(T, K),
                r_sf=rsb, r_t=rdeq.reshape(T, K))


def prep_mxfp4_plain(x, gamma=None, eps=1e-5):
    """Plain MXFP4 of Xn (32-element blocks), the MXFP4 comparator.  Returns
    dict xn, inv, s_g (= 1), codes [T,K], sf [T,K/32], x_t."""
    xn, inv = rmsnorm(x, gamma, eps)
    T, K = xn.shape
    c, sb, deq = mx_quant(xn.reshape(T, K // 32, 32))
    return dict(xn=xn, inv=inv, s_g=np.float32(1.0), codes=c.reshape(T, K), sf=sb, x_t=deq.reshape(T, K))


def pack_weight_mx(w):
    """The shared weight payload in MXFP4: W in R^{K x D} quantized per
    output column with one E8M0 scale per 64 K (the sparse path's
    granularity); the dense path's per-32 view repeats each scale byte.
    Returns codes [D,K], sf64 [D,K/64], sf32 [D,K/32], s_w = 1, w_t [K,D]
    dequantized (float64)."""
    w = np.asarray(w, dtype=np.float32)
    K, D = w.shape
    c, sb, deq = mx_quant(w.T.reshape(D, K // 64, 64))
    return dict(codes=c.reshape(D, K), sf64=sb, sf32=np.repeat(sb, 2, axis=-1), s_w=np.float32(1.0),
                w_t=deq.reshape(D, K).T.astype(np.float64))


def linear_mx(p, wq):
    """Float64 GEMM of MXFP4-SharQ (or of the plain MXFP4 comparator when p
    has "codes"): each operand's dequantized values times the weight view it
    is paired with (per-64 for the backbone, per-32 for dense operands)."""
    K, D = wq["w_t"].shape
    T = p["xn"].shape[0]
    w64 = (e2m1_decode(wq["codes"]).reshape(D, K // 64, 64) * e8m0_decode(wq["sf64"])[..., None]).reshape(D, K).T
    w32 = (e2m1_decode(wq["codes"]).reshape(D, K // 32, 32) * e8m0_decode(wq["sf32"])[..., None]).reshape(D, K).T
    if "codes" in p:  # plain MXFP4
        a = (e2m1_decode(p["codes"]).reshape(T, K // 32, 32) * e8m0_decode(p["sf"])[..., None]).reshape(T, K)
        return a @ w32
    vals = (e2m1_decode(p["sp_codes"]).reshape(T, K // 64, 32) * e8m0_decode(p["sp_sf"])[..., None]).reshape(T, K // 2)
    keep_el = np.repeat(p["keep"], 2, axis=-1).reshape(T, K)
    a_sp = np.zeros((T, K), dtype=np.float64)
    a_sp[keep_el] = vals.reshape(-1)
    a_r = (e2m1_decode(p["r_codes"]).reshape(T, K // 32, 32) * e8m0_decode(p["r_sf"])[..., None]).reshape(T, K)
    return a_sp @ w64 + a_r @ w32


def residual_add(x, res):
    """The residual-stream update a pre-norm decoder layer performs before
    the next RMSNorm, fused into the preparation step (the kasblo.com
    explainer notes that RMSNorm and the preceding epilogues are fused into
    the preparation kernel): h = bf16_rn(f32(x + res)) for bf16 x and res
    (float32 [T, K] holding bf16 values) -- the float32 sum, rounded to
    nearest even in bfloat16, as a bf16 framework computes it."""
    x = np.asarray(x, dtype=np.float32)
    r = np.asarray(res, dtype=np.float32)
    return bf16_round((x + r).astype(np.float32))


def bf16_round_f64(x):
    """Round float64 to the nearest bfloat16 (ties to even) in ONE rounding,
    not through float32; returns float32.  bfloat16 keeps 8 significant bits
    and float32's exponent range: the quantum of a value in [2^e, 2^(e+1)) is
    2^(e-7), and 2^-133 below 2^-126.  Finite inputs; the sign of zero is
    kept."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                     # x = m 2^e, 1/2 <= |m| < 1
    q = np.maximum(e, -125) - 8            # log2 of the quantum
    r = np.ldexp(np.round(np.ldexp(x, -q)), q)  # x / 2^q is exact; np.round ties to even
    return np.copysign(r, x).astype(np.float32)


def _bf16_midpoint(x):
    """True where float64 x lies exactly halfway between two bfloat16s."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.maximum(e, -125) - 8
    t = np.ldexp(x, -q)
    return (t - np.floor(t)) == 0.5


def silu_bf16(g):
    """SiLU of bf16 values rounded once to bfloat16 (ties cannot occur: silu(g)
    is transcendental for g != 0).  silu(g) = g / (1 + e^-g), evaluated in
    float64 in three forms that avoid overflow and cancellation:
      g >= 1:   g / (1 + e^-g)
      g <= -1:  g e^g / (1 + e^g)
      |g| < 1:  g/2 + d with d = (g/2) tanh(g/2) >= 0 (silu(g) - g/2 = d), kept
                as the float64 pair hi + lo (Knuth's two-sum), so that a hi
                lying exactly on a bf16 midpoint -- g/2 for tiny g -- rounds
                in the direction of lo.
    silu(+inf) = +inf, silu(-inf) = -0, NaN stays NaN.  Input: float32 holding
    bf16 values; returns float32 holding bf16 values."""
    with np.errstate(invalid="ignore"):  # signalling NaN patterns
        g = np.asarray(g, dtype=np.float32).astype(np.float64)
    fin = np.isfinite(g)
    gf = np.where(fin, g, 0.0)
    with np.errstate(over="ignore", under="ignore", invalid="ignore"):
        e = np.exp(-np.abs(gf))                              # in (0, 1]
        big = np.where(gf >= 0, gf / (1.0 + e), gf * e / (1.0 + e))
        a = gf / 2.0                                         # exact
        d = a * np.tanh(a)
        hi = a + d
        bb = hi - a
        lo = (a - (hi - bb)) + (d - bb)                      # hi + lo = a + d exactly
    small = np.abs(gf) < 1.0
    hi = np.where(small, hi, big)
    lo = np.where(small, lo, 0.0)
    r = bf16_round_f64(hi).astype(np.float64)
    # a hi exactly halfway between two bf16s goes to the neighbour on lo's side
    # (half a quantum away; the quantum is that of the lower neighbour)
    tie = _bf16_midpoint(hi) & (lo != 0.0)
    _, ex = np.frexp(hi)
    quantum = np.ldexp(1.0, np.maximum(ex, -125) - 8)
    r = np.where(tie, hi + np.sign(lo) * quantum / 2.0, r)
    # silu(g) has the sign of g (silu(g) / g = sigmoid(g) > 0), zeros included
    out = np.copysign(r, gf).astype(np.float32)
    out = np.where(fin, out, np.where(np.isnan(g), np.float32(np.nan),
                                      np.where(g > 0, np.float32(np.inf), np.float32(-0.0))))
    return out.astype(np.float32)


def silu_mul(gate, up):
    """The SwiGLU product the down projection of a Llama-style MLP takes,
    fused into its preparation step (the kasblo.com explainer, section 4 on
    fusing the preparation: the epilogues before it join the prep kernel):
        h = bf16_rn(f32(silu_bf16(gate) * up))
    for bf16 gate and up (float32 arrays holding bf16 values) -- the SiLU
    rounded to bf16 as a bf16 framework stores it, then the bf16 product (two
    bf16 values multiply exactly in float32 unless the product underflows;
    the float32 product is rounded to bf16)."""
    s = silu_bf16(gate)
    u = np.asarray(up, dtype=np.float32)
    with np.errstate(over="ignore", under="ignore"):
        return bf16_round((s * u).astype(np.float32))


def prep_nvfp4(x, gamma=None, eps=1e-5):
    """Plain NVFP4 preparation, the comparator the SharQ evaluation reports
    as "NVFP4" (xllm-io review, Table 1; the kasblo.com explainer lists the
    official repository's NVFP4 mode): RMSNorm, the same PTS global scale, and
    every 16-element block of Xn quantized directly, with no mask and no
    residual.  Returns dict xn, inv, s_g, gmax, codes [T,K], sf [T,K/16],
    x_t [T,K] (dequantized, float32)."""
    xn, inv = rmsnorm(x, gamma, eps)
    T, K = xn.shape
    s_g, gmax = pts_scale(xn)
    c, sb, deq = nvfp4_quant(xn.reshape(T, K // 16, 16), s_g)
    return dict(xn=xn, inv=inv, s_g=s_g, gmax=gmax, codes=c.reshape(T, K),
                sf=sb, x_t=deq.reshape(T, K))


def linear_nvfp4(p, wq):
    """Dense NVFP4 GEMM of the plain-NVFP4 comparator in float64."""
    T, K = p["xn"].shape
    a = (e2m1_decode(p["codes"]).reshape(T, K // 16, 16)
         * e4m3_decode(p["sf"])[..., None]).reshape(T, K)
    D = wq["w_t"].shape[1]
    w16 = (e2m1_decode(wq["codes"]).reshape(D, K // 16, 16)
           * e4m3_decode(wq["sf16"])[..., None]).reshape(D, K).T
    return (a @ w16) * (_row_scale(p["s_g"], a.shape[0]) * np.float64(wq["s_w"]))

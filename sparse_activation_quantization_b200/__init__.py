"""Python binding of the SharQ CUDA library (``libsharq.so``, sm_100a).

Argument marshalling only: every step of the path runs in the library's
kernels.  PyTorch is used for device memory and streams.  The functions with
``sharq_`` names mirror the C ABI of ``include/sharq.h`` one to one (raw
device pointers as ints, ctypes structs for the views); ``PackedWeight``,
``PreparedAct`` and ``linear`` are conveniences that allocate the buffers
with torch and call those functions.

There is no CPU or PyTorch fallback: if the library is missing or the device
is not sm_100, the calls raise.
"""
import ctypes
import os

__all__ = [
    "SharqError", "SharqAct", "SharqWeight", "lib", "library_path",
    "SHARQ_MODE_SHARQ", "SHARQ_MODE_NVFP4", "SHARQ_MODE_SHARQ_TOKEN", "SHARQ_MODE_SPARSE_ONLY",
    "SHARQ_MODE_DENSE_DENSE", "SHARQ_MODE_SPARSE_SPARSE", "SHARQ_MODE_MXFP4", "SHARQ_MODE_MXFP4_PLAIN",
    "SHARQ_FMT_NVFP4", "SHARQ_FMT_MXFP4", "SHARQ_OUT_BF16", "SHARQ_OUT_F32",
    "sharq_weight_bytes_fmt", "sharq_weight_view_fmt",
    "sharq_weight_bytes", "sharq_act_bytes", "sharq_workspace_bytes",
    "sharq_weight_view", "sharq_act_view", "sharq_pack_weight", "sharq_prep",
    "sharq_linear", "sharq_linear_grouped", "sharq_check_status",
    "sharq_status_string", "sharq_abi_version", "sharq_prep_noalloc", "sharq_prep_linear", "prep_linear",
    "sharq_prep_residual", "sharq_prep_silu_mul",
    "PackedWeight", "PreparedAct", "Workspace", "linear", "EXPORTED_SYMBOLS",
]

SHARQ_MODE_SHARQ = 0
SHARQ_MODE_NVFP4 = 1
SHARQ_MODE_SHARQ_TOKEN = 2
SHARQ_MODE_SPARSE_ONLY = 3
SHARQ_MODE_DENSE_DENSE = 4
SHARQ_MODE_SPARSE_SPARSE = 5
SHARQ_MODE_MXFP4 = 6
SHARQ_MODE_MXFP4_PLAIN = 7
SHARQ_FMT_NVFP4 = 0
SHARQ_FMT_MXFP4 = 1
SHARQ_OUT_BF16 = 0
SHARQ_OUT_F32 = 1

EXPORTED_SYMBOLS = (
    "sharq_weight_bytes", "sharq_act_bytes", "sharq_workspace_bytes", "sharq_weight_view",
    "sharq_act_view", "sharq_pack_weight", "sharq_prep", "sharq_linear", "sharq_linear_grouped",
    "sharq_check_status", "sharq_status_string", "sharq_abi_version", "sharq_prep_noalloc",
    "sharq_prep_linear", "sharq_weight_bytes_fmt", "sharq_weight_view_fmt", "sharq_prep_residual",
    "sharq_prep_silu_mul",
)

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libsharq.so")
_lib = None


class SharqError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        name = lib().sharq_status_string(status).decode() if _lib else str(status)
        super().__init__(f"{where}: {name} ({status})")


class SharqWeight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf32", ctypes.c_void_p), ("sf16", ctypes.c_void_p),
                ("s_w", ctypes.c_void_p), ("K", ctypes.c_int), ("D", ctypes.c_int), ("E", ctypes.c_int),
                ("fmt", ctypes.c_int)]


class SharqAct(ctypes.Structure):
    _fields_ = [("sp_codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("sp_sf", ctypes.c_void_p),
                ("r_codes", ctypes.c_void_p), ("r_sf", ctypes.c_void_p), ("inv_rms", ctypes.c_void_p),
                ("s_g", ctypes.c_void_p), ("gmax_bits", ctypes.c_void_p),
                ("T", ctypes.c_int), ("Tp", ctypes.c_int), ("K", ctypes.c_int), ("mode", ctypes.c_int),
                ("r_meta", ctypes.c_void_p)]


def lib():
    """Load libsharq.so (in-tree build); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"{library_path} missing: build it with "
                               "`python -m sparse_activation_quantization_b200.build`")
        L = ctypes.CDLL(library_path)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        W, A = ctypes.POINTER(SharqWeight), ctypes.POINTER(SharqAct)
        sig = {
            "sharq_weight_bytes": (sz, [i, i, i]),
            "sharq_act_bytes": (sz, [i, i, i]),
            "sharq_workspace_bytes": (sz, [i, i, i, i]),
            "sharq_weight_view": (i, [vp, i, i, i, W]),
            "sharq_weight_bytes_fmt": (sz, [i, i, i, i]),
            "sharq_weight_view_fmt": (i, [vp, i, i, i, i, W]),
            "sharq_act_view": (i, [vp, i, i, i, A]),
            "sharq_pack_weight": (i, [vp, W, vp]),
            "sharq_prep": (i, [vp, vp, ctypes.c_float, vp, A, vp]),
            "sharq_prep_noalloc": (i, [vp, vp, ctypes.c_float, vp, A, vp]),
            "sharq_prep_residual": (i, [vp, vp, vp, vp, ctypes.c_float, A, vp]),
            "sharq_prep_silu_mul": (i, [vp, vp, vp, vp, ctypes.c_float, A, vp]),
            "sharq_linear": (i, [A, W, vp, i, vp, sz, vp]),
            "sharq_prep_linear": (i, [vp, vp, ctypes.c_float, i, A, W, vp, i, vp, sz, vp]),
            "sharq_linear_grouped": (i, [A, vp, W, vp, i, vp, sz, vp]),
            "sharq_check_status": (i, [vp, vp]),
            "sharq_status_string": (ctypes.c_char_p, [i]),
            "sharq_abi_version": (i, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(status, where):
    if status != 0:
        raise SharqError(status, where)
    return status

# ----------------------------------------------------------- C ABI mirror ---


def sharq_abi_version():
    return lib().sharq_abi_version()


def sharq_status_string(status):
    return lib().sharq_status_string(status).decode()


def sharq_weight_bytes(K, D, E=1):
    return lib().sharq_weight_bytes(K, D, E)


def sharq_weight_bytes_fmt(K, D, E=1, fmt=SHARQ_FMT_NVFP4):
    return lib().sharq_weight_bytes_fmt(K, D, E, fmt)


def sharq_act_bytes(T, K, mode=SHARQ_MODE_SHARQ):
    return lib().sharq_act_bytes(T, K, mode)


def sharq_workspace_bytes(T, K, D, E=1):
    return lib().sharq_workspace_bytes(T, K, D, E)


def sharq_weight_view(d_buf, K, D, E=1):
    w = SharqWeight()
    _check(lib().sharq_weight_view(d_buf, K, D, E, ctypes.byref(w)), "sharq_weight_view")
    return w


def sharq_weight_view_fmt(d_buf, K, D, E=1, fmt=SHARQ_FMT_NVFP4):
    w = SharqWeight()
    _check(lib().sharq_weight_view_fmt(d_buf, K, D, E, fmt, ctypes.byref(w)), "sharq_weight_view_fmt")
    return w


def sharq_act_view(d_buf, T, K, mode=SHARQ_MODE_SHARQ):
    a = SharqAct()
    _check(lib().sharq_act_view(d_buf, T, K, mode, ctypes.byref(a)), "sharq_act_view")
    return a


def sharq_pack_weight(d_W, w, stream):
    return _check(lib().sharq_pack_weight(d_W, ctypes.byref(w), stream), "sharq_pack_weight")


def sharq_prep(d_X, d_gamma, eps, d_row_index, a, stream):
    return _check(lib().sharq_prep(d_X, d_gamma, eps, d_row_index, ctypes.byref(a), stream), "sharq_prep")


def sharq_prep_noalloc(d_X, d_gamma, eps, d_row_index, a, stream):
    return _check(lib().sharq_prep_noalloc(d_X, d_gamma, eps, d_row_index, ctypes.byref(a), stream),
                  "sharq_prep_noalloc")


def sharq_prep_residual(d_X, d_res, d_res_out, d_gamma, eps, a, stream):
    return _check(lib().sharq_prep_residual(d_X, d_res, d_res_out, d_gamma, eps, ctypes.byref(a), stream),
                  "sharq_prep_residual")


def sharq_prep_silu_mul(d_gate, d_up, d_h, d_gamma, eps, a, stream):
    return _check(lib().sharq_prep_silu_mul(d_gate, d_up, d_h, d_gamma, eps, ctypes.byref(a), stream),
                  "sharq_prep_silu_mul")


def sharq_linear(a, w, d_Y, out_dtype, d_ws, ws_bytes, stream):
    return _check(lib().sharq_linear(ctypes.byref(a), ctypes.byref(w), d_Y, out_dtype, d_ws, ws_bytes, stream),
                  "sharq_linear")


def sharq_prep_linear(d_X, d_gamma, eps, T, a, w, d_Y, out_dtype, d_ws, ws_bytes, stream):
    return _check(lib().sharq_prep_linear(d_X, d_gamma, eps, T, ctypes.byref(a) if a is not None else None,
                                          ctypes.byref(w), d_Y, out_dtype, d_ws, ws_bytes, stream),
                  "sharq_prep_linear")


def sharq_linear_grouped(a, d_offsets, w, d_Y, out_dtype, d_ws, ws_bytes, stream):
    return _check(lib().sharq_linear_grouped(ctypes.byref(a), d_offsets, ctypes.byref(w), d_Y, out_dtype,
                                             d_ws, ws_bytes, stream), "sharq_linear_grouped")


def sharq_check_status(d_ws, stream):
    return lib().sharq_check_status(d_ws, stream)

# ------------------------------------------------- torch conveniences ------


def _torch():
    import torch
    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _buffer(nbytes, device):
    torch = _torch()
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


class PackedWeight:
    """Device buffer + view of a packed weight (sharq_pack_weight).

    W: bf16 CUDA tensor [K, D] (or [E, K, D] for grouped experts); fmt:
    SHARQ_FMT_NVFP4 or SHARQ_FMT_MXFP4 (for the MXFP4 activation modes)."""

    def __init__(self, W, stream=None, fmt=SHARQ_FMT_NVFP4):
        torch = _torch()
        if W.dtype != torch.bfloat16 or not W.is_cuda:
            raise TypeError("W must be a bf16 CUDA tensor")
        W = W.contiguous()
        E, K, D = (1, *W.shape) if W.dim() == 2 else W.shape
        self.K, self.D, self.E, self.fmt = K, D, E, fmt
        nbytes = sharq_weight_bytes_fmt(K, D, E, fmt)
        if nbytes == 0:
            raise SharqError(-2, "sharq_weight_bytes_fmt")
        self.buf = _buffer(nbytes, W.device)
        self.view = sharq_weight_view_fmt(self.buf.data_ptr(), K, D, E, fmt)
        sharq_pack_weight(W.data_ptr(), self.view, _stream_ptr(stream))

    def s_w(self):
        torch = _torch()
        off = self.view.s_w - self.buf.data_ptr()
        return self.buf[off:off + 4 * self.E].view(torch.float32)


class PreparedAct:
    """Device buffer + view of a prepared activation (output of sharq_prep)."""

    def __init__(self, T, K, mode=SHARQ_MODE_SHARQ, device="cuda"):
        nbytes = sharq_act_bytes(T, K, mode)
        if nbytes == 0:
            raise SharqError(-2, "sharq_act_bytes")
        self.T, self.K, self.mode = T, K, mode
        self.buf = _buffer(nbytes, device)
        self.view = sharq_act_view(self.buf.data_ptr(), T, K, mode)
        self.reset()

    def reset(self):
        """Zero the 256-byte scalar block (the prep's sync words, and s_g
        outside the per-token mode), as the C ABI requires before the first
        sharq_prep on a buffer."""
        off = self.view.gmax_bits - 16 - self.buf.data_ptr()
        self.buf[off:off + 256].zero_()

    def prep(self, X, gamma=None, eps=1e-5, row_index=None, stream=None):
        sharq_prep(X.data_ptr() if X is not None else None,
                   gamma.data_ptr() if gamma is not None else None, float(eps),
                   row_index.data_ptr() if row_index is not None else None,
                   self.view, _stream_ptr(stream))
        return self

    def prep_residual(self, X, res, res_out=None, gamma=None, eps=1e-5, stream=None):
        """sharq_prep of h = bf16(X + res); h goes to res_out (which may be
        res itself) when given."""
        sharq_prep_residual(X.data_ptr() if X is not None else None,
                            res.data_ptr() if res is not None else None,
                            res_out.data_ptr() if res_out is not None else None,
                            gamma.data_ptr() if gamma is not None else None, float(eps),
                            self.view, _stream_ptr(stream))
        return self

    def prep_silu_mul(self, gate, up, h_out=None, gamma=None, eps=1e-5, stream=None):
        """sharq_prep of h = bf16(silu(gate) * up); h goes to h_out when given."""
        sharq_prep_silu_mul(gate.data_ptr() if gate is not None else None,
                            up.data_ptr() if up is not None else None,
                            h_out.data_ptr() if h_out is not None else None,
                            gamma.data_ptr() if gamma is not None else None, float(eps),
                            self.view, _stream_ptr(stream))
        return self

    def region(self, name, nbytes):
        """uint8 tensor aliasing one field of the view (for inspection)."""
        off = getattr(self.view, name) - self.buf.data_ptr()
        return self.buf[off:off + nbytes]


class Workspace:
    """Zero-initialised workspace for sharq_linear (error word + scratch)."""

    def __init__(self, T, K, D, E=1, device="cuda"):
        self.nbytes = sharq_workspace_bytes(T, K, D, E)
        if self.nbytes == 0:
            raise SharqError(-2, "sharq_workspace_bytes")
        self.buf = _torch().zeros(self.nbytes, dtype=_torch().uint8, device=device)

    def check(self, stream=None):
        return sharq_check_status(self.buf.data_ptr(), _stream_ptr(stream))


def linear(act, weight, out_dtype=None, out=None, ws=None, group_offsets=None, stream=None):
    """Y = SharQ(X) W through sharq_linear (or sharq_linear_grouped when
    group_offsets, a device int32 tensor [E+1], is given)."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    code = SHARQ_OUT_F32 if out_dtype == torch.float32 else SHARQ_OUT_BF16
    if out is None:
        out = torch.empty((act.T, weight.D), dtype=out_dtype, device=act.buf.device)
    if ws is None:
        ws = Workspace(act.T, act.K, weight.D, weight.E, device=act.buf.device)
    s = _stream_ptr(stream)
    if group_offsets is None:
        sharq_linear(act.view, weight.view, out.data_ptr(), code, ws.buf.data_ptr(), ws.nbytes, s)
    else:
        sharq_linear_grouped(act.view, group_offsets.data_ptr(), weight.view, out.data_ptr(), code,
                             ws.buf.data_ptr(), ws.nbytes, s)
    return out


def prep_linear(X, gamma, eps, weight, act=None, out_dtype=None, out=None, ws=None, stream=None):
    """Y = SharQ(X) W in one call (sharq_prep_linear): a single fused kernel for
    T <= 32 rows, prep into `act` + linear above that."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    code = SHARQ_OUT_F32 if out_dtype == torch.float32 else SHARQ_OUT_BF16
    T, K = X.shape
    if out is None:
        out = torch.empty((T, weight.D), dtype=out_dtype, device=X.device)
    if ws is None:
        ws = Workspace(T, K, weight.D, 1, device=X.device)
    if act is None and T > 32:
        act = PreparedAct(T, K, device=X.device)
    sharq_prep_linear(X.data_ptr(), gamma.data_ptr() if gamma is not None else None, float(eps), T,
                      act.view if act is not None else None, weight.view, out.data_ptr(), code,
                      ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream))
    return out

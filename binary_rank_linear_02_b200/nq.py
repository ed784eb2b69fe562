"""ctypes binding of libnq (include/nq.h): argument marshalling only.

Every step of the factorised linear runs in the CUDA library; this module turns torch
tensors / numpy arrays into the plain pointers, sizes and stream handle of the C ABI and
raises ``NQError`` on a non-zero status.  There is no fallback: if ``libnq.so`` is
missing or cannot be loaded, importing this module raises.

Same names as the C entry points: ``nq_pack_signs``, ``nq_unpack_signs``,
``nq_lowrank_linear_fwd``, ``nq_bits_per_weight``, ``nq_status_string``,
``nq_workspace_reserve``, ``nq_cast_f32_to_bf16``, ``nq_rms_normalize_bf16``; plus
tensor-level conveniences ``pack_signs``, ``unpack_signs``, ``lowrank_linear_fwd``,
``lowrank_linear_fwd_grouped``, ``cast_f32_to_bf16`` and ``rms_normalize_bf16``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnq.so")

NQ_OK = 0
NQ_ERR_NULL = -1
NQ_ERR_SHAPE = -2
NQ_ERR_ALIGN = -3
NQ_ERR_BATCH = -4
NQ_ERR_VALUE = -5
NQ_ERR_CUDA = -6
NQ_ERR_TIMEOUT = -7
NQ_ERR_NOMEM = -8
NQ_ERR_PTRKIND = -9
NQ_ERR_NOALLOC_LIMIT = -10
NQ_DECODE_MAX_BATCH = 8
NQ_NOALLOC_MAX_RANK = 4096


class nq_linear_desc(ctypes.Structure):
    """One layer of nq_lowrank_linear_fwd_grouped (see include/nq.h)."""

    _fields_ = [("x", ctypes.c_void_p), ("Upk", ctypes.c_void_p), ("Vpk", ctypes.c_void_p),
                ("s1", ctypes.c_void_p), ("s2", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("m", ctypes.c_int64), ("n", ctypes.c_int64), ("r", ctypes.c_int64)]


class nq_linear_desc_ex(ctypes.Structure):
    """One layer of nq_lowrank_linear_fwd_grouped_ex: the layer plus optional bf16 outputs."""

    _fields_ = [("base", nq_linear_desc), ("y_bf16", ctypes.c_void_p), ("y_rmsnorm_bf16", ctypes.c_void_p)]


class NQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {nq_status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m binary_rank_linear_02_b200.build` "
            "(this package has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    p, i64 = ctypes.c_void_p, ctypes.c_int64
    L.nq_pack_signs.argtypes = [p, i64, i64, p, p]
    L.nq_pack_signs.restype = ctypes.c_int
    L.nq_unpack_signs.argtypes = [p, i64, i64, p, p]
    L.nq_transpose_signs.argtypes = [p, i64, i64, p, p]
    L.nq_lowrank_linear_bwd_input.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, p]
    L.nq_lowrank_linear_bwd_scales.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, p]
    L.nq_lowrank_linear_bwd_factors.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, p, p]
    L.nq_unpack_signs.restype = ctypes.c_int
    L.nq_lowrank_linear_fwd.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, p]
    L.nq_lowrank_linear_fwd.restype = ctypes.c_int
    L.nq_bits_per_weight.argtypes = [i64, i64, i64]
    L.nq_bits_per_weight.restype = ctypes.c_double
    L.nq_status_string.argtypes = [ctypes.c_int]
    L.nq_status_string.restype = ctypes.c_char_p
    L.nq_workspace_reserve.argtypes = [i64, i64, i64, i64]
    L.nq_workspace_reserve.restype = ctypes.c_int
    L.nq_version.restype = ctypes.c_int
    L.nq_lowrank_linear_fwd_noalloc.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, p]
    L.nq_lowrank_linear_fwd_noalloc.restype = ctypes.c_int
    L.nq_lowrank_linear_fwd_grouped.argtypes = [p, ctypes.c_int, i64, p]
    L.nq_lowrank_linear_fwd_grouped.restype = ctypes.c_int
    L.nq_lowrank_linear_fwd_grouped_ex.argtypes = [p, ctypes.c_int, i64, p]
    L.nq_lowrank_linear_fwd_grouped_ex.restype = ctypes.c_int
    L.nq_device_status.argtypes = [p]
    L.nq_device_status.restype = ctypes.c_int
    L.nq_selftest_wait_timeout.argtypes = [i64, p]
    L.nq_selftest_wait_timeout.restype = ctypes.c_int
    L.nq_cast_f32_to_bf16.argtypes = [p, i64, p, p]
    L.nq_cast_f32_to_bf16.restype = ctypes.c_int
    L.nq_rms_normalize_bf16.argtypes = [p, i64, i64, p, p]
    L.nq_rms_normalize_bf16.restype = ctypes.c_int
    L.nq_lowrank_linear_fwd_envelope.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, p, p]
    L.nq_lowrank_linear_fwd_envelope.restype = ctypes.c_int
    L.nq_bits_per_weight_envelope.argtypes = [i64, i64, i64, i64]
    L.nq_bits_per_weight_envelope.restype = ctypes.c_double
    i32, f64 = ctypes.c_int, ctypes.c_double
    L.nq_admm_init.argtypes = [p, i64, i64, i64, p, i32, p, p, p, p, p, p, p, p, p]
    L.nq_admm_init.restype = ctypes.c_int
    L.nq_admm_iterate.argtypes = [p, i64, i64, i64, p, p, p, p, p, p, p, p, i32, f64, f64, p]
    L.nq_admm_iterate.restype = ctypes.c_int
    L.nq_admm_factorize.argtypes = [p, i64, i64, i64, p, i32, i32, f64, f64, p, p, p, p, p, p]
    L.nq_admm_factorize.restype = ctypes.c_int
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


# ------------------------------------------------------------------ raw C names

def nq_pack_signs(signs_ptr: int, rows: int, cols: int, out_ptr: int, stream: int = 0) -> int:
    return _lib.nq_pack_signs(signs_ptr, rows, cols, out_ptr, stream)


def nq_unpack_signs(packed_ptr: int, rows: int, cols: int, out_ptr: int, stream: int = 0) -> int:
    return _lib.nq_unpack_signs(packed_ptr, rows, cols, out_ptr, stream)


def nq_transpose_signs(packed_ptr: int, rows: int, cols: int, out_ptr: int, stream: int = 0) -> int:
    return _lib.nq_transpose_signs(packed_ptr, rows, cols, out_ptr, stream)


def nq_lowrank_linear_bwd_input(dy_ptr, UpkT_ptr, VpkT_ptr, s1_ptr, s2_ptr, m, n, r, batch, dx_ptr, stream=0) -> int:
    return _lib.nq_lowrank_linear_bwd_input(dy_ptr, UpkT_ptr, VpkT_ptr, s1_ptr, s2_ptr, m, n, r, batch, dx_ptr, stream)


def nq_lowrank_linear_bwd_scales(x_ptr, dy_ptr, Upk_ptr, Vpk_ptr, UpkT_ptr, VpkT_ptr, s1_ptr, s2_ptr, m, n, r, batch,
                                 ds1_ptr, ds2_ptr, stream=0) -> int:
    return _lib.nq_lowrank_linear_bwd_scales(x_ptr, dy_ptr, Upk_ptr, Vpk_ptr, UpkT_ptr, VpkT_ptr, s1_ptr, s2_ptr, m, n,
                                             r, batch, ds1_ptr, ds2_ptr, stream)


def nq_lowrank_linear_bwd_factors(x_ptr, dy_ptr, Vpk_ptr, UpkT_ptr, s1_ptr, s2_ptr, m, n, r, batch, dU_ptr, dV_ptr,
                                  stream=0) -> int:
    return _lib.nq_lowrank_linear_bwd_factors(x_ptr, dy_ptr, Vpk_ptr, UpkT_ptr, s1_ptr, s2_ptr, m, n, r, batch, dU_ptr,
                                              dV_ptr, stream)


def nq_lowrank_linear_fwd(x_ptr, Upk_ptr, Vpk_ptr, s1_ptr, s2_ptr, m, n, r, batch, y_ptr, stream=0) -> int:
    return _lib.nq_lowrank_linear_fwd(x_ptr, Upk_ptr, Vpk_ptr, s1_ptr, s2_ptr, m, n, r, batch, y_ptr, stream)


def nq_lowrank_linear_fwd_noalloc(x_ptr, Upk_ptr, Vpk_ptr, s1_ptr, s2_ptr, m, n, r, batch, y_ptr, stream=0) -> int:
    return _lib.nq_lowrank_linear_fwd_noalloc(x_ptr, Upk_ptr, Vpk_ptr, s1_ptr, s2_ptr, m, n, r, batch, y_ptr, stream)


def nq_lowrank_linear_fwd_grouped(descs_ptr, count, batch, stream=0) -> int:
    return _lib.nq_lowrank_linear_fwd_grouped(descs_ptr, count, batch, stream)


def nq_lowrank_linear_fwd_grouped_ex(descs_ptr, count, batch, stream=0) -> int:
    return _lib.nq_lowrank_linear_fwd_grouped_ex(descs_ptr, count, batch, stream)


def nq_bits_per_weight(m: int, n: int, r: int) -> float:
    return _lib.nq_bits_per_weight(m, n, r)


def nq_cast_f32_to_bf16(src_ptr, count, dst_ptr, stream=0) -> int:
    return _lib.nq_cast_f32_to_bf16(src_ptr, count, dst_ptr, stream)


def nq_rms_normalize_bf16(src_ptr, rows, cols, dst_ptr, stream=0) -> int:
    return _lib.nq_rms_normalize_bf16(src_ptr, rows, cols, dst_ptr, stream)


def nq_status_string(status: int) -> str:
    return _lib.nq_status_string(status).decode()


def nq_workspace_reserve(m: int, n: int, r: int, batch: int) -> int:
    return _lib.nq_workspace_reserve(m, n, r, batch)


def nq_device_status(stream: int = 0) -> int:
    return _lib.nq_device_status(stream)


def device_status(stream=None) -> None:
    """Synchronise and raise NQError if a kernel recorded a timed-out device wait."""
    import torch

    h = int(stream) if stream is not None else torch.cuda.current_stream().cuda_stream
    _check(_lib.nq_device_status(h), "nq_device_status")


def nq_selftest_wait_timeout(limit_ns: int, stream: int = 0) -> int:
    return _lib.nq_selftest_wait_timeout(limit_ns, stream)


def nq_version() -> int:
    return _lib.nq_version()


# ------------------------------------------------------------------ tensor conveniences

def _ptr(a) -> int:
    if a is None:
        return 0
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"], "array must be C-contiguous"
        return a.ctypes.data
    assert a.is_contiguous(), "tensor must be contiguous"
    return a.data_ptr()


def _stream(stream, *tensors) -> int:
    if stream is not None:
        return int(stream)
    import torch

    for t in tensors:
        if isinstance(t, torch.Tensor) and t.is_cuda:
            return torch.cuda.current_stream(t.device).cuda_stream
    return 0


def _check(status: int, where: str) -> None:
    if status != NQ_OK:
        raise NQError(status, where)


def pack_signs(signs, out=None, stream=None):
    """rows x cols int8 signs (torch tensor or numpy array) -> rows x ceil(cols/32) words."""
    rows, cols = signs.shape
    wpr = (cols + 31) // 32
    if out is None:
        if isinstance(signs, np.ndarray):
            out = np.empty((rows, wpr), dtype=np.uint32)
        else:
            import torch

            out = torch.empty((rows, wpr), dtype=torch.int32, device=signs.device)
    _check(_lib.nq_pack_signs(_ptr(signs), rows, cols, _ptr(out), _stream(stream, signs)), "nq_pack_signs")
    return out


def unpack_signs(packed, cols: int, out=None, stream=None):
    rows = packed.shape[0]
    if out is None:
        if isinstance(packed, np.ndarray):
            out = np.empty((rows, cols), dtype=np.int8)
        else:
            import torch

            out = torch.empty((rows, cols), dtype=torch.int8, device=packed.device)
    _check(_lib.nq_unpack_signs(_ptr(packed), rows, cols, _ptr(out), _stream(stream, packed)), "nq_unpack_signs")
    return out


def transpose_signs(packed, rows: int, cols: int, out=None, stream=None):
    """rows x ceil(cols/32) packed words -> cols x ceil(rows/32) words of the transpose."""
    wpr_out = (rows + 31) // 32
    if out is None:
        if isinstance(packed, np.ndarray):
            out = np.empty((cols, wpr_out), dtype=np.uint32)
        else:
            import torch

            out = torch.empty((cols, wpr_out), dtype=torch.int32, device=packed.device)
    _check(_lib.nq_transpose_signs(_ptr(packed), rows, cols, _ptr(out), _stream(stream, packed)),
           "nq_transpose_signs")
    return out


def lowrank_linear_bwd_input(dy, UpkT, VpkT, s1, s2, m: int, n: int, r: int, dx=None, stream=None):
    """dx (batch x n, float32) = s2 * (V (U^T (s1 * dy))), the gradient of the layer's
    output with respect to its input.

    dy: batch x m bfloat16 (device or host); UpkT: r x m/32 = transpose_signs(Upk, m, r) and
    VpkT: n x r/32 = transpose_signs(Vpk, r, n) (device); s1: m and s2: n fp16 (device).
    """
    batch = dy.shape[0] if dy.dim() == 2 else 1
    if dx is None:
        import torch

        dx = torch.empty((batch, n), dtype=torch.float32, device=dy.device,
                         pin_memory=(not dy.is_cuda and torch.cuda.is_available()))
    st = _lib.nq_lowrank_linear_bwd_input(_ptr(dy), _ptr(UpkT), _ptr(VpkT), _ptr(s1), _ptr(s2), m, n, r, batch,
                                          _ptr(dx), _stream(stream, dy, UpkT, dx))
    _check(st, "nq_lowrank_linear_bwd_input")
    return dx


def lowrank_linear_bwd_scales(x, dy, Upk, Vpk, UpkT, VpkT, s1, s2, m: int, n: int, r: int, stream=None):
    """(ds1 (m,), ds2 (n,)) float32 device tensors: the gradients with respect to s1 and s2
    for input x (batch x n bf16) and output gradient dy (batch x m bf16), all on the device."""
    import torch

    batch = x.shape[0] if x.dim() == 2 else 1
    ds1 = torch.empty((m,), dtype=torch.float32, device=x.device)
    ds2 = torch.empty((n,), dtype=torch.float32, device=x.device)
    st = _lib.nq_lowrank_linear_bwd_scales(_ptr(x), _ptr(dy), _ptr(Upk), _ptr(Vpk), _ptr(UpkT), _ptr(VpkT), _ptr(s1),
                                           _ptr(s2), m, n, r, batch, _ptr(ds1), _ptr(ds2), _stream(stream, x, dy))
    _check(st, "nq_lowrank_linear_bwd_scales")
    return ds1, ds2


def lowrank_linear_bwd_factors(x, dy, Vpk, UpkT, s1, s2, m: int, n: int, r: int, stream=None):
    """(dU (m x r), dV (n x r)) float32 device tensors: the straight-through gradients of the
    factors for input x (batch x n bf16) and output gradient dy (batch x m bf16)."""
    import torch

    batch = x.shape[0] if x.dim() == 2 else 1
    dU = torch.empty((m, r), dtype=torch.float32, device=x.device)
    dV = torch.empty((n, r), dtype=torch.float32, device=x.device)
    st = _lib.nq_lowrank_linear_bwd_factors(_ptr(x), _ptr(dy), _ptr(Vpk), _ptr(UpkT), _ptr(s1), _ptr(s2), m, n, r, batch,
                                            _ptr(dU), _ptr(dV), _stream(stream, x, dy))
    _check(st, "nq_lowrank_linear_bwd_factors")
    return dU, dV


def lowrank_linear_fwd(x, Upk, Vpk, s1, s2, m: int, n: int, r: int, y=None, stream=None):
    """y (batch x m, float32) = s1 * (U (V^T (s2 * x))).

    x: batch x n bfloat16 (device or host); Upk: m x r/32 and Vpk: r x n/32 packed words
    (device); s1: m and s2: n fp16 (device).  y defaults to a new float32 tensor on x's
    device.
    """
    batch = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        import torch

        y = torch.empty((batch, m), dtype=torch.float32, device=x.device,
                        pin_memory=(not x.is_cuda and torch.cuda.is_available()))
    st = _lib.nq_lowrank_linear_fwd(_ptr(x), _ptr(Upk), _ptr(Vpk), _ptr(s1), _ptr(s2), m, n, r, batch,
                                    _ptr(y), _stream(stream, x, Upk, y))
    _check(st, "nq_lowrank_linear_fwd")
    return y


def make_descs(layers):
    """ctypes array of nq_linear_desc from (x, Upk, Vpk, s1, s2, y, m, n, r) tuples."""
    arr = (nq_linear_desc * len(layers))()
    for i, (x, Upk, Vpk, s1, s2, y, m, n, r) in enumerate(layers):
        arr[i] = nq_linear_desc(_ptr(x), _ptr(Upk), _ptr(Vpk), _ptr(s1), _ptr(s2), _ptr(y), m, n, r)
    return arr


def make_descs_ex(layers):
    """ctypes array of nq_linear_desc_ex from (x, Upk, Vpk, s1, s2, y, m, n, r, y_bf16, y_norm)
    tuples; the last two may be None."""
    arr = (nq_linear_desc_ex * len(layers))()
    for i, (x, Upk, Vpk, s1, s2, y, m, n, r, yb, yn) in enumerate(layers):
        arr[i] = nq_linear_desc_ex(nq_linear_desc(_ptr(x), _ptr(Upk), _ptr(Vpk), _ptr(s1), _ptr(s2), _ptr(y), m, n, r),
                                   _ptr(yb), _ptr(yn))
    return arr


def lowrank_linear_fwd_grouped_ex(layers, batch: int, stream=None):
    """Grouped forward with optional bf16 outputs: layers are (x, Upk, Vpk, s1, s2, y, m, n, r,
    y_bf16 or None, y_rmsnorm_bf16 or None)."""
    arr = make_descs_ex(layers)
    h = _stream(stream, *(l[0] for l in layers))
    _check(_lib.nq_lowrank_linear_fwd_grouped_ex(ctypes.addressof(arr), len(layers), batch, h),
           "nq_lowrank_linear_fwd_grouped_ex")


def lowrank_linear_fwd_grouped(layers, batch: int, stream=None):
    """Run independent layers [(x, Upk, Vpk, s1, s2, y, m, n, r), ...] in one grouped call."""
    arr = make_descs(layers)
    h = _stream(stream, *(l[0] for l in layers))
    _check(_lib.nq_lowrank_linear_fwd_grouped(ctypes.addressof(arr), len(layers), batch, h),
           "nq_lowrank_linear_fwd_grouped")


def cast_f32_to_bf16(src, dst=None, stream=None):
    """bf16 bit patterns (int16 tensor of src's shape) of a float32 device tensor."""
    import torch

    if dst is None:
        dst = torch.empty(src.shape, dtype=torch.int16, device=src.device)
    _check(_lib.nq_cast_f32_to_bf16(_ptr(src), src.numel(), _ptr(dst), _stream(stream, src)), "nq_cast_f32_to_bf16")
    return dst


def rms_normalize_bf16(src, dst=None, stream=None):
    """Row-wise bf16(src / rms(src)) of a 2-D float32 device tensor (int16 patterns)."""
    import torch

    rows, cols = src.shape
    if dst is None:
        dst = torch.empty((rows, cols), dtype=torch.int16, device=src.device)
    _check(_lib.nq_rms_normalize_bf16(_ptr(src), rows, cols, _ptr(dst), _stream(stream, src)),
           "nq_rms_normalize_bf16")
    return dst


def bits_per_weight(m: int, n: int, r: int) -> float:
    return _lib.nq_bits_per_weight(m, n, r)


def workspace_reserve(m: int, n: int, r: int, batch: int) -> None:
    _check(_lib.nq_workspace_reserve(m, n, r, batch), "nq_workspace_reserve")


# ------------------------------------------------------------------ LB-ADMM initialiser

class AdmmState:
    """Device state of the ADMM iteration: latent A (m x r), B (n x r), projections Z_A, Z_B,
    duals L_A, L_B, row scales s_A (m), s_B (n), all fp32 tensors on the current device."""

    def __init__(self, m: int, n: int, r: int, device=None):
        import torch

        dev = device if device is not None else torch.device("cuda")
        f = dict(dtype=torch.float32, device=dev)
        self.m, self.n, self.r = m, n, r
        self.A, self.ZA, self.LA = (torch.empty((m, r), **f) for _ in range(3))
        self.B, self.ZB, self.LB = (torch.empty((n, r), **f) for _ in range(3))
        self.sA, self.sB = torch.empty(m, **f), torch.empty(n, **f)

    def ptrs(self):
        return [_ptr(t) for t in (self.A, self.B, self.ZA, self.ZB, self.LA, self.LB, self.sA, self.sB)]


def admm_init(W, m: int, n: int, r: int, Omega, power_iters: int = 1, stream=None) -> AdmmState:
    """Start of the initialiser on W (m x n bfloat16 bits, int16/bfloat16 tensor) from Omega (n x r fp32)."""
    st = AdmmState(m, n, r, W.device)
    _check(_lib.nq_admm_init(_ptr(W), m, n, r, _ptr(Omega), power_iters, *st.ptrs(), _stream(stream, W)),
           "nq_admm_init")
    return st


def admm_iterate(W, st: AdmmState, iters: int, lam0: float = 0.2, growth: float = 1.05, stream=None) -> AdmmState:
    _check(_lib.nq_admm_iterate(_ptr(W), st.m, st.n, st.r, *st.ptrs(), iters, lam0, growth, _stream(stream, W)),
           "nq_admm_iterate")
    return st


def admm_factorize(W, m: int, n: int, r: int, Omega, iters: int = 40, lam0: float = 0.2, growth: float = 1.05,
                   power_iters: int = 1, stream=None):
    """The whole initialiser: returns (Upk, Vpk, s1, s2, rel_err) with the forward pass's
    packings (Upk m x r/32, Vpk r x n/32 int32 views of the words; s1, s2 fp16 bits as int16)."""
    import torch

    dev = W.device
    Upk = torch.empty((m, r // 32), dtype=torch.int32, device=dev)
    Vpk = torch.empty((r, n // 32), dtype=torch.int32, device=dev)
    s1 = torch.empty(m, dtype=torch.int16, device=dev)
    s2 = torch.empty(n, dtype=torch.int16, device=dev)
    err = ctypes.c_double(0.0)
    _check(_lib.nq_admm_factorize(_ptr(W), m, n, r, _ptr(Omega), power_iters, iters, lam0, growth, _ptr(Upk),
                                  _ptr(Vpk), _ptr(s1), _ptr(s2), ctypes.byref(err), _stream(stream, W)),
           "nq_admm_factorize")
    return Upk, Vpk, s1, s2, err.value


# ------------------------------------------------------------------ rank-l envelope variant

def lowrank_linear_fwd_envelope(x, Upk, Vpk, a, b, m: int, n: int, r: int, y=None, stream=None):
    """y = sum_q a_q * (U (V^T (b_q * x))): a is l x m fp16 bits, b is l x n (device tensors)."""
    import torch

    batch = x.shape[0]
    l = a.shape[0]
    if y is None:
        y = torch.empty((batch, m), dtype=torch.float32, device=x.device)
    st = _lib.nq_lowrank_linear_fwd_envelope(_ptr(x), _ptr(Upk), _ptr(Vpk), _ptr(a), _ptr(b), l, m, n, r, batch,
                                             _ptr(y), _stream(stream, x, y))
    _check(st, "nq_lowrank_linear_fwd_envelope")
    return y


def bits_per_weight_envelope(m: int, n: int, r: int, l: int) -> float:
    return _lib.nq_bits_per_weight_envelope(m, n, r, l)


"""CPU fp64 oracle for the low-rank binary factorised linear (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``binary_rank_linear_02_b200``) never does, and
the oracle imports nothing from it: the two share no code.  The arithmetic lives in
``nq_oracle.c`` (plain C, fp64); this module only compiles it with gcc and marshals
numpy arrays through ctypes.

Definition followed (hardwired.dev, section "Jak NanoQuant funguje"; rapidrecap.app,
section "Quantization Technique"): W = diag(s1) U V^T diag(s2) with +1/-1 factors,
y = s1 * (U (V^T (s2 * x))).  See the header of ``nq_oracle.c`` for the storage format
and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ORC_OK = 0
ORC_ERR_ARG = -1
ORC_ERR_VALUE = -5


def build(force: bool = False) -> str:
    """Compile ``nq_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load(path: str) -> ctypes.CDLL:
    L = ctypes.CDLL(path)
    i64, p = ctypes.c_int64, ctypes.c_void_p
    L.orc_pack_signs.argtypes = [p, i64, i64, p]
    L.orc_unpack_signs.argtypes = [p, i64, i64, p]
    L.orc_lowrank_linear_fwd.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p]
    L.orc_stage1.argtypes = [p, p, p, i64, i64, i64, p]
    L.orc_lowrank_linear_bwd_input.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p]
    L.orc_transpose_signs.argtypes = [p, i64, i64, p]
    L.orc_lowrank_linear_bwd_scales.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, p]
    L.orc_lowrank_linear_bwd_factors.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, p]
    L.orc_lowrank_linear_fwd_envelope.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, p]
    L.orc_bits_per_weight_envelope.argtypes = [i64, i64, i64, i64]
    L.orc_bits_per_weight_envelope.restype = ctypes.c_double
    L.orc_bits_per_weight.argtypes = [i64, i64, i64]
    L.orc_bits_per_weight.restype = ctypes.c_double
    L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_double.restype = ctypes.c_double
    L.orc_f16_to_double.argtypes = [ctypes.c_uint16]
    L.orc_f16_to_double.restype = ctypes.c_double
    L.orc_num_threads.restype = ctypes.c_int
    L.orc_round_to_bf16.argtypes = [ctypes.c_double]
    L.orc_round_to_bf16.restype = ctypes.c_uint16
    L.orc_round_array_bf16.argtypes = [p, i64, p]
    L.orc_rms_normalize_bf16.argtypes = [p, i64, i64, p]
    return L


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def words_per_row(cols: int) -> int:
    return (cols + 31) // 32


class Oracle:
    """The oracle's entry points over one compiled copy of ``nq_oracle.c``."""

    def __init__(self, lib_path: str):
        self.lib = _load(lib_path)

    def pack_signs(self, signs: np.ndarray) -> np.ndarray:
        """rows x cols int8 signs -> rows x ceil(cols/32) uint32 (bit 1 = +1, LSB first)."""
        s = np.ascontiguousarray(signs, dtype=np.int8)
        rows, cols = s.shape
        out = np.zeros((rows, words_per_row(cols)), dtype=np.uint32)
        st = self.lib.orc_pack_signs(_ptr(s), rows, cols, _ptr(out))
        if st != ORC_OK:
            raise ValueError(f"orc_pack_signs failed with status {st}")
        return out

    def unpack_signs(self, packed: np.ndarray, cols: int) -> np.ndarray:
        p = np.ascontiguousarray(packed, dtype=np.uint32)
        rows = p.shape[0]
        assert p.shape[1] == words_per_row(cols)
        out = np.zeros((rows, cols), dtype=np.int8)
        st = self.lib.orc_unpack_signs(_ptr(p), rows, cols, _ptr(out))
        if st != ORC_OK:
            raise ValueError(f"orc_unpack_signs failed with status {st}")
        return out

    def lowrank_linear_bwd_input(self, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r) -> np.ndarray:
        """dx (batch x n, float64) = s2 * (V (U^T (s1 * dy))): the gradient of the layer's
        output with respect to its input, for the same packings as the forward pass.

        dy_bits: batch x m uint16 bfloat16 patterns; the other arguments as in
        ``lowrank_linear_fwd``.
        """
        dy = np.ascontiguousarray(dy_bits, dtype=np.uint16).reshape(-1, m)
        batch = dy.shape[0]
        U = np.ascontiguousarray(Upk, dtype=np.uint32)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        a = np.ascontiguousarray(s1_bits, dtype=np.uint16)
        b = np.ascontiguousarray(s2_bits, dtype=np.uint16)
        assert U.shape == (m, words_per_row(r)) and V.shape == (r, words_per_row(n))
        assert a.shape == (m,) and b.shape == (n,)
        dx = np.zeros((batch, n), dtype=np.float64)
        if batch == 0:
            return dx
        st = self.lib.orc_lowrank_linear_bwd_input(
            _ptr(dy), _ptr(U), _ptr(V), _ptr(a), _ptr(b), m, n, r, batch, _ptr(dx))
        if st != ORC_OK:
            raise ValueError(f"orc_lowrank_linear_bwd_input failed with status {st}")
        return dx

    def lowrank_linear_bwd_scales(self, x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
        """(ds1 (m,), ds2 (n,)) float64: the gradients with respect to the scale vectors for
        input x (batch x n bf16 patterns) and output gradient dy (batch x m bf16 patterns)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
        dy = np.ascontiguousarray(dy_bits, dtype=np.uint16).reshape(-1, m)
        assert x.shape[0] == dy.shape[0]
        U = np.ascontiguousarray(Upk, dtype=np.uint32)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        a = np.ascontiguousarray(s1_bits, dtype=np.uint16)
        b = np.ascontiguousarray(s2_bits, dtype=np.uint16)
        assert U.shape == (m, words_per_row(r)) and V.shape == (r, words_per_row(n))
        ds1 = np.zeros(m, dtype=np.float64)
        ds2 = np.zeros(n, dtype=np.float64)
        st = self.lib.orc_lowrank_linear_bwd_scales(
            _ptr(x), _ptr(dy), _ptr(U), _ptr(V), _ptr(a), _ptr(b), m, n, r, x.shape[0], _ptr(ds1), _ptr(ds2))
        if st != ORC_OK:
            raise ValueError(f"orc_lowrank_linear_bwd_scales failed with status {st}")
        return ds1, ds2

    def lowrank_linear_bwd_factors(self, x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
        """(dU (m x r), dV (n x r)) float64: the straight-through gradients of the factors,
        dU = diag(s1) dy^T t and dV = diag(s2) x^T u with t = V^T (s2 * x), u = U^T (s1 * dy)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
        dy = np.ascontiguousarray(dy_bits, dtype=np.uint16).reshape(-1, m)
        assert x.shape[0] == dy.shape[0]
        U = np.ascontiguousarray(Upk, dtype=np.uint32)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        a = np.ascontiguousarray(s1_bits, dtype=np.uint16)
        b = np.ascontiguousarray(s2_bits, dtype=np.uint16)
        assert U.shape == (m, words_per_row(r)) and V.shape == (r, words_per_row(n))
        dU = np.zeros((m, r), dtype=np.float64)
        dV = np.zeros((n, r), dtype=np.float64)
        st = self.lib.orc_lowrank_linear_bwd_factors(
            _ptr(x), _ptr(dy), _ptr(U), _ptr(V), _ptr(a), _ptr(b), m, n, r, x.shape[0], _ptr(dU), _ptr(dV))
        if st != ORC_OK:
            raise ValueError(f"orc_lowrank_linear_bwd_factors failed with status {st}")
        return dU, dV

    def transpose_signs(self, packed: np.ndarray, rows: int, cols: int) -> np.ndarray:
        """rows x ceil(cols/32) packed words -> cols x ceil(rows/32) words of the transpose."""
        p = np.ascontiguousarray(packed, dtype=np.uint32)
        assert p.shape == (rows, words_per_row(cols))
        out = np.zeros((cols, words_per_row(rows)), dtype=np.uint32)
        st = self.lib.orc_transpose_signs(_ptr(p), rows, cols, _ptr(out))
        if st != ORC_OK:
            raise ValueError(f"orc_transpose_signs failed with status {st}")
        return out

    def lowrank_linear_fwd(self, x_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r) -> np.ndarray:
        """y (batch x m, float64) = s1 * (U (V^T (s2 * x))).

        x_bits: batch x n uint16 bfloat16 patterns; s1_bits/s2_bits: uint16 fp16 patterns;
        Upk: m x ceil(r/32) uint32; Vpk: r x ceil(n/32) uint32.
        """
        x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
        batch = x.shape[0]
        U = np.ascontiguousarray(Upk, dtype=np.uint32)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        a = np.ascontiguousarray(s1_bits, dtype=np.uint16)
        b = np.ascontiguousarray(s2_bits, dtype=np.uint16)
        assert U.shape == (m, words_per_row(r)) and V.shape == (r, words_per_row(n))
        assert a.shape == (m,) and b.shape == (n,)
        y = np.zeros((batch, m), dtype=np.float64)
        if batch == 0:
            return y
        st = self.lib.orc_lowrank_linear_fwd(
            _ptr(x), _ptr(U), _ptr(V), _ptr(a), _ptr(b), m, n, r, batch, _ptr(y))
        if st != ORC_OK:
            raise ValueError(f"orc_lowrank_linear_fwd failed with status {st}")
        return y

    def lowrank_linear_fwd_envelope(self, x_bits, Upk, Vpk, a_bits, b_bits, m, n, r) -> np.ndarray:
        """y (batch x m, float64) = sum_q a_q * (U (V^T (b_q * x))): the rank-l envelope
        variant.  a_bits: l x m, b_bits: l x n uint16 fp16 patterns (l = 1 is the forward)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
        batch = x.shape[0]
        a = np.ascontiguousarray(a_bits, dtype=np.uint16).reshape(-1, m)
        b = np.ascontiguousarray(b_bits, dtype=np.uint16).reshape(-1, n)
        l = a.shape[0]
        assert b.shape == (l, n) and l >= 1
        U = np.ascontiguousarray(Upk, dtype=np.uint32)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        assert U.shape == (m, words_per_row(r)) and V.shape == (r, words_per_row(n))
        y = np.zeros((batch, m), dtype=np.float64)
        if batch == 0:
            return y
        st = self.lib.orc_lowrank_linear_fwd_envelope(_ptr(x), _ptr(U), _ptr(V), _ptr(a), _ptr(b), l, m, n, r,
                                                      batch, _ptr(y))
        if st != ORC_OK:
            raise ValueError(f"orc_lowrank_linear_fwd_envelope: status {st}")
        return y

    def bits_per_weight_envelope(self, m: int, n: int, r: int, l: int) -> float:
        return self.lib.orc_bits_per_weight_envelope(m, n, r, l)

    def stage1(self, x_bits, Vpk, s2_bits, n, r) -> np.ndarray:
        """t (batch x r, float64) = V^T (s2 * x)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
        V = np.ascontiguousarray(Vpk, dtype=np.uint32)
        b = np.ascontiguousarray(s2_bits, dtype=np.uint16)
        t = np.zeros((x.shape[0], r), dtype=np.float64)
        st = self.lib.orc_stage1(_ptr(x), _ptr(V), _ptr(b), n, r, x.shape[0], _ptr(t))
        if st != ORC_OK:
            raise ValueError(f"orc_stage1 failed with status {st}")
        return t

    def bits_per_weight(self, m: int, n: int, r: int) -> float:
        return self.lib.orc_bits_per_weight(m, n, r)

    def bf16_to_double(self, bits: int) -> float:
        return self.lib.orc_bf16_to_double(bits)

    def f16_to_double(self, bits: int) -> float:
        return self.lib.orc_f16_to_double(bits)

    def num_threads(self) -> int:
        return self.lib.orc_num_threads()

    # ---------------------------------------------------------------- decode chain

    def round_to_bf16(self, v) -> np.ndarray:
        """Nearest bfloat16 bit patterns (ties to even) of an array of doubles."""
        a = np.ascontiguousarray(v, dtype=np.float64)
        out = np.zeros(a.shape, dtype=np.uint16)
        st = self.lib.orc_round_array_bf16(_ptr(a), a.size, _ptr(out))
        if st != ORC_OK:
            raise ValueError(f"orc_round_array_bf16 failed with status {st}")
        return out

    def rms_normalize_bf16(self, y) -> np.ndarray:
        """bf16(y / rms(y)) row by row, rms over the last axis."""
        a = np.ascontiguousarray(y, dtype=np.float64)
        a2 = a.reshape(-1, a.shape[-1])
        out = np.zeros(a2.shape, dtype=np.uint16)
        st = self.lib.orc_rms_normalize_bf16(_ptr(a2), a2.shape[0], a2.shape[1], _ptr(out))
        if st != ORC_OK:
            raise ValueError(f"orc_rms_normalize_bf16 failed with status {st}")
        return out.reshape(a.shape)

    def chain_block(self, h_bits, w) -> dict:
        """One block of the decode chain (the reading stated in nq_oracle.c).

        h_bits: batch x n bf16 patterns; w: {name: (Upk, Vpk, s1_bits, s2_bits, m, n, r)}
        for q, k, v, o, gate, up, down.  Returns every layer's y (float64), the bf16 inputs
        of o and down, and the next block's input "h_next".
        """
        out = {}
        for name in ("q", "k", "v", "gate", "up"):
            out[name] = self.lowrank_linear_fwd(h_bits, *w[name])
        out["x_o"] = self.round_to_bf16(out["v"])
        out["x_down"] = self.round_to_bf16(out["up"])
        out["o"] = self.lowrank_linear_fwd(out["x_o"], *w["o"])
        out["down"] = self.lowrank_linear_fwd(out["x_down"], *w["down"])
        out["h_next"] = self.rms_normalize_bf16(out["down"])
        return out

    def decode_chain(self, h0_bits, blocks) -> np.ndarray:
        """The whole chain: the input of each block is the previous block's h_next."""
        h = h0_bits
        for w in blocks:
            h = self.chain_block(h, w)["h_next"]
        return h


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def pack_signs(signs):
    return default().pack_signs(signs)


def unpack_signs(packed, cols):
    return default().unpack_signs(packed, cols)


def lowrank_linear_fwd(x_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
    return default().lowrank_linear_fwd(x_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r)


def lowrank_linear_fwd_envelope(x_bits, Upk, Vpk, a_bits, b_bits, m, n, r):
    return default().lowrank_linear_fwd_envelope(x_bits, Upk, Vpk, a_bits, b_bits, m, n, r)


def bits_per_weight_envelope(m, n, r, l):
    return default().bits_per_weight_envelope(m, n, r, l)


def stage1(x_bits, Vpk, s2_bits, n, r):
    return default().stage1(x_bits, Vpk, s2_bits, n, r)


def bits_per_weight(m, n, r):
    return default().bits_per_weight(m, n, r)


def num_threads():
    return default().num_threads()


def round_to_bf16(v):
    return default().round_to_bf16(v)


def rms_normalize_bf16(y):
    return default().rms_normalize_bf16(y)


def chain_block(h_bits, w):
    return default().chain_block(h_bits, w)


def decode_chain(h0_bits, blocks):
    return default().decode_chain(h0_bits, blocks)


def lowrank_linear_bwd_input(dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
    return default().lowrank_linear_bwd_input(dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r)


def transpose_signs(packed, rows, cols):
    return default().transpose_signs(packed, rows, cols)


def lowrank_linear_bwd_scales(x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
    return default().lowrank_linear_bwd_scales(x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r)


def lowrank_linear_bwd_factors(x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r):
    return default().lowrank_linear_bwd_factors(x_bits, dy_bits, Upk, Vpk, s1_bits, s2_bits, m, n, r)

"""The C-ABI library without a GPU: it loads, exports every entry point that
include/nq.h declares, rejects bad arguments on the host before touching a device, and
its host-memory pack / unpack path and storage accounting agree with the oracle and
the golden values."""
import ctypes
import os
import re

import numpy as np
import pytest

import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nq():
    from binary_rank_linear_02_b200 import build

    build.build()
    from binary_rank_linear_02_b200 import nq as mod

    return mod


def declared_functions():
    text = open(os.path.join(ROOT, "include", "nq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nq_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(nq):
    names = declared_functions()
    assert {"nq_pack_signs", "nq_unpack_signs", "nq_lowrank_linear_fwd", "nq_bits_per_weight"} <= set(names)
    lib = ctypes.CDLL(nq.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(nq):
    for code in range(0, -10, -1):
        s = nq.nq_status_string(code)
        assert s.startswith("NQ_")
    assert "unknown" in nq.nq_status_string(-99)


def test_bits_per_weight_golden(nq):
    for (m, n, r, num, den) in pins.load_bits_per_weight():
        assert nq.bits_per_weight(m, n, r) == num / den
    assert nq.bits_per_weight(0, 1, 1) == -1.0
    assert nq.bits_per_weight(1, 1, -3) == -1.0


def test_host_pack_matches_oracle_and_golden(nq, orc):
    for name, signs, expected in pins.load_pack_patterns():
        got = nq.pack_signs(signs)
        assert np.array_equal(got, expected), name
    from binary_rank_linear_02_b200 import synth

    for rows, cols, seed in ((7, 64, 5), (3, 100, 6), (1, 1, 7), (4, 31, 8)):
        s = synth.signs(rows, cols, seed)
        s[0, 0] = 0
        got = nq.pack_signs(s)
        assert np.array_equal(got, orc.pack_signs(s))
        back = nq.unpack_signs(got, cols)
        assert np.array_equal(back, np.where(s >= 0, 1, -1).astype(np.int8))


def test_host_pack_rejects_bad_values(nq):
    bad = np.array([[1, -1, 3, 0]], dtype=np.int8)
    out = np.zeros((1, 1), dtype=np.uint32)
    assert nq.nq_pack_signs(bad.ctypes.data, 1, 4, out.ctypes.data, 0) == nq.NQ_ERR_VALUE


def test_pack_argument_errors(nq):
    out = np.zeros((1, 1), dtype=np.uint32)
    s = np.ones((1, 4), dtype=np.int8)
    assert nq.nq_pack_signs(0, 1, 4, out.ctypes.data, 0) == nq.NQ_ERR_NULL
    assert nq.nq_pack_signs(s.ctypes.data, -1, 4, out.ctypes.data, 0) == nq.NQ_ERR_SHAPE
    assert nq.nq_pack_signs(s.ctypes.data, 0, 4, out.ctypes.data, 0) == nq.NQ_OK
    assert nq.nq_unpack_signs(0, 1, 4, s.ctypes.data, 0) == nq.NQ_ERR_NULL


def test_forward_argument_errors(nq):
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    p = [base + 1024 * i for i in range(6)]
    f = nq.nq_lowrank_linear_fwd
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, -1, p[5], 0) == nq.NQ_ERR_BATCH
    assert f(p[0], p[1], p[2], p[3], p[4], 100, 128, 128, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 0, 128, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 64, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 1 << 17, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, 0, p[5], 0) == nq.NQ_OK
    assert f(0, p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_NULL
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, 1, 0, 0) == nq.NQ_ERR_NULL
    assert f(p[0] + 2, p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_ALIGN
    assert f(p[0], p[1], p[2] + 8, p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_ALIGN
    # weights in host memory are refused (they must live on the device)
    assert f(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_PTRKIND
    assert nq.nq_workspace_reserve(128, 100, 128, 1) == nq.NQ_ERR_SHAPE
    assert nq.nq_workspace_reserve(128, 128, 128, -2) == nq.NQ_ERR_BATCH


def test_host_transpose_matches_oracle(nq, orc):
    """The host-memory transpose (calling thread) equals the oracle's, ragged shapes included."""
    from binary_rank_linear_02_b200 import synth

    for (rows, cols, seed) in ((70, 45, 81), (1, 100, 82), (129, 3, 83), (64, 96, 84)):
        packed = orc.pack_signs(synth.signs(rows, cols, seed))
        got = nq.transpose_signs(packed, rows, cols)
        assert np.array_equal(got, orc.transpose_signs(packed, rows, cols)), (rows, cols)


def test_transpose_and_backward_argument_errors(nq):
    out = np.zeros((4, 1), dtype=np.uint32)
    packed = np.zeros((1, 1), dtype=np.uint32)
    t = nq.nq_transpose_signs
    assert t(0, 1, 4, out.ctypes.data, 0) == nq.NQ_ERR_NULL
    assert t(packed.ctypes.data, 1, 4, 0, 0) == nq.NQ_ERR_NULL
    assert t(packed.ctypes.data, -1, 4, out.ctypes.data, 0) == nq.NQ_ERR_SHAPE
    assert t(packed.ctypes.data, 1, -4, out.ctypes.data, 0) == nq.NQ_ERR_SHAPE
    assert t(packed.ctypes.data, 0, 4, out.ctypes.data, 0) == nq.NQ_OK
    # the input gradient is the forward with the factors exchanged: the same checks, the
    # shape rules applying to (m' = n, n' = m)
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    p = [base + 1024 * i for i in range(6)]
    b = nq.nq_lowrank_linear_bwd_input
    assert b(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, -1, p[5], 0) == nq.NQ_ERR_BATCH
    assert b(p[0], p[1], p[2], p[3], p[4], 100, 128, 128, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert b(p[0], p[1], p[2], p[3], p[4], 128, 128, 64, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert b(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, 0, p[5], 0) == nq.NQ_OK
    assert b(0, p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_NULL
    assert b(p[0] + 2, p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_ALIGN
    assert b(p[0], p[1], p[2], p[3], p[4], 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_PTRKIND
    g = nq.nq_lowrank_linear_bwd_scales
    q = [base + 1024 * i for i in range(10)]
    assert g(*q[:8], 128, 128, 128, -1, q[8], q[9], 0) == nq.NQ_ERR_BATCH
    assert g(*q[:8], 100, 128, 128, 1, q[8], q[9], 0) == nq.NQ_ERR_SHAPE
    assert g(*q[:8], 128, 128, 128, 1, 0, 0, 0) == nq.NQ_OK  # nothing to compute
    assert g(0, *q[1:8], 128, 128, 128, 1, q[8], q[9], 0) == nq.NQ_ERR_NULL
    assert g(*q[:7], q[7] + 4, 128, 128, 128, 1, q[8], q[9], 0) == nq.NQ_ERR_ALIGN
    assert g(*q[:8], 128, 128, 128, 1, q[8], q[9], 0) == nq.NQ_ERR_PTRKIND
    f = nq.nq_lowrank_linear_bwd_factors
    assert f(*q[:6], 128, 128, 128, -1, q[6], q[7], 0) == nq.NQ_ERR_BATCH
    assert f(*q[:6], 128, 130, 128, 1, q[6], q[7], 0) == nq.NQ_ERR_SHAPE
    assert f(*q[:6], 128, 128, 128, 1, 0, 0, 0) == nq.NQ_OK  # nothing to compute
    assert f(*q[:5], 0, 128, 128, 128, 1, q[6], q[7], 0) == nq.NQ_ERR_NULL
    assert f(*q[:6], 128, 128, 128, 1, q[6] + 8, q[7], 0) == nq.NQ_ERR_ALIGN
    assert f(*q[:6], 128, 128, 128, 1, q[6], q[7], 0) == nq.NQ_ERR_PTRKIND


def test_grouped_argument_errors(nq):
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    ptr = [base + 1024 * i for i in range(6)]
    good = nq.nq_linear_desc(ptr[0], ptr[1], ptr[2], ptr[3], ptr[4], ptr[5], 128, 128, 128)
    arr = (nq.nq_linear_desc * 2)(good, good)
    f = nq.nq_lowrank_linear_fwd_grouped
    a = ctypes.addressof(arr)
    assert f(a, 2, -1, 0) == nq.NQ_ERR_BATCH
    assert f(a, -1, 1, 0) == nq.NQ_ERR_SHAPE
    assert f(a, 0, 1, 0) == nq.NQ_OK
    assert f(a, 2, 0, 0) == nq.NQ_OK
    assert f(0, 2, 1, 0) == nq.NQ_ERR_NULL
    arr[1].n = 96
    assert f(a, 2, 1, 0) == nq.NQ_ERR_SHAPE
    arr[1].n = 128
    arr[1].Vpk = ptr[2] + 4
    assert f(a, 2, 1, 0) == nq.NQ_ERR_ALIGN
    arr[1].Vpk = ptr[2]
    arr[0].s1 = 0
    assert f(a, 2, 1, 0) == nq.NQ_ERR_NULL
    arr[0].s1 = ptr[3]
    assert f(a, 2, 1, 0) == nq.NQ_ERR_PTRKIND  # host memory is refused


def test_chain_helper_argument_errors(nq):
    buf = np.zeros(1 << 14, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    src, dst = base, base + 4096
    cast, norm = nq.nq_cast_f32_to_bf16, nq.nq_rms_normalize_bf16
    assert cast(src, -1, dst, 0) == nq.NQ_ERR_SHAPE
    assert cast(src, 0, dst, 0) == nq.NQ_OK
    assert cast(0, 8, dst, 0) == nq.NQ_ERR_NULL
    assert cast(src, 8, 0, 0) == nq.NQ_ERR_NULL
    assert cast(src + 4, 8, dst, 0) == nq.NQ_ERR_ALIGN
    assert cast(src, 8, dst + 2, 0) == nq.NQ_ERR_ALIGN
    assert cast(src, 8, dst, 0) == nq.NQ_ERR_PTRKIND  # host memory is refused
    assert norm(src, -1, 8, dst, 0) == nq.NQ_ERR_SHAPE
    assert norm(src, 2, 0, dst, 0) == nq.NQ_ERR_SHAPE
    assert norm(src, 1 << 31, 8, dst, 0) == nq.NQ_ERR_SHAPE
    assert norm(src, 0, 8, dst, 0) == nq.NQ_OK
    assert norm(0, 2, 8, dst, 0) == nq.NQ_ERR_NULL
    assert norm(src, 2, 8, dst + 8, 0) == nq.NQ_ERR_ALIGN
    assert norm(src, 2, 8, dst, 0) == nq.NQ_ERR_PTRKIND


def test_chain_module_checks_shapes(nq):
    """The chain driver refuses blocks whose layers do not fit the wiring (host-side check,
    before any device work)."""
    import torch

    from binary_rank_linear_02_b200 import chain

    t = torch.zeros(4, dtype=torch.int32)
    w = {name: (t, t, t, t, m, n, r) for (name, m, n, r) in
         [("q", 256, 256, 128), ("k", 256, 256, 128), ("v", 256, 256, 128), ("o", 256, 256, 128),
          ("gate", 384, 256, 128), ("up", 384, 256, 128), ("down", 384, 256, 128)]}
    with pytest.raises(ValueError, match="down"):
        chain.DecodeChain([w], 1)
    with pytest.raises(ValueError):
        chain.DecodeChain([], 1)


def test_grouped_ex_argument_errors(nq):
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    ptr = [base + 1024 * i for i in range(8)]
    good = nq.nq_linear_desc(ptr[0], ptr[1], ptr[2], ptr[3], ptr[4], ptr[5], 128, 128, 128)
    arr = (nq.nq_linear_desc_ex * 2)(nq.nq_linear_desc_ex(good, 0, 0), nq.nq_linear_desc_ex(good, ptr[6], ptr[7]))
    f = nq.nq_lowrank_linear_fwd_grouped_ex
    a = ctypes.addressof(arr)
    assert f(a, 2, -1, 0) == nq.NQ_ERR_BATCH
    assert f(a, 0, 1, 0) == nq.NQ_OK
    assert f(0, 2, 1, 0) == nq.NQ_ERR_NULL
    arr[1].base.m = 100
    assert f(a, 2, 1, 0) == nq.NQ_ERR_SHAPE
    arr[1].base.m = 128
    arr[1].y_bf16 = ptr[6] + 2
    assert f(a, 2, 1, 0) == nq.NQ_ERR_ALIGN
    arr[1].y_bf16 = ptr[6]
    arr[1].y_rmsnorm_bf16 = ptr[7] + 8
    assert f(a, 2, 1, 0) == nq.NQ_ERR_ALIGN
    arr[1].y_rmsnorm_bf16 = ptr[7]
    assert f(a, 2, 1, 0) == nq.NQ_ERR_PTRKIND  # host memory is refused


def test_selftest_argument_errors(nq):
    assert nq.nq_selftest_wait_timeout(10, 0) == nq.NQ_ERR_VALUE
    assert nq.nq_selftest_wait_timeout(10**11, 0) == nq.NQ_ERR_VALUE


def test_admm_argument_errors(nq):
    """The LB-ADMM calls check shapes, values, pointers and alignment on the host, before
    any device work (so these run without a GPU)."""
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    p = [base + 1024 * i for i in range(10)]
    L = nq.lib()
    fz = L.nq_admm_factorize
    assert fz(p[0], 256, 256, 512, p[1], 1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_SHAPE  # r > m
    assert fz(p[0], 256, 200, 128, p[1], 1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_SHAPE
    assert fz(p[0], 256, 256, 128, p[1], 1, 10, 0.0, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_VALUE
    assert fz(p[0], 256, 256, 128, p[1], -1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_VALUE
    assert fz(p[0], 256, 256, 128, p[1], 1, -3, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_VALUE
    assert fz(0, 256, 256, 128, p[1], 1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_NULL
    assert fz(p[0] + 4, 256, 256, 128, p[1], 1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_ALIGN
    # host memory is refused: the initialiser works on device buffers
    assert fz(p[0], 256, 256, 128, p[1], 1, 10, 0.2, 1.05, p[2], p[3], p[4], p[5], None, 0) == nq.NQ_ERR_PTRKIND
    st = [p[2 + i] for i in range(8)]
    assert L.nq_admm_init(p[0], 256, 256, 128, 0, 1, *st, 0) == nq.NQ_ERR_NULL
    assert L.nq_admm_init(p[0], 256, 256, 128, p[1], 65, *st, 0) == nq.NQ_ERR_VALUE
    assert L.nq_admm_init(p[0], 256, 256, 128, p[1], 1, *st, 0) == nq.NQ_ERR_PTRKIND
    assert L.nq_admm_iterate(p[0], 256, 256, 128, *st, 1, 0.2, 0.0, 0) == nq.NQ_ERR_VALUE
    assert L.nq_admm_iterate(p[0], 256, 256, 100, *st, 1, 0.2, 1.05, 0) == nq.NQ_ERR_SHAPE
    assert L.nq_admm_iterate(p[0], 256, 256, 128, *st, 1, 0.2, 1.05, 0) == nq.NQ_ERR_PTRKIND


def test_envelope_bits_per_weight_and_host_errors(nq):
    """(r + 16 l)(m + n)/(m n) by hand: 4096 x 4096, r = 1664 -> 1696/2048 at l = 2,
    1728/2048 at l = 4; l = 1 equals nq_bits_per_weight; argument errors on the host."""
    assert nq.lib().nq_bits_per_weight_envelope(4096, 4096, 1664, 2) == 0.828125
    assert nq.lib().nq_bits_per_weight_envelope(4096, 4096, 1664, 4) == 0.84375
    assert nq.lib().nq_bits_per_weight_envelope(11008, 4096, 2432, 1) == nq.nq_bits_per_weight(11008, 4096, 2432)
    assert nq.lib().nq_bits_per_weight_envelope(4096, 4096, 1664, 0) == -1.0
    buf = np.zeros(1 << 16, dtype=np.uint8)
    base = (buf.ctypes.data + 255) // 256 * 256
    p = [base + 2048 * i for i in range(6)]
    f = nq.lib().nq_lowrank_linear_fwd_envelope
    assert f(p[0], p[1], p[2], p[3], p[4], 2, 128, 128, 128, -1, p[5], 0) == nq.NQ_ERR_BATCH
    assert f(p[0], p[1], p[2], p[3], p[4], 0, 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_VALUE
    assert f(p[0], p[1], p[2], p[3], p[4], 2, 100, 128, 128, 1, p[5], 0) == nq.NQ_ERR_SHAPE
    assert f(p[0], p[1], p[2], 0, p[4], 2, 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_NULL
    assert f(p[0], p[1], p[2], p[3] + 2, p[4], 2, 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_ALIGN
    assert f(p[0], p[1], p[2], p[3], p[4], 2, 128, 128, 128, 1, p[5], 0) == nq.NQ_ERR_PTRKIND
    assert f(p[0], p[1], p[2], p[3], p[4], 2, 128, 128, 128, 0, p[5], 0) == nq.NQ_OK

"""Checks that tie the CPU oracle to facts fixed outside itself.

Each function takes an ``oracle.Oracle`` and raises AssertionError on a mismatch, so the
same checks run on the real oracle (they must pass) and on deliberately broken copies of
it (each copy must fail at least one).  Sources of truth, none of them the oracle:
  * hand-worked numbers in tests/golden/ (each file states its derivation and passage);
  * the materialised weight diag(s1) U V^T diag(s2) built with numpy from the int8
    signs, then one numpy matrix-vector product (a different order of operations and a
    different reader of the signs than the oracle's bit reader);
  * closed forms (all-(+1) signs, rank 1), invariances (negating column k of both U and
    V), linearity, and numpy's / torch's own fp16 and bf16 conversions.
"""
from __future__ import annotations

import os

import numpy as np

from binary_rank_linear_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def load_pack_patterns():
    rows = []
    with open(os.path.join(GOLDEN, "pack_patterns.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, cols, pattern, words = [p.strip() for p in line.split("|")]
            cols = int(cols)
            kind, arg = pattern.split(":")
            if kind == "all":
                s = np.full(cols, int(arg), dtype=np.int8)
            elif kind == "alt":
                first = int(arg)
                s = np.array([first if c % 2 == 0 else -first for c in range(cols)], dtype=np.int8)
            elif kind == "one":
                s = np.full(cols, -1, dtype=np.int8)
                s[int(arg)] = 1
            else:
                raise ValueError(kind)
            expected = np.array([int(w, 16) for w in words.split()], dtype=np.uint32)
            rows.append((name, s.reshape(1, cols), expected.reshape(1, -1)))
    return rows


def load_bits_per_weight():
    out = []
    with open(os.path.join(GOLDEN, "bits_per_weight.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            m, n, r, num, den = (int(v) for v in line.split())
            out.append((m, n, r, num, den))
    return out


def dense_reference(x_bits, U, V, s1_bits, s2_bits):
    """y = x W^T with W = diag(s1) U V^T diag(s2), materialised with numpy in float64."""
    x = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    s1 = synth.f16_bits_to_f32(s1_bits).astype(np.float64)
    s2 = synth.f16_bits_to_f32(s2_bits).astype(np.float64)
    W = (s1[:, None] * (U.astype(np.float64) @ V.astype(np.float64).T)) * s2[None, :]
    return x @ W.T


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- individual pins

def pin_decoders(o):
    """Every finite fp16 / bf16 bit pattern decodes to numpy's / the IEEE value."""
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        f16 = allbits.view(np.float16).astype(np.float64)
        bf16 = synth.bf16_bits_to_f32(allbits).astype(np.float64)
    for b in range(0, 1 << 16, 7):  # a stride that visits every exponent and both signs
        if np.isfinite(f16[b]):
            assert o.f16_to_double(b) == f16[b], f"fp16 {b:#06x}"
        if np.isfinite(bf16[b]):
            assert o.bf16_to_double(b) == bf16[b], f"bf16 {b:#06x}"
    for b in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x8001, 0xFBFF):
        assert o.f16_to_double(b) == f16[b]
    for b in (0x0001, 0x007F, 0x0080, 0x3F80, 0x7F7F, 0x8001, 0xC000):
        assert o.bf16_to_double(b) == bf16[b]


def pin_pack_patterns(o):
    for name, signs, expected in load_pack_patterns():
        got = o.pack_signs(signs)
        assert got.shape == expected.shape and np.array_equal(got, expected), name
        back = o.unpack_signs(got, signs.shape[1])
        assert np.array_equal(back, np.where(signs >= 0, 1, -1)), name


def pin_pack_roundtrip(o):
    for rows, cols, seed in ((3, 70, 1), (17, 128, 2), (5, 33, 3)):
        s = synth.signs(rows, cols, seed)
        p = o.pack_signs(s)
        assert p.shape == (rows, (cols + 31) // 32)
        assert np.array_equal(o.unpack_signs(p, cols), s)
        # the words count the +1 entries: popcount of each row = number of +1 in it
        pc = np.array([sum(bin(int(w)).count("1") for w in row) for row in p])
        assert np.array_equal(pc, (s > 0).sum(axis=1))


def pin_handworked(o):
    g = _golden_kv("handworked_small.txt")
    m, n, r, batch = (int(g[k][0]) for k in ("m", "n", "r", "batch"))
    x = np.array([int(v, 16) for v in g["x_bf16"]], dtype=np.uint16).reshape(batch, n)
    s1 = np.array([int(v, 16) for v in g["s1_f16"]], dtype=np.uint16)
    s2 = np.array([int(v, 16) for v in g["s2_f16"]], dtype=np.uint16)
    U = np.array([int(v) for v in g["U_signs"]], dtype=np.int8).reshape(m, r)
    V = np.array([int(v) for v in g["V_signs"]], dtype=np.int8).reshape(n, r)
    Upk = np.array([int(v, 16) for v in g["Upk"]], dtype=np.uint32).reshape(m, 1)
    Vpk = np.array([int(v, 16) for v in g["Vpk"]], dtype=np.uint32).reshape(r, 1)
    assert np.array_equal(o.pack_signs(U), Upk)
    assert np.array_equal(o.pack_signs(np.ascontiguousarray(V.T)), Vpk)
    t = o.stage1(x, Vpk, s2, n, r)
    assert np.array_equal(t, np.array([float(v) for v in g["t"]]).reshape(batch, r))
    y = o.lowrank_linear_fwd(x, Upk, Vpk, s1, s2, m, n, r)
    assert np.array_equal(y, np.array([float(v) for v in g["y"]]).reshape(batch, m))


def _case(m, n, r, batch, seed):
    U = synth.signs(m, r, seed, "U")
    V = synth.signs(n, r, seed, "V")
    s1 = synth.scales_f16(m, seed, "s1")
    s2 = synth.scales_f16(n, seed, "s2")
    x = synth.activations_bf16(batch, n, seed)
    return x, U, V, s1, s2


def _fwd(o, x, U, V, s1, s2):
    m, r = U.shape
    n = V.shape[0]
    return o.lowrank_linear_fwd(x, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2, m, n, r)


def pin_dense_materialised(o):
    """Factorised evaluation equals the materialised dense product (fp64, 1e-12)."""
    for (m, n, r, batch, seed) in ((8, 12, 3, 2, 11), (33, 40, 7, 3, 12), (64, 64, 64, 2, 13), (5, 70, 40, 1, 14)):
        x, U, V, s1, s2 = _case(m, n, r, batch, seed)
        y = _fwd(o, x, U, V, s1, s2)
        y_ref = dense_reference(x, U, V, s1, s2)
        assert y.shape == (batch, m)
        assert rel_err(y, y_ref) <= 1e-12, (m, n, r, rel_err(y, y_ref))


def pin_column_negation(o):
    """Negating column k of both U and V leaves y bit-identical (t_k and U_ik flip together)."""
    x, U, V, s1, s2 = _case(48, 64, 9, 2, 21)
    y0 = _fwd(o, x, U, V, s1, s2)
    for k in (0, 4, 8):
        U2, V2 = U.copy(), V.copy()
        U2[:, k] *= -1
        V2[:, k] *= -1
        assert np.array_equal(_fwd(o, x, U2, V2, s1, s2), y0), k
    # negating only one factor's column changes y (so the check above has teeth)
    U3 = U.copy()
    U3[:, 4] *= -1
    assert not np.array_equal(_fwd(o, x, U3, V, s1, s2), y0)


def pin_closed_forms(o):
    m, n, batch = 24, 40, 2
    x, _, _, s1, s2 = _case(m, n, 1, batch, 31)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    s1f = synth.f16_bits_to_f32(s1).astype(np.float64)
    s2f = synth.f16_bits_to_f32(s2).astype(np.float64)
    # all signs +1: y_i = s1_i * r * sum_j s2_j x_j
    for r in (1, 5, 32):
        U = np.ones((m, r), dtype=np.int8)
        V = np.ones((n, r), dtype=np.int8)
        y = _fwd(o, x, U, V, s1, s2)
        expect = s1f[None, :] * r * (xf @ s2f)[:, None]
        assert rel_err(y, expect) <= 1e-13
    # rank 1: y = s1 * u * (v . (s2 * x))
    u = synth.signs(m, 1, 32)
    v = synth.signs(n, 1, 33)
    y = _fwd(o, x, u, v, s1, s2)
    expect = (s1f * u[:, 0])[None, :] * ((xf * s2f[None, :]) @ v[:, 0].astype(np.float64))[:, None]
    assert rel_err(y, expect) <= 1e-13


def pin_linearity(o):
    m, n, r = 20, 48, 6
    _, U, V, s1, s2 = _case(m, n, r, 1, 41)
    rng = np.random.default_rng(41)
    # small-integer activations: x1, x2 and x1 + x2 are all exact in bfloat16
    x1 = rng.integers(-8, 9, size=(2, n)).astype(np.float32)
    x2 = rng.integers(-8, 9, size=(2, n)).astype(np.float32)
    b = synth.f32_to_bf16_bits
    y1 = _fwd(o, b(x1), U, V, s1, s2)
    y2 = _fwd(o, b(x2), U, V, s1, s2)
    y12 = _fwd(o, b(x1 + x2), U, V, s1, s2)
    assert rel_err(y12, y1 + y2) <= 1e-12
    y3 = _fwd(o, b(-2 * x1), U, V, s1, s2)
    assert np.array_equal(y3, -2 * y1)
    # y is linear in s1: doubling every s1 (exact in fp16) doubles y exactly
    s1d = (synth.f16_bits_to_f32(s1) * 2).astype(np.float16).view(np.uint16)
    assert np.array_equal(_fwd(o, b(x1), U, V, s1d, s2), 2 * y1)


def pin_bits_per_weight(o):
    for (m, n, r, num, den) in load_bits_per_weight():
        assert o.bits_per_weight(m, n, r) == num / den, (m, n, r)
        # the same figure from the sizes of the stored buffers
        packed_bytes = m * ((r + 31) // 32) * 4 + r * ((n + 31) // 32) * 4
        scale_bytes = 2 * (m + n)
        assert 8 * (packed_bytes + scale_bytes) / (m * n) == num / den
    for bad in ((0, 4, 4), (4, -1, 4), (4, 4, 0)):
        assert o.bits_per_weight(*bad) == -1.0


def load_bf16_rounding():
    rows = []
    with open(os.path.join(GOLDEN, "bf16_rounding.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            mant, expo, hexbits = line.split()[:3]
            rows.append((int(mant), int(expo), int(hexbits, 16)))
    return rows


def pin_bf16_rounding(o):
    """Hand-worked roundings, then torch's own float32 -> bfloat16 cast (round to nearest
    even) on float32 values that cover normals, subnormals and exact half-way points."""
    import math

    import torch

    for mant, expo, want in load_bf16_rounding():
        v = math.ldexp(mant, expo)
        got = int(o.round_to_bf16(np.array([v]))[0])
        assert got == want, (mant, expo, hex(got), hex(want))
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 1 << 32, size=20000, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]              # finite values only
    halfway = (rng.integers(0, 1 << 16, size=4000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    halfway = halfway[(halfway & 0x7F800000) != 0x7F800000]
    f32 = np.concatenate([bits, halfway]).view(np.float32)
    want = torch.from_numpy(f32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.round_to_bf16(f32.astype(np.float64))
    assert np.array_equal(got, want)
    assert int(o.round_to_bf16(np.array([float("inf")]))[0]) == 0x7F80
    assert int(o.round_to_bf16(np.array([-0.0]))[0]) == 0x8000


def pin_rms_normalize(o):
    """Closed forms of y / sqrt(mean(y^2)) and its invariances."""
    # a constant row normalises to exactly 1.0; negative constants to -1.0
    c = np.full((2, 96), 0.37)
    c[1] = -5.25
    out = o.rms_normalize_bf16(c)
    assert np.all(out[0] == 0x3F80) and np.all(out[1] == 0xBF80)
    # (3, 4): mean square 12.5, so 3/sqrt(12.5) = 0.8485... -> 217/256 and
    # 4/sqrt(12.5) = 1.1314 -> 145/128, by hand from the bfloat16 spacing
    assert o.rms_normalize_bf16(np.array([[3.0, 4.0]])).tolist() == [[0x3F59, 0x3F91]]
    # one non-zero entry among n: it becomes +-sqrt(n) (n = 64 -> 8.0 exactly)
    e = np.zeros((1, 64))
    e[0, 5] = -0.001
    out = o.rms_normalize_bf16(e)
    assert out[0, 5] == 0xC100 and np.all(np.delete(out[0], 5) == 0)
    # scaling by a power of two and negation change nothing / flip the sign bit only
    rng = np.random.default_rng(12)
    y = rng.standard_normal((3, 4096)) * 1.7
    base = o.rms_normalize_bf16(y)
    assert np.array_equal(o.rms_normalize_bf16(y * 2.0 ** 9), base)
    assert np.array_equal(o.rms_normalize_bf16(-y), base ^ 0x8000)
    # the output has unit root-mean-square up to the bfloat16 rounding (relative 2^-9)
    vals = torch_bf16_to_f64(base)
    assert np.all(np.abs(np.sqrt(np.mean(vals ** 2, axis=1)) - 1.0) < 2.0 ** -8)
    # a zero row stays zero (signed zeros kept)
    z = np.array([[0.0, -0.0, 0.0]])
    assert o.rms_normalize_bf16(z).tolist() == [[0x0000, 0x8000, 0x0000]]


def _tiny_chain_weights(seed, d=64, f=96, ra=32, rf=48):
    shapes = {"q": (d, d, ra), "k": (d, d, ra), "v": (d, d, ra), "o": (d, d, ra),
              "gate": (f, d, rf), "up": (f, d, rf), "down": (d, f, rf)}
    w, dense = {}, {}
    for name, (m, n, r) in shapes.items():
        U = synth.signs(m, r, seed, name, "U")
        V = synth.signs(n, r, seed, name, "V")
        s1 = synth.scales_f16(m, seed, name, "s1")
        s2 = synth.scales_f16(n, seed, name, "s2")
        dense[name] = (U, V, s1, s2)
        w[name] = (None, None, s1, s2, m, n, r)
    return w, dense


def pin_chain_block(o):
    """One block of the decode chain against the same wiring built from materialised
    dense layers (numpy), torch's bfloat16 cast and a numpy root-mean-square."""
    import torch

    w, dense = _tiny_chain_weights(31)
    for name, (U, V, s1, s2) in dense.items():
        _, _, _, _, m, n, r = w[name]
        w[name] = (o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2, m, n, r)
    h = synth.activations_bf16(2, 64, 31, "h")

    def ref(x_bits, name):
        return dense_reference(x_bits, *dense[name])

    def to_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32).to(
            torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    out = o.chain_block(h, w)
    for name in ("q", "k", "v", "gate", "up"):
        assert rel_err(out[name], ref(h, name)) <= 1e-12, name
    assert np.array_equal(out["x_o"], to_bf16(out["v"]))
    assert np.array_equal(out["x_down"], to_bf16(out["up"]))
    assert rel_err(out["o"], ref(out["x_o"], "o")) <= 1e-12
    assert rel_err(out["down"], ref(out["x_down"], "down")) <= 1e-12
    y = out["down"]
    want = y / np.sqrt(np.mean(y * y, axis=1, keepdims=True))
    got = torch_bf16_to_f64(out["h_next"])
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want))
    # the chain feeds each block's h_next to the next block
    w2 = dict(w)
    h2 = o.decode_chain(h, [w, w2])
    assert np.array_equal(h2, o.chain_block(out["h_next"], w2)["h_next"])


def dense_input_gradient(dy_bits, U, V, s1_bits, s2_bits):
    """dx = dy W with W = diag(s1) U V^T diag(s2), materialised with numpy in float64."""
    dy = synth.bf16_bits_to_f32(dy_bits).astype(np.float64)
    s1 = synth.f16_bits_to_f32(s1_bits).astype(np.float64)
    s2 = synth.f16_bits_to_f32(s2_bits).astype(np.float64)
    W = (s1[:, None] * (U.astype(np.float64) @ V.astype(np.float64).T)) * s2[None, :]
    return dy @ W


def _bwd(o, dy, U, V, s1, s2):
    m, r = U.shape
    n = V.shape[0]
    return o.lowrank_linear_bwd_input(dy, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2, m, n, r)


def pin_bwd_input_dense(o):
    """The input gradient equals dy W for the materialised dense weight (fp64, 1e-12), on
    shapes where m, n and r all differ (a swapped operand cannot line up)."""
    for (m, n, r, batch, seed) in ((8, 12, 3, 2, 51), (33, 40, 7, 3, 52), (5, 70, 40, 1, 53)):
        _, U, V, s1, s2 = _case(m, n, r, batch, seed)
        dy = synth.activations_bf16(batch, m, seed, "dy")
        dx = _bwd(o, dy, U, V, s1, s2)
        assert dx.shape == (batch, n)
        assert rel_err(dx, dense_input_gradient(dy, U, V, s1, s2)) <= 1e-12, (m, n, r)


def pin_bwd_input_adjoint(o):
    """The adjoint identity <y(x), dy> = <x, dx(dy)> ties the input gradient to the forward
    pass: both sides are the bilinear form dy^T W x (fp64, 1e-12 relative)."""
    for (m, n, r, batch, seed) in ((24, 40, 9, 3, 61), (64, 32, 17, 2, 62)):
        x, U, V, s1, s2 = _case(m, n, r, batch, seed)
        dy = synth.activations_bf16(batch, m, seed, "dy")
        y = _fwd(o, x, U, V, s1, s2)
        dx = _bwd(o, dy, U, V, s1, s2)
        lhs = float(np.sum(y * synth.bf16_bits_to_f32(dy).astype(np.float64)))
        rhs = float(np.sum(synth.bf16_bits_to_f32(x).astype(np.float64) * dx))
        assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0), (m, n, r, lhs, rhs)


def _bwd_scales(o, x, dy, U, V, s1, s2):
    m, r = U.shape
    n = V.shape[0]
    return o.lowrank_linear_bwd_scales(x, dy, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2,
                                       m, n, r)


def pin_bwd_scales_linear_in_scale(o):
    """L = sum(dy * y) is linear in every scale entry, so dL/ds1_i = (L(s1) - L(s1 with
    entry i set to 0)) / s1_i, and likewise for s2_j; L taken from the forward oracle."""
    m, n, r, batch = 12, 20, 5, 3
    x, U, V, s1, s2 = _case(m, n, r, batch, 81)
    dy = synth.activations_bf16(batch, m, 81, "dy")
    dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
    ds1, ds2 = _bwd_scales(o, x, dy, U, V, s1, s2)
    assert ds1.shape == (m,) and ds2.shape == (n,)

    def loss(a, b):
        return float(np.sum(dyf * _fwd(o, x, U, V, a, b)))

    L0 = loss(s1, s2)
    s1f = synth.f16_bits_to_f32(s1).astype(np.float64)
    s2f = synth.f16_bits_to_f32(s2).astype(np.float64)
    for i in (0, 5, m - 1):
        a = s1.copy()
        a[i] = 0
        fd = (L0 - loss(a, s2)) / s1f[i]
        assert abs(fd - ds1[i]) <= 1e-11 * max(1.0, abs(fd)), (i, fd, ds1[i])
    for j in (0, 7, n - 1):
        b = s2.copy()
        b[j] = 0
        fd = (L0 - loss(s1, b)) / s2f[j]
        assert abs(fd - ds2[j]) <= 1e-11 * max(1.0, abs(fd)), (j, fd, ds2[j])


def pin_bwd_scales_dense(o):
    """ds1 = sum_b dy_b (.) (U V^T diag(s2) x_b) and ds2 = sum_b x_b (.) (V U^T diag(s1) dy_b),
    with the factors materialised by numpy (fp64, 1e-12)."""
    for (m, n, r, batch, seed) in ((9, 14, 4, 2, 82), (40, 24, 11, 3, 83)):
        x, U, V, s1, s2 = _case(m, n, r, batch, seed)
        dy = synth.activations_bf16(batch, m, seed, "dy")
        ds1, ds2 = _bwd_scales(o, x, dy, U, V, s1, s2)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
        s1f = synth.f16_bits_to_f32(s1).astype(np.float64)
        s2f = synth.f16_bits_to_f32(s2).astype(np.float64)
        UV = U.astype(np.float64) @ V.astype(np.float64).T  # m x n
        z = (xf * s2f[None, :]) @ UV.T                      # batch x m
        w = (dyf * s1f[None, :]) @ UV                       # batch x n
        assert rel_err(ds1, np.sum(dyf * z, axis=0)) <= 1e-12
        assert rel_err(ds2, np.sum(xf * w, axis=0)) <= 1e-12


def pin_bwd_factors_sign_flip(o):
    """L = sum(dy * y) is linear in every entry of U (and of V), so negating U[i][k] changes
    L by -2 U[i][k] dU[i][k]: dU[i][k] = (L(U) - L(U with entry (i, k) negated)) / (2 U[i][k]),
    L from the forward oracle; likewise dV."""
    m, n, r, batch = 10, 14, 6, 3
    x, U, V, s1, s2 = _case(m, n, r, batch, 91)
    dy = synth.activations_bf16(batch, m, 91, "dy")
    dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
    dU, dV = o.lowrank_linear_bwd_factors(x, dy, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2,
                                          m, n, r)
    assert dU.shape == (m, r) and dV.shape == (n, r)

    def loss(Ux, Vx):
        return float(np.sum(dyf * _fwd(o, x, Ux, Vx, s1, s2)))

    L0 = loss(U, V)
    for (i, k) in ((0, 0), (4, 3), (m - 1, r - 1)):
        U2 = U.copy()
        U2[i, k] *= -1
        fd = (L0 - loss(U2, V)) / (2.0 * U[i, k])
        assert abs(fd - dU[i, k]) <= 1e-11 * max(1.0, abs(fd)), (i, k, fd, dU[i, k])
    for (j, k) in ((0, 1), (7, 5), (n - 1, 0)):
        V2 = V.copy()
        V2[j, k] *= -1
        fd = (L0 - loss(U, V2)) / (2.0 * V[j, k])
        assert abs(fd - dV[j, k]) <= 1e-11 * max(1.0, abs(fd)), (j, k, fd, dV[j, k])


def pin_bwd_factors_dense(o):
    """dU = diag(s1) dy^T (x diag(s2) V) and dV = diag(s2) x^T (dy diag(s1) U), numpy fp64."""
    m, n, r, batch = 24, 18, 7, 4
    x, U, V, s1, s2 = _case(m, n, r, batch, 92)
    dy = synth.activations_bf16(batch, m, 92, "dy")
    dU, dV = o.lowrank_linear_bwd_factors(x, dy, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), s1, s2,
                                          m, n, r)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
    s1f = synth.f16_bits_to_f32(s1).astype(np.float64)
    s2f = synth.f16_bits_to_f32(s2).astype(np.float64)
    t = (xf * s2f[None, :]) @ V.astype(np.float64)   # batch x r
    u = (dyf * s1f[None, :]) @ U.astype(np.float64)  # batch x r
    assert rel_err(dU, s1f[:, None] * (dyf.T @ t)) <= 1e-12
    assert rel_err(dV, s2f[:, None] * (xf.T @ u)) <= 1e-12


def pin_transpose_signs(o):
    """The packed transpose is numpy's transpose of the unpacked signs (ragged shapes
    included), and transposing twice gives the original words back."""
    for (rows, cols, seed) in ((70, 45, 71), (32, 32, 72), (1, 100, 73), (129, 3, 74)):
        s = synth.signs(rows, cols, seed)
        p = o.pack_signs(s)
        t = o.transpose_signs(p, rows, cols)
        assert t.shape == (cols, (rows + 31) // 32)
        assert np.array_equal(o.unpack_signs(t, rows), s.T)
        assert np.array_equal(o.transpose_signs(t, cols, rows), p)


def _envelope_case(m, n, r, l, batch, seed):
    x, U, V, _, _ = _case(m, n, r, batch, seed)
    a = np.stack([synth.scales_f16(m, seed, "env-a", q) for q in range(l)])
    b = np.stack([synth.scales_f16(n, seed, "env-b", q) for q in range(l)])
    return x, U, V, a, b


def _env(o, x, U, V, a, b):
    m, r = U.shape
    n = V.shape[0]
    return o.lowrank_linear_fwd_envelope(x, o.pack_signs(U), o.pack_signs(np.ascontiguousarray(V.T)), a, b, m, n, r)


def pin_envelope_l1_is_forward(o):
    """A rank-1 envelope is the plain s1/s2 scaling: bit for bit the forward pass."""
    for (m, n, r, batch, seed) in ((8, 12, 3, 2, 61), (64, 96, 32, 3, 62)):
        x, U, V, a, b = _envelope_case(m, n, r, 1, batch, seed)
        assert np.array_equal(_env(o, x, U, V, a, b), _fwd(o, x, U, V, a[0], b[0]))


def pin_envelope_dense(o):
    """The envelope evaluation equals the materialised weight (sum_q a_q b_q^T) (.) (U V^T)
    applied to x by numpy (fp64, 1e-12), for l = 2, 3, 4."""
    for (m, n, r, l, batch, seed) in ((8, 12, 3, 2, 2, 63), (33, 40, 7, 3, 3, 64), (64, 64, 64, 4, 2, 65)):
        x, U, V, a, b = _envelope_case(m, n, r, l, batch, seed)
        af = a.view(np.float16).astype(np.float64)
        bf = b.view(np.float16).astype(np.float64)
        W = (af.T @ bf) * (U.astype(np.float64) @ V.T.astype(np.float64))
        xd = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        y = _env(o, x, U, V, a, b)
        assert y.shape == (batch, m)
        assert rel_err(y, xd @ W.T) <= 1e-12, (m, n, r, l)


def pin_envelope_repeated_term(o):
    """Two equal envelope terms (a, b), (a, b) give exactly the single term (2a, b): doubling
    is exact in fp16 and in double, so the two results agree bit for bit."""
    x, U, V, a, b = _envelope_case(40, 24, 8, 1, 2, 66)
    a2 = (a.view(np.float16) * np.float16(2)).view(np.uint16)
    y_two = _env(o, x, U, V, np.concatenate([a, a]), np.concatenate([b, b]))
    assert np.array_equal(y_two, _env(o, x, U, V, a2, b))


def pin_envelope_column_negation(o):
    """Negating column k of both U and V leaves every envelope term, and so y, bit-identical."""
    x, U, V, a, b = _envelope_case(24, 40, 9, 3, 2, 67)
    U2, V2 = U.copy(), V.copy()
    U2[:, 4] *= -1
    V2[:, 4] *= -1
    assert np.array_equal(_env(o, x, U, V, a, b), _env(o, x, U2, V2, a, b))


def pin_envelope_bits_per_weight(o):
    """(r + 16 l)(m + n) / (m n), worked by hand: 4096 x 4096, r = 1664: l = 1 gives
    1680/2048 = 0.8203125, l = 2 gives 1696/2048 = 0.828125, l = 4 gives 1728/2048 =
    0.84375 (since (m + n)/(m n) = 8192/16777216 = 1/2048)."""
    assert o.bits_per_weight_envelope(4096, 4096, 1664, 1) == 0.8203125
    assert o.bits_per_weight_envelope(4096, 4096, 1664, 2) == 0.828125
    assert o.bits_per_weight_envelope(4096, 4096, 1664, 4) == 0.84375
    assert o.bits_per_weight_envelope(4096, 4096, 1664, 1) == o.bits_per_weight(4096, 4096, 1664)
    for bad in ((0, 4, 4, 1), (4, 4, 4, 0)):
        assert o.bits_per_weight_envelope(*bad) == -1.0


def torch_bf16_to_f64(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


ALL_PINS = [
    pin_decoders,
    pin_pack_patterns,
    pin_pack_roundtrip,
    pin_handworked,
    pin_dense_materialised,
    pin_column_negation,
    pin_closed_forms,
    pin_linearity,
    pin_bits_per_weight,
    pin_bf16_rounding,
    pin_rms_normalize,
    pin_chain_block,
    pin_bwd_input_dense,
    pin_bwd_input_adjoint,
    pin_transpose_signs,
    pin_bwd_scales_linear_in_scale,
    pin_bwd_scales_dense,
    pin_bwd_factors_sign_flip,
    pin_bwd_factors_dense,
    pin_envelope_l1_is_forward,
    pin_envelope_dense,
    pin_envelope_repeated_term,
    pin_envelope_column_negation,
    pin_envelope_bits_per_weight,
]

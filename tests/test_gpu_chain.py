"""The decode chain on the GPU against the CPU oracle, through the C ABI.

Chain wiring (the library's reading; the pages print no model around the layers): each
block's input h feeds q, k, v, gate and up; o reads bf16(v's y), down reads bf16(up's y);
the next block's input is bf16(down's y / rms(down's y)).

Checks:
  * the two glue kernels alone: the cast bit for bit against the oracle's rounding of the
    same float32 values (NaN compared as NaN), the RMS normalisation within one bfloat16
    unit in the last place (the oracle forms the RMS in float64, the kernel in float32,
    so a value within rounding error of a half-way point may round either way);
  * every step of the chain on the GPU's own inputs to that step ("teacher forcing"):
    each layer's y at the forward's bar (max|y - y_ref| / max|y_ref| <= 2e-3), the casts
    bit for bit, the normalisation within one unit in the last place;
  * the whole chain against the oracle's own chain from the same input.  The two chains
    round their intermediate vectors to bfloat16 independently; wherever a value sits
    within the forward's error of a rounding boundary the two round it apart by one unit
    in the last place (at most 2^-7 of the value), the normalisation keeps the scale, the
    random +-1 layers carry a relative difference through at about its size, and the
    differences of successive blocks are independent, so they add up like a random walk.
    Bound used: root-mean-square relative difference <= 2^-7 * sqrt(blocks) (one unit on
    every element in every block), and cosine similarity >= 1 - 2^-9.  Measured on a
    B200: 1.8e-2 after the 32 Llama-2-7B-shaped blocks (bound 4.4e-2), cosine 0.99983.
"""
import numpy as np
import pytest

from binary_rank_linear_02_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3
ULP_REL = 2.0 ** -7  # largest spacing of bfloat16 relative to the value


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from binary_rank_linear_02_b200 import nq as mod

    return mod


@pytest.fixture(scope="module")
def chain_mod(nq):
    from binary_rank_linear_02_b200 import chain

    return chain


def bf16_to_f64(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits).view(np.uint16)).astype(np.float64)


def rel_err(y, y_ref):
    return float(np.max(np.abs(np.asarray(y, np.float64) - y_ref)) / np.max(np.abs(y_ref)))


def within_one_ulp(got_bits, want_bits):
    """Element-wise: equal, or adjacent bfloat16 values of the same sign."""
    g = np.asarray(got_bits).view(np.uint16).astype(np.int64)
    w = np.asarray(want_bits).view(np.uint16).astype(np.int64)
    same_sign = (g >> 15) == (w >> 15)
    return (g == w) | (same_sign & (np.abs(g - w) == 1))


def to_device(blocks):
    dev = torch.device("cuda")
    out = []
    for w in blocks:
        d = {}
        for name, (U, V, s1, s2, m, n, r) in w.items():
            d[name] = (torch.from_numpy(U.view(np.int32)).to(dev), torch.from_numpy(V.view(np.int32)).to(dev),
                       torch.from_numpy(s1.view(np.int16)).to(dev), torch.from_numpy(s2.view(np.int16)).to(dev),
                       m, n, r)
        out.append(d)
    return out


# ---------------------------------------------------------------------- glue kernels

def special_f32():
    f = np.float32
    vals = [0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, f(3.4028235e38), f(-3.4028235e38), f(1e-40), f(-1e-45),
            f(1.0 + 2 ** -8), f(1.0 + 3 * 2 ** -8), f(2.0 - 2 ** -8), f(1.17549435e-38), f(3.3895314e38),
            f(3.3961776e38)]
    return np.array(vals, dtype=np.float32)


@pytest.mark.parametrize("count", [1, 7, 8, 9, 4099, 15104])
def test_cast_matches_oracle(nq, orc, count):
    rng = np.random.default_rng(count)
    src = (rng.standard_normal(count) * np.exp(rng.uniform(-30, 30, count))).astype(np.float32)
    sp = special_f32()
    src[: min(count, sp.size)] = sp[: min(count, sp.size)]
    got = nq.cast_f32_to_bf16(torch.from_numpy(src).cuda()).cpu().numpy().view(np.uint16)
    want = orc.round_to_bf16(src.astype(np.float64))
    assert np.array_equal(got, want)


def test_cast_nan_stays_nan(nq):
    src = np.array([np.nan, -np.nan, 1.0, np.nan] * 4, dtype=np.float32)
    got = nq.cast_f32_to_bf16(torch.from_numpy(src).cuda()).cpu().numpy().view(np.uint16)
    is_nan = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
    assert np.array_equal(is_nan, np.isnan(src))


@pytest.mark.parametrize("rows,cols", [(1, 4096), (3, 4096), (8, 11008), (5, 100), (2, 1), (4, 8)])
def test_rms_normalize_matches_oracle(nq, orc, rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    src = (rng.standard_normal((rows, cols)) * rng.uniform(0.01, 50.0, (rows, 1))).astype(np.float32)
    got = nq.rms_normalize_bf16(torch.from_numpy(src).cuda()).cpu().numpy().view(np.uint16)
    want = orc.rms_normalize_bf16(src.astype(np.float64))
    ok = within_one_ulp(got, want)
    assert ok.all()
    assert np.mean(got != want) <= 0.01


def test_rms_normalize_zero_and_constant_rows(nq, orc):
    src = np.zeros((3, 64), dtype=np.float32)
    src[0, 1::2] = -0.0
    src[1, :] = 0.75
    src[2, :] = -3.0
    got = nq.rms_normalize_bf16(torch.from_numpy(src).cuda()).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, orc.rms_normalize_bf16(src.astype(np.float64)))
    assert np.all(got[1] == 0x3F80) and np.all(got[2] == 0xBF80)


def test_glue_argument_errors(nq):
    L = nq.lib()
    a = torch.zeros(64, dtype=torch.float32, device="cuda")
    b = torch.zeros(64, dtype=torch.int16, device="cuda")
    assert L.nq_cast_f32_to_bf16(a.data_ptr(), -1, b.data_ptr(), 0) == nq.NQ_ERR_SHAPE
    assert L.nq_cast_f32_to_bf16(None, 8, b.data_ptr(), 0) == nq.NQ_ERR_NULL
    assert L.nq_cast_f32_to_bf16(a.data_ptr() + 4, 8, b.data_ptr(), 0) == nq.NQ_ERR_ALIGN
    assert L.nq_cast_f32_to_bf16(a.data_ptr(), 0, None, 0) == nq.NQ_OK
    assert L.nq_rms_normalize_bf16(a.data_ptr(), 2, 0, b.data_ptr(), 0) == nq.NQ_ERR_SHAPE
    assert L.nq_rms_normalize_bf16(a.data_ptr(), 2, 8, b.data_ptr() + 2, 0) == nq.NQ_ERR_ALIGN
    assert L.nq_rms_normalize_bf16(a.data_ptr(), 0, 8, None, 0) == nq.NQ_OK
    host = np.zeros(64, dtype=np.float32)
    assert L.nq_cast_f32_to_bf16(host.ctypes.data, 8, b.data_ptr(), 0) == nq.NQ_ERR_PTRKIND


# ---------------------------------------------------------------------- the chain

def check_chain(orc, ch, blocks, check_blocks):
    torch.cuda.synchronize()
    h = ch.h.cpu().numpy().view(np.uint16)
    ys = {k: v.cpu().numpy() for k, v in ch.y.items()}
    x_o = ch.x_o.cpu().numpy().view(np.uint16)
    x_down = ch.x_down.cpu().numpy().view(np.uint16)
    for i in check_blocks:
        w = blocks[i]
        for name in ("q", "k", "v", "gate", "up"):
            ref = orc.lowrank_linear_fwd(h[i], *w[name])
            assert rel_err(ys[name][i], ref) <= TOL, (i, name, rel_err(ys[name][i], ref))
        assert np.array_equal(x_o[i], orc.round_to_bf16(ys["v"][i].astype(np.float64))), i
        assert np.array_equal(x_down[i], orc.round_to_bf16(ys["up"][i].astype(np.float64))), i
        for name, xin in (("o", x_o[i]), ("down", x_down[i])):
            ref = orc.lowrank_linear_fwd(xin, *w[name])
            assert rel_err(ys[name][i], ref) <= TOL, (i, name, rel_err(ys[name][i], ref))
        want = orc.rms_normalize_bf16(ys["down"][i].astype(np.float64))
        assert within_one_ulp(h[i + 1], want).all(), i
        assert np.mean(h[i + 1] != want) <= 0.01, i
    # the whole chain against the oracle's own chain from the same input
    ref_last = bf16_to_f64(orc.decode_chain(h[0], blocks))
    got_last = bf16_to_f64(h[len(blocks)])
    nb = len(blocks)
    rms_rel = np.linalg.norm(got_last - ref_last) / np.linalg.norm(ref_last)
    cos = float(np.sum(got_last * ref_last) / (np.linalg.norm(got_last) * np.linalg.norm(ref_last)))
    print(f"chain of {nb} blocks: rms relative difference {rms_rel:.3e}, cosine {cos:.6f}")
    assert rms_rel <= ULP_REL * np.sqrt(nb)
    assert cos >= 1 - 2.0 ** -9


@pytest.mark.parametrize("batch", [1, 3, 8])
def test_small_chain(nq, chain_mod, orc, batch):
    blocks = synth.chain_weights(6, synth.CHAIN_SMALL_LAYERS, 40 + batch)
    ch = chain_mod.DecodeChain(to_device(blocks), batch)
    h0 = synth.activations_bf16(batch, 256, 40 + batch, "h0")
    ch.run(torch.from_numpy(h0.view(np.int16)).cuda())
    check_chain(orc, ch, blocks, range(len(blocks)))


def test_chain_7b_shapes_32_blocks(nq, chain_mod, orc):
    """The full decode chain: 32 Llama-2-7B-shaped blocks at batch 1, every step checked."""
    blocks = synth.chain_weights(synth.CHAIN_7B_BLOCKS, synth.LLAMA2_7B_LAYERS, 5)
    ch = chain_mod.DecodeChain(to_device(blocks), 1)
    h0 = synth.activations_bf16(1, 4096, 5, "h0")
    ch.run(torch.from_numpy(h0.view(np.int16)).cuda())
    first = ch.h[-1].clone()
    # a second pass over the same input gives the same bits (no state carried between steps)
    ch.run(torch.from_numpy(h0.view(np.int16)).cuda())
    assert torch.equal(first, ch.h[-1])
    check_chain(orc, ch, blocks, range(len(blocks)))


def test_chain_in_cuda_graph(nq, chain_mod):
    """Replaying a captured chain gives the eager chain's bits."""
    blocks = synth.chain_weights(4, synth.CHAIN_SMALL_LAYERS, 77)
    ch = chain_mod.DecodeChain(to_device(blocks), 1)
    h0 = torch.from_numpy(synth.activations_bf16(1, 256, 77, "h0").view(np.int16)).cuda()
    ch.run(h0)
    torch.cuda.synchronize()
    eager = ch.h.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    ch.h.zero_()
    ch.h[0].copy_(h0.view(1, 256))
    with torch.cuda.graph(g, stream=s):
        ch.run()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ch.h, eager)


# ---------------------------------------------------------------------- grouped_ex

@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_grouped_ex_optional_outputs(nq, orc, batch):
    """y of every layer is the plain grouped call's y; y_bf16 is bf16(y) bit for bit;
    y_rmsnorm_bf16 is within one unit of the oracle's normalisation of the same y.  Two
    calls in a row give the same bits (the arrival counters reset themselves)."""
    dev = torch.device("cuda")
    shapes = [(512, 256, 128), (384, 512, 256), (1024, 384, 128)]
    layers, plain = [], []
    keep = []
    for li, (m, n, r) in enumerate(shapes):
        U = synth.random_words(m, r // 32, 90 + batch, li, "U")
        V = synth.random_words(r, n // 32, 90 + batch, li, "V")
        s1 = synth.scales_f16(m, 90 + batch, li, "s1")
        s2 = synth.scales_f16(n, 90 + batch, li, "s2")
        x = synth.activations_bf16(batch, n, 90 + batch, li)
        t = [torch.from_numpy(a.view(v)).to(dev) for a, v in ((x, np.int16), (U, np.int32), (V, np.int32),
                                                              (s1, np.int16), (s2, np.int16))]
        y = torch.empty((batch, m), dtype=torch.float32, device=dev)
        y2 = torch.empty_like(y)
        yb = torch.empty((batch, m), dtype=torch.int16, device=dev) if li != 1 else None
        yn = torch.empty((batch, m), dtype=torch.int16, device=dev) if li != 0 else None
        keep += [t, y, y2, yb, yn]
        layers.append((t[0], t[1], t[2], t[3], t[4], y, m, n, r, yb, yn))
        plain.append((t[0], t[1], t[2], t[3], t[4], y2, m, n, r))
    nq.lowrank_linear_fwd_grouped(plain, batch)
    nq.lowrank_linear_fwd_grouped_ex(layers, batch)
    torch.cuda.synchronize()
    first = [(l[9].clone() if l[9] is not None else None, l[10].clone() if l[10] is not None else None)
             for l in layers]
    nq.lowrank_linear_fwd_grouped_ex(layers, batch)
    torch.cuda.synchronize()
    for li, l in enumerate(layers):
        y = l[5]
        assert torch.equal(y, plain[li][5]), li
        y64 = y.cpu().numpy().astype(np.float64)
        if l[9] is not None:
            got = l[9].cpu().numpy().view(np.uint16)
            assert np.array_equal(got, orc.round_to_bf16(y64)), li
            assert torch.equal(l[9], first[li][0])
        if l[10] is not None:
            got = l[10].cpu().numpy().view(np.uint16)
            want = orc.rms_normalize_bf16(y64)
            assert within_one_ulp(got, want).all(), li
            assert np.mean(got != want) <= 0.01, li
            assert torch.equal(l[10], first[li][1])

"""CUDA path against the CPU oracle on activations that stress its number formats.

The decode kernels quantise s2 (.) x per 1024-column chunk and t per token to 14-bit
integers with one power-of-two exponent each; the prefill kernels carry x' and T in fp16
under one power of two per token.  N(0, 1) activations never reach the edges of those
formats, so these cases do:

  * outlier channels: a few columns of every 1024-column chunk at 10^2..10^4 times the
    typical magnitude (the "massive activations" of decoder hidden states): one entry
    sets a chunk's exponent and the other 1021 are quantised against it;
  * a wide dynamic range inside every chunk: magnitudes 2^-20 .. 2^10;
  * tokens of very different magnitude in one call (1e-20 .. 1e20): each token keeps its
    own exponent;
  * on the prefill path, x' = s2 x beyond fp16's range at both ends (|x'| ~ 6e4 and
    ~ 1e-8), where a plain fp16 x' or T would overflow or fall into subnormals.

Every output is compared with the fp64 oracle.  Two bars, both at 2e-3: the global
max|y - y_ref| / max|y_ref| of the factorised-linear benchmarks, and the same ratio per
token (each token against its own largest output), which a call mixing tiny and huge
tokens would fail if a token lost precision to another.
"""
import numpy as np
import pytest

from binary_rank_linear_02_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from binary_rank_linear_02_b200 import nq as mod

    return mod


def errors(y, y_ref):
    """(global, worst per-token) relative error."""
    y = np.asarray(y, dtype=np.float64)
    diff = np.abs(y - y_ref)
    glob = float(diff.max() / np.abs(y_ref).max())
    per_tok = float(np.max(diff.max(axis=1) / np.abs(y_ref).max(axis=1)))
    return glob, per_tok


class Layer:
    """One factorised layer with seeded signs and scales and the given bf16 activations."""

    def __init__(self, orc, nq, m, n, r, x, seed):
        self.m, self.n, self.r, self.batch = m, n, r, x.shape[0]
        U = synth.signs(m, r, seed, "U")
        Vt = np.ascontiguousarray(synth.signs(n, r, seed, "V").T)
        self.s1 = synth.scales_f16(m, seed, "s1")
        self.s2 = synth.scales_f16(n, seed, "s2")
        self.x = x
        self.Upk_o = orc.pack_signs(U)
        self.Vpk_o = orc.pack_signs(Vt)
        dev = torch.device("cuda")
        self.Upk = nq.pack_signs(torch.from_numpy(U).to(dev))
        self.Vpk = nq.pack_signs(torch.from_numpy(Vt).to(dev))
        self.s1_d = torch.from_numpy(self.s1.view(np.int16)).to(dev)
        self.s2_d = torch.from_numpy(self.s2.view(np.int16)).to(dev)
        self.x_d = torch.from_numpy(x.view(np.int16)).to(dev)

    def gpu(self, nq):
        y = nq.lowrank_linear_fwd(self.x_d, self.Upk, self.Vpk, self.s1_d, self.s2_d, self.m, self.n, self.r)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def oracle(self, orc, rows=None):
        x = self.x if rows is None else np.ascontiguousarray(self.x[rows])
        return orc.lowrank_linear_fwd(x, self.Upk_o, self.Vpk_o, self.s1, self.s2, self.m, self.n, self.r)


def check(y, ref):
    glob, per_tok = errors(y, ref)
    assert np.all(np.isfinite(y))
    assert glob <= TOL, f"global relative error {glob:.3e}"
    assert per_tok <= TOL, f"per-token relative error {per_tok:.3e}"


# The decode configurations' layer shapes: Llama-2-7B q, gate, down; Llama-2-70B q, k, gate, down.
DECODE_SHAPES = [
    ("7b-q", 4096, 4096, 1664),
    ("7b-gate", 11008, 4096, 2432),
    ("7b-down", 4096, 11008, 2432),
    ("70b-q", 8192, 8192, 2432),
    ("70b-k", 1024, 8192, 384),
    ("70b-gate", 28672, 8192, 3840),
    ("70b-down", 8192, 28672, 3840),
]


# ------------------------------------------------------------------ decode (batch <= 8)

@pytest.mark.parametrize("batch", [1, 4, 8])
@pytest.mark.parametrize("name,m,n,r", DECODE_SHAPES)
def test_decode_outlier_channels(nq, orc, name, m, n, r, batch):
    """Three outlier columns per 1024-column chunk, 10^2..10^4 times the rest."""
    x = synth.activations_outliers_bf16(batch, n, 31, name)
    L = Layer(orc, nq, m, n, r, x, seed=3100 + m + n + r)
    check(L.gpu(nq), L.oracle(orc))


@pytest.mark.parametrize("name,m,n,r", DECODE_SHAPES)
def test_decode_single_huge_outlier(nq, orc, name, m, n, r):
    """One entry per token at 10^4 (the top of the outlier range) and nothing else above
    N(0, 1): the entry's chunk quantises its other 1023 columns at ~2^-13 of their own
    spread, and that chunk dominates t."""
    x = synth.activations_outliers_bf16(2, n, 32, name, per_chunk=1, chunk=n, lo=1e4, hi=1e4)
    L = Layer(orc, nq, m, n, r, x, seed=3200 + m + n + r)
    check(L.gpu(nq), L.oracle(orc))


@pytest.mark.parametrize("batch", [1, 8])
@pytest.mark.parametrize("name,m,n,r", DECODE_SHAPES)
def test_decode_wide_dynamic_range(nq, orc, name, m, n, r, batch):
    """Magnitudes 2^-20 .. 2^10 mixed in every chunk."""
    x = synth.activations_wide_range_bf16(batch, n, 33, name)
    L = Layer(orc, nq, m, n, r, x, seed=3300 + m + n + r)
    check(L.gpu(nq), L.oracle(orc))


TOKEN_SCALES = {
    2: [1e-20, 1e20],
    4: [1e-6, 1e6, 1.0, 1e-3],
    8: [1e-20, 1e-6, 1e-3, 1.0, 1e3, 1e6, 1e20, 1e-4],
}


@pytest.mark.parametrize("batch", [2, 4, 8])
@pytest.mark.parametrize("name,m,n,r", DECODE_SHAPES[:4])
def test_decode_tokens_of_different_magnitude(nq, orc, name, m, n, r, batch):
    """Tokens from 1e-20 to 1e20 times N(0, 1) in one call: each keeps its precision."""
    x = synth.activations_token_scaled_bf16(n, 34, TOKEN_SCALES[batch], name)
    L = Layer(orc, nq, m, n, r, x, seed=3400 + m + n + r)
    check(L.gpu(nq), L.oracle(orc))


@pytest.mark.parametrize("block,batch", [("7b", 1), ("7b", 4), ("7b", 8), ("70b", 1), ("70b", 4)])
def test_grouped_block_outliers(nq, orc, block, batch):
    """The benchmark's grouped decode call (seven layers of one block) with outlier
    channels in every layer's input and, for the attention projections, mixed token
    magnitudes: every output against the oracle."""
    shapes = synth.LLAMA2_7B_LAYERS if block == "7b" else synth.LLAMA2_70B_LAYERS
    layers = []
    for i, (name, m, n, r) in enumerate(shapes):
        if i % 2 == 0:
            x = synth.activations_outliers_bf16(batch, n, 35, block, name)
        else:
            x = synth.activations_token_scaled_bf16(n, 35, [10.0 ** (4 * ((b % 3) - 1)) for b in range(batch)],
                                                    block, name)
        layers.append(Layer(orc, nq, m, n, r, x, seed=3500 + 10 * i + batch))
    ys = [torch.empty((batch, L.m), dtype=torch.float32, device="cuda") for L in layers]
    nq.lowrank_linear_fwd_grouped([(L.x_d, L.Upk, L.Vpk, L.s1_d, L.s2_d, y, L.m, L.n, L.r)
                                   for L, y in zip(layers, ys)], batch)
    torch.cuda.synchronize()
    for L, y in zip(layers, ys):
        check(y.cpu().numpy(), L.oracle(orc))


# ------------------------------------------------------------------ prefill (batch > 8)

PREFILL_SHAPES = [("small", 512, 512, 128), ("7b-gate", 11008, 4096, 2432), ("7b-down", 4096, 11008, 2432)]


def prefill_check(nq, orc, L, sample=None):
    y = L.gpu(nq)
    if sample is None:
        check(y, L.oracle(orc))
    else:
        check(y[sample], L.oracle(orc, sample))


@pytest.mark.parametrize("batch", [9, 16, 64, 128])
@pytest.mark.parametrize("name,m,n,r", PREFILL_SHAPES)
def test_prefill_tokens_of_different_magnitude(nq, orc, name, m, n, r, batch):
    """Prefill batches (the persistent split-K kernel up to 64 tokens, the tile kernel
    above) whose tokens span 1e-20 .. 1e20: x' of the tiny tokens lies far below fp16's
    smallest subnormal and T of the huge ones far above its largest value, unless each
    token carries its own power of two."""
    scales = [10.0 ** (((7 * b) % 41) - 20) for b in range(batch)]
    x = synth.activations_token_scaled_bf16(n, 36, scales, name, batch)
    L = Layer(orc, nq, m, n, r, x, seed=3600 + m + n + r)
    sample = None if m * r * batch <= 512 * 128 * 128 else np.arange(0, batch, max(1, batch // 16))
    prefill_check(nq, orc, L, sample)


@pytest.mark.parametrize("xmag", [3e6, 1e-6])
@pytest.mark.parametrize("batch", [16, 128])
def test_prefill_x_prime_at_fp16_limits(nq, orc, xmag, batch):
    """Every token at the same extreme scale on the Llama-2-7B gate shape: s2 x ~ 6e4
    (fp16's largest finite values; a plain fp16 T would overflow) or ~ 2e-8 (below fp16's
    smallest subnormal)."""
    m, n, r = 11008, 4096, 2432
    x = synth.activations_token_scaled_bf16(n, 37, [xmag] * batch, batch)
    L = Layer(orc, nq, m, n, r, x, seed=3700 + batch)
    prefill_check(nq, orc, L, np.arange(0, batch, max(1, batch // 16)))


@pytest.mark.parametrize("batch", [16, 128])
@pytest.mark.parametrize("kind", ["outliers", "wide"])
def test_prefill_outliers_and_wide_range(nq, orc, kind, batch):
    """The decode cases' activations on the prefill path (7B gate shape)."""
    m, n, r = 11008, 4096, 2432
    if kind == "outliers":
        x = synth.activations_outliers_bf16(batch, n, 38)
    else:
        x = synth.activations_wide_range_bf16(batch, n, 38)
    L = Layer(orc, nq, m, n, r, x, seed=3800 + batch)
    prefill_check(nq, orc, L, np.arange(0, batch, max(1, batch // 16)))


def test_zero_token_beside_huge_ones(nq, orc):
    """A token of zeros among large tokens, on both paths: its outputs are exactly zero."""
    m, n, r = 4096, 4096, 1664
    for batch in (4, 16):
        x = synth.activations_token_scaled_bf16(n, 39, [1e6] * batch, batch)
        x[1] = 0
        L = Layer(orc, nq, m, n, r, x, seed=3900 + batch)
        y = L.gpu(nq)
        assert np.all(y[1] == 0.0)
        ref = L.oracle(orc)
        keep = [b for b in range(batch) if b != 1]
        check(y[keep], ref[keep])

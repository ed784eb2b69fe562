"""CUDA path against the CPU oracle, through the C ABI, on seeded synthetic inputs.

Bar: packing bit-exact; the forward within max|y - y_ref| / max|y_ref| <= 2e-3 (the
tolerance the factorised-linear benchmarks state for bf16 inputs with fp32
accumulation).  Small cases are compared element by element; at full benchmark sizes
the oracle computes every output of the decode configurations, and a sample of token
rows of the large prefill batches.
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


def rel_err(y, y_ref):
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))


class Case:
    """One factorised layer: signs, scales and activations from the seeded generators,
    stored once by the oracle and once by the CUDA packer."""

    def __init__(self, orc, nq, m, n, r, batch, seed, U=None, V=None, x=None):
        self.m, self.n, self.r, self.batch = m, n, r, batch
        self.U = synth.signs(m, r, seed, "U") if U is None else U
        self.V = synth.signs(n, r, seed, "V") if V is None else V
        self.s1 = synth.scales_f16(m, seed, "s1")
        self.s2 = synth.scales_f16(n, seed, "s2")
        self.x = synth.activations_bf16(batch, n, seed) if x is None else x
        self.Upk_o = orc.pack_signs(self.U)
        self.Vpk_o = orc.pack_signs(np.ascontiguousarray(self.V.T))
        dev = torch.device("cuda")
        self.Upk = nq.pack_signs(torch.from_numpy(self.U).to(dev))
        self.Vpk = nq.pack_signs(torch.from_numpy(np.ascontiguousarray(self.V.T)).to(dev))
        self.s1_d = torch.from_numpy(self.s1.view(np.int16)).to(dev)
        self.s2_d = torch.from_numpy(self.s2.view(np.int16)).to(dev)
        self.x_d = torch.from_numpy(self.x.view(np.int16)).to(dev)

    def gpu(self, x_d=None):
        x_d = self.x_d if x_d is None else x_d
        y = nq_mod().lowrank_linear_fwd(x_d, self.Upk, self.Vpk, self.s1_d, self.s2_d, self.m, self.n, self.r)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def oracle(self, orc, rows=None):
        x = self.x if rows is None else self.x[rows]
        return orc.lowrank_linear_fwd(x, self.Upk_o, self.Vpk_o, self.s1, self.s2, self.m, self.n, self.r)


def nq_mod():
    from binary_rank_linear_02_b200 import nq as mod

    return mod


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 100), (128, 4096), (3, 33), (64, 1)])
def test_pack_device_bit_exact(nq, orc, rows, cols):
    s = synth.signs(rows, cols, 3, rows, cols)
    s[0, 0] = 0
    got = nq.pack_signs(torch.from_numpy(s).cuda()).cpu().numpy().view(np.uint32)
    assert np.array_equal(got, orc.pack_signs(s))
    back = nq.unpack_signs(torch.from_numpy(got.view(np.int32)).cuda(), cols).cpu().numpy()
    assert np.array_equal(back, np.where(s >= 0, 1, -1))


def test_pack_device_golden_patterns(nq):
    import pins

    for name, signs, expected in pins.load_pack_patterns():
        got = nq.pack_signs(torch.from_numpy(signs).cuda()).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, expected), name


def test_pack_device_rejects_bad_values(nq):
    s = torch.ones((4, 64), dtype=torch.int8, device="cuda")
    s[2, 17] = 5
    out = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    st = nq.nq_pack_signs(s.data_ptr(), 4, 64, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == nq.NQ_ERR_VALUE


# ------------------------------------------------------------------ forward, small and ragged

SMALL = [
    (512, 512, 128, 1),     # the single-layer workload
    (512, 512, 128, 2),
    (512, 512, 128, 4),
    (512, 512, 128, 5),
    (512, 512, 128, 8),
    (384, 640, 256, 3),
    (128, 128, 128, 1),     # one tile everywhere
    (256, 2176, 2176, 2),   # 17 column blocks: a full chunk plus a ragged one, both stages
    (1152, 384, 1664, 7),
    (512, 512, 128, 9),     # first prefill batches
    (512, 512, 128, 16),
    (640, 384, 256, 33),
]


@pytest.mark.parametrize("m,n,r,batch", [
    (128, 131072, 128, 1),   # 1024 column blocks: 16 per stage-1 CTA, two chunks through the ring
    (256, 98304, 256, 5),    # 768 column blocks: 12 per CTA, a full chunk and a ragged one
    (384, 70144, 128, 2),    # just past 64 splits of 8 column blocks
    (256, 512, 16384, 8),    # deep rank: 128 stage-1 row blocks, 16 stage-2 column spans
    (262144, 128, 128, 1),   # tall output: 2048 stage-2 row tiles
])
def test_forward_wide_input(nq, orc, m, n, r, batch):
    """Extreme shapes: very wide layers, where a stage-1 CTA takes several 1024-column
    chunks (the split count is capped) through its ring; a deep rank that stage 2 holds on
    chip in many spans; a very tall output."""
    c = Case(orc, nq, m, n, r, batch, seed=77 + n)
    assert rel_err(c.gpu(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("m,n,r,batch", SMALL)
def test_forward_small(nq, orc, m, n, r, batch):
    c = Case(orc, nq, m, n, r, batch, seed=1000 + m + n + r + batch)
    y = c.gpu()
    y_ref = c.oracle(orc)
    assert y.shape == (batch, m)
    assert rel_err(y, y_ref) <= TOL


def test_forward_deterministic(nq, orc):
    c = Case(orc, nq, 1024, 4096, 1664, 3, seed=7)
    a, b = c.gpu(), c.gpu()
    assert np.array_equal(a, b)


def test_forward_special_signs(nq, orc):
    m, n, r = 256, 512, 128
    ones_u = np.ones((m, r), np.int8)
    ones_v = np.ones((n, r), np.int8)
    for U, V in ((ones_u, ones_v), (-ones_u, ones_v), (ones_u, -ones_v)):
        c = Case(orc, nq, m, n, r, 2, seed=11, U=U, V=V)
        assert rel_err(c.gpu(), c.oracle(orc)) <= TOL


def test_forward_column_negation(nq, orc):
    m, n, r = 512, 1024, 256
    base = Case(orc, nq, m, n, r, 2, seed=21)
    U2, V2 = base.U.copy(), base.V.copy()
    U2[:, 5] *= -1
    V2[:, 5] *= -1
    U2[:, 200] *= -1
    V2[:, 200] *= -1
    neg = Case(orc, nq, m, n, r, 2, seed=21, U=U2, V=V2)
    assert np.array_equal(neg.oracle(orc), base.oracle(orc))
    y_ref = base.oracle(orc)
    assert rel_err(base.gpu(), y_ref) <= TOL
    assert rel_err(neg.gpu(), y_ref) <= TOL


def test_forward_zero_input(nq, orc):
    c = Case(orc, nq, 256, 256, 128, 2, seed=5, x=np.zeros((2, 256), np.uint16))
    assert np.all(c.gpu() == 0.0)


def test_forward_host_buffers(nq, orc):
    c = Case(orc, nq, 512, 512, 128, 3, seed=9)
    x_host = torch.from_numpy(c.x.view(np.int16)).pin_memory()
    y_dev = c.gpu()
    y_host = nq.lowrank_linear_fwd(x_host, c.Upk, c.Vpk, c.s1_d, c.s2_d, c.m, c.n, c.r)
    assert not y_host.is_cuda
    assert np.array_equal(y_host.numpy(), y_dev)
    x_pageable = torch.from_numpy(c.x.view(np.int16).copy())
    y_out = torch.empty((3, 512), dtype=torch.float32)
    nq.lowrank_linear_fwd(x_pageable, c.Upk, c.Vpk, c.s1_d, c.s2_d, c.m, c.n, c.r, y=y_out)
    assert np.array_equal(y_out.numpy(), y_dev)


# ------------------------------------------------------------------ full benchmark shapes

@pytest.mark.parametrize("name,m,n,r", synth.LLAMA2_7B_LAYERS[3:])
@pytest.mark.parametrize("batch", [1, 8])
def test_forward_llama2_7b_shapes(nq, orc, name, m, n, r, batch):
    c = Case(orc, nq, m, n, r, batch, seed=sum(map(ord, name)))
    assert rel_err(c.gpu(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("name,m,n,r", [synth.LLAMA2_70B_LAYERS[i] for i in (0, 1, 4, 6)])
@pytest.mark.parametrize("batch", [1, 4])
def test_forward_llama2_70b_shapes(nq, orc, name, m, n, r, batch):
    c = Case(orc, nq, m, n, r, batch, seed=70 + len(name))
    assert rel_err(c.gpu(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", list(synth.PREFILL_BATCHES))
def test_forward_prefill_sweep_sampled(nq, orc, batch):
    _, m, n, r = synth.PREFILL_SHAPE
    c = Case(orc, nq, m, n, r, batch, seed=400 + batch)
    y = c.gpu()
    rng = np.random.default_rng(batch)
    rows = np.unique(np.concatenate([[0, batch - 1], rng.choice(batch, size=min(batch, 14), replace=False)]))
    assert rel_err(y[rows], c.oracle(orc, rows)) <= TOL


# ------------------------------------------------------------------ tensor-core prefill tiles

@pytest.mark.parametrize("m,n,r,batch", [
    (128, 128, 128, 9),       # one M tile, one N tile of 64, ragged
    (256, 384, 256, 64),      # exact N tile of 64
    (384, 256, 384, 65),      # N tile of 128, ragged
    (256, 512, 128, 300),     # three N tiles of 128, ragged tail
    (128, 256, 256, 1025),    # N tiles of 256, one token in the last
    (1408, 640, 896, 517),    # several M tiles in both GEMMs
    (256, 4096, 128, 9),      # split K: one row block in GEMM 1, two in GEMM 2, 9 tokens
    (512, 2048, 384, 40),     # split K with a partial last 16-token group
    (2432, 512, 1280, 64),    # split K in GEMM 1, 19 row blocks in GEMM 2
    (128, 8192, 128, 17),     # one row block each: the most splits
    (128, 512, 128, 300),     # 64-wide token tiles in both GEMMs
    (1024, 256, 896, 3000),   # 144-wide tiles in GEMM 1, 176-wide in GEMM 2 (not multiples of 32)
])
def test_prefill_tiles(nq, orc, m, n, r, batch):
    c = Case(orc, nq, m, n, r, batch, seed=m * 7 + batch)
    y = c.gpu()
    nq.device_status()
    assert rel_err(y, c.oracle(orc)) <= TOL


def test_prefill_split_k_deterministic(nq, orc):
    # few row blocks: K is split over many CTAs and the partials are added in split order
    c = Case(orc, nq, 384, 4096, 256, 16, seed=31)
    a, b = c.gpu(), c.gpu()
    nq.device_status()
    assert np.array_equal(a, b)
    assert rel_err(a, c.oracle(orc)) <= TOL


def test_prefill_deterministic_and_status(nq, orc):
    c = Case(orc, nq, 512, 1024, 384, 200, seed=3)
    a, b = c.gpu(), c.gpu()
    nq.device_status()
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ grouped calls

@pytest.mark.parametrize("batch", [1, 3, 8, 20])
def test_grouped_matches_single_calls(nq, orc, batch):
    """Up to 8 tokens a grouped call gives each layer the bits of its single call.  At 20
    tokens the grouped call of these four small layers runs the decode kernels over token
    chunks (8 + 8 + 4) and a single call the prefill GEMMs: both within the tolerance."""
    shapes = [(512, 512, 128), (384, 640, 256), (1024, 256, 384), (256, 2176, 128)]
    cases = [Case(orc, nq, m, n, r, batch, seed=900 + i) for i, (m, n, r) in enumerate(shapes)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        single = c.gpu()
        if batch <= 8:
            assert np.array_equal(y.cpu().numpy(), single)
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL
        assert rel_err(single, c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [9, 12, 20])
def test_grouped_token_chunks(nq, orc, batch):
    """A grouped call of more than 8 tokens that takes the decode kernels in token chunks
    (the seven Llama-2-7B-shaped layers, 9 to 20 tokens): every output within the tolerance
    of the oracle, and each chunk's rows the bits of a grouped call on those tokens alone."""
    cases = [Case(orc, nq, m, n, r, batch, seed=2960 + 10 * batch + i)
             for i, (_, m, n, r) in enumerate(synth.LLAMA2_7B_LAYERS)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    parts = []
    for b0 in range(0, batch, 8):
        b1 = min(batch, b0 + 8)
        yp = [torch.empty((b1 - b0, c.m), dtype=torch.float32, device="cuda") for c in cases]
        nq.lowrank_linear_fwd_grouped([(c.x_d[b0:b1], c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                       for c, y in zip(cases, yp)], b1 - b0)
        parts.append(yp)
    torch.cuda.synchronize()
    for i, (c, y) in enumerate(zip(cases, ys)):
        got = y.cpu().numpy()
        assert rel_err(got, c.oracle(orc)) <= TOL, i
        assert np.array_equal(got, np.concatenate([p[i].cpu().numpy() for p in parts])), i


def test_grouped_more_than_one_launch(nq, orc):
    batch = 2
    cases = [Case(orc, nq, 256, 256, 128, batch, seed=950 + i) for i in range(19)]
    ys = [torch.empty((batch, 256), dtype=torch.float32, device="cuda") for _ in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [1, 8])
def test_grouped_llama2_7b_block(nq, orc, batch):
    """The benchmark's decode step: the seven Llama-2-7B-shaped layers in one grouped call
    (the launch configuration bench.py times), every output checked."""
    cases = [Case(orc, nq, m, n, r, batch, seed=960 + i) for i, (_, m, n, r) in enumerate(synth.LLAMA2_7B_LAYERS)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [2, 3, 5])
def test_grouped_llama2_7b_block_other_batches(nq, orc, batch):
    """The seven-layer decode step at the batch sizes between the benchmarked ones: one
    token group with two and three tokens (one wave of the balanced stage-2 plan), and the
    first batch that needs two token groups."""
    cases = [Case(orc, nq, m, n, r, batch, seed=1960 + 10 * batch + i)
             for i, (_, m, n, r) in enumerate(synth.LLAMA2_7B_LAYERS)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [1, 4])
def test_grouped_mixed_sizes(nq, orc, batch):
    """A large layer grouped with small ones: the stage-2 plan gives each small layer a
    single CTA (at least one per layer) and the large one the rest; stage 1 mixes one-split
    and many-split layers."""
    shapes = [(11008, 4096, 2432), (128, 128, 128), (256, 2176, 128), (384, 640, 256)]
    cases = [Case(orc, nq, m, n, r, batch, seed=2900 + i) for i, (m, n, r) in enumerate(shapes)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [1, 2, 3, 4])
def test_grouped_llama2_70b_block(nq, orc, batch):
    """The Llama-2-70B-shaped block in one grouped call (up to 28 column splits per layer,
    a 3840-column stage-2 span), every output checked.  At 2-4 tokens stage 2 streams the
    weights through one persistent CTA per SM, and 256-row units that straddle two CTAs'
    shares are finished by the last of them."""
    cases = [Case(orc, nq, m, n, r, batch, seed=980 + i) for i, (_, m, n, r) in enumerate(synth.LLAMA2_70B_LAYERS)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        assert rel_err(y.cpu().numpy(), c.oracle(orc)) <= TOL


# ------------------------------------------------------------------ failure path

def test_device_wait_timeout_is_reported_and_cleared(nq, orc):
    """A bounded device wait that runs out (a barrier nothing arrives on, 2 ms limit) is
    reported once by nq_device_status as NQ_ERR_TIMEOUT, then cleared, and the context
    keeps working."""
    s = torch.cuda.current_stream().cuda_stream
    assert nq.nq_selftest_wait_timeout(2_000_000, s) == nq.NQ_OK
    assert nq.nq_device_status(s) == nq.NQ_ERR_TIMEOUT
    assert nq.nq_device_status(s) == nq.NQ_OK
    with pytest.raises(nq.NQError):
        nq.nq_selftest_wait_timeout(2_000_000, s)
        nq.device_status(s)
    nq.device_status(s)
    c = Case(orc, nq, 256, 512, 128, 20, seed=5)
    assert rel_err(c.gpu(), c.oracle(orc)) <= TOL
    assert nq.nq_selftest_wait_timeout(10, s) == nq.NQ_ERR_VALUE


@pytest.mark.parametrize("batch", [1, 5, 20])
def test_grouped_host_buffers(nq, orc, batch):
    """Grouped call with x and y in host memory (pinned and pageable mixed, one layer's
    buffers on the device): same bits as the device-buffer call."""
    shapes = [(512, 512, 128), (384, 640, 256), (1024, 256, 384)]
    cases = [Case(orc, nq, m, n, r, batch, seed=950 + i) for i, (m, n, r) in enumerate(shapes)]
    dev_layers, host_layers, host_ys = [], [], []
    for i, c in enumerate(cases):
        y_dev = torch.empty((batch, c.m), dtype=torch.float32, device="cuda")
        dev_layers.append((c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y_dev, c.m, c.n, c.r))
        if i == 2:  # device buffers in a call that also has host ones
            xh, yh = c.x_d, torch.empty((batch, c.m), dtype=torch.float32, device="cuda")
        elif i == 1:  # pageable host memory
            xh = np.ascontiguousarray(c.x)
            yh = np.zeros((batch, c.m), dtype=np.float32)
        else:  # pinned host memory
            xh = torch.from_numpy(c.x.view(np.int16)).pin_memory()
            yh = torch.empty((batch, c.m), dtype=torch.float32).pin_memory()
        host_layers.append((xh, c.Upk, c.Vpk, c.s1_d, c.s2_d, yh, c.m, c.n, c.r))
        host_ys.append(yh)
    nq.lowrank_linear_fwd_grouped(dev_layers, batch)
    nq.lowrank_linear_fwd_grouped(host_layers, batch, stream=torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    for i, c in enumerate(cases):
        want = dev_layers[i][5].cpu().numpy()
        got = host_ys[i].cpu().numpy() if isinstance(host_ys[i], torch.Tensor) else host_ys[i]
        assert np.array_equal(got, want), i
        assert rel_err(got, c.oracle(orc)) <= TOL


@pytest.mark.parametrize("batch", [1, 5, 20])
def test_grouped_pinned_repeated_calls(nq, orc, batch):
    """The same grouped call with pinned host x and y made again and again (the library
    replays such calls from a captured CUDA graph after their first occurrence): every call
    reads the x it is given at that moment, also after the workspace was regrown in between,
    and returns the device-buffer call's bits."""
    shapes = [(512, 512, 128), (384, 640, 256), (1024, 256, 384)]
    cases = [Case(orc, nq, m, n, r, batch, seed=970 + i) for i, (m, n, r) in enumerate(shapes)]
    xh = [torch.empty((batch, c.n), dtype=torch.int16).pin_memory() for c in cases]
    yh = [torch.empty((batch, c.m), dtype=torch.float32).pin_memory() for c in cases]
    host_layers = [(xh[i], c.Upk, c.Vpk, c.s1_d, c.s2_d, yh[i], c.m, c.n, c.r) for i, c in enumerate(cases)]
    for k in range(5):
        if k == 3:  # a call with a larger pinned x grows the staging buffer (a new generation)
            big = Case(orc, nq, 128, 1 << 18, 128, 8, seed=990)
            big_x = torch.from_numpy(big.x.view(np.int16)).pin_memory()
            nq.lowrank_linear_fwd(big_x, big.Upk, big.Vpk, big.s1_d, big.s2_d, big.m, big.n, big.r)
        xs = [synth.activations_bf16(batch, c.n, 1000 + 10 * k + i) for i, c in enumerate(cases)]
        for i in range(len(cases)):
            xh[i].copy_(torch.from_numpy(xs[i].view(np.int16)))
            yh[i].fill_(float("nan"))
        nq.lowrank_linear_fwd_grouped(host_layers, batch)
        dev_ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
        nq.lowrank_linear_fwd_grouped(
            [(torch.from_numpy(xs[i].view(np.int16)).cuda(), c.Upk, c.Vpk, c.s1_d, c.s2_d, dev_ys[i], c.m, c.n, c.r)
             for i, c in enumerate(cases)], batch)
        torch.cuda.synchronize()
        for i, c in enumerate(cases):
            assert np.array_equal(yh[i].numpy(), dev_ys[i].cpu().numpy()), (k, i)
        if k in (0, 4):
            for i, c in enumerate(cases):
                want = orc.lowrank_linear_fwd(xs[i], c.Upk_o, c.Vpk_o, c.s1, c.s2, c.m, c.n, c.r)
                assert rel_err(yh[i].numpy(), want) <= TOL, (k, i)


@pytest.mark.parametrize("batch", [2, 3, 4, 5, 8, 12])
def test_tokens_are_independent(nq, orc, batch):
    """Each token's result does not depend on the other tokens of the call: every row of a
    grouped decode call of 2..12 tokens (one and two token groups, the token-major and the
    column-major fragment builds, one and several stage-2 spans, the stage-2 sum of the
    split partials and the stage-1 hand-off, token chunks above 8) equals, bit for bit, the
    same grouped call on that token alone."""
    shapes = [(512, 512, 128), (384, 640, 256), (11008, 4096, 2432)]
    cases = [Case(orc, nq, m, n, r, batch, seed=3100 + 10 * batch + i) for i, (m, n, r) in enumerate(shapes)]
    ys = [torch.empty((batch, c.m), dtype=torch.float32, device="cuda") for c in cases]
    nq.lowrank_linear_fwd_grouped([(c.x_d, c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                   for c, y in zip(cases, ys)], batch)
    singles = []
    for b in range(batch):
        y1 = [torch.empty((1, c.m), dtype=torch.float32, device="cuda") for c in cases]
        nq.lowrank_linear_fwd_grouped([(c.x_d[b:b + 1], c.Upk, c.Vpk, c.s1_d, c.s2_d, y, c.m, c.n, c.r)
                                       for c, y in zip(cases, y1)], 1)
        singles.append(y1)
    torch.cuda.synchronize()
    for i, (c, y) in enumerate(zip(cases, ys)):
        got = y.cpu().numpy()
        assert np.array_equal(got, np.concatenate([s[i].cpu().numpy() for s in singles])), (i, batch)
        assert rel_err(got, c.oracle(orc)) <= TOL


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs a second GPU to hold foreign device memory")
def test_rejects_another_gpus_memory(nq, orc):
    """Device memory of another GPU (no peer access is assumed) is refused on the host with
    NQ_ERR_PTRKIND, before anything is launched: as weights, as x and as y."""
    c = Case(orc, nq, 512, 512, 128, 1, seed=4100)
    torch.cuda.set_device(0)
    other = {k: v.to("cuda:1") for k, v in dict(x=c.x_d, Upk=c.Upk, s1=c.s1_d).items()}
    y = torch.empty((1, 512), dtype=torch.float32, device="cuda:0")
    y1 = torch.empty((1, 512), dtype=torch.float32, device="cuda:1")
    h = torch.cuda.current_stream(0).cuda_stream
    base = dict(x=c.x_d, Upk=c.Upk, Vpk=c.Vpk, s1=c.s1_d, s2=c.s2_d, y=y)
    for key, val in list(other.items()) + [("y", y1)]:
        a = dict(base, **{key: val})
        st = nq.nq_lowrank_linear_fwd(a["x"].data_ptr(), a["Upk"].data_ptr(), a["Vpk"].data_ptr(), a["s1"].data_ptr(),
                                      a["s2"].data_ptr(), 512, 512, 128, 1, a["y"].data_ptr(), h)
        assert st == nq.NQ_ERR_PTRKIND, key

"""The rank-l envelope variant (nq_lowrank_linear_fwd_envelope) against the fp64 oracle's
envelope forward, through the C ABI: l = 1 bit for bit equal to nq_lowrank_linear_fwd,
l = 2 and 4 within the forward's 2e-3 bar (globally and per token), on decode and
prefill batches and the Llama-2-7B layer shapes."""
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


def errors(y, ref):
    y = np.asarray(y, np.float64)
    d = np.abs(y - ref)
    return float(d.max() / np.abs(ref).max()), float(np.max(d.max(axis=1) / np.abs(ref).max(axis=1)))


class Env:
    def __init__(self, orc, nq, m, n, r, l, batch, seed):
        self.m, self.n, self.r, self.l = m, n, r, l
        U = synth.signs(m, r, seed, "U")
        Vt = np.ascontiguousarray(synth.signs(n, r, seed, "V").T)
        self.a = np.stack([synth.scales_f16(m, seed, "env-a", q) for q in range(l)])
        self.b = np.stack([synth.scales_f16(n, seed, "env-b", q) for q in range(l)])
        self.x = synth.activations_bf16(batch, n, seed)
        self.Upk_o, self.Vpk_o = orc.pack_signs(U), orc.pack_signs(Vt)
        dev = torch.device("cuda")
        self.Upk = nq.pack_signs(torch.from_numpy(U).to(dev))
        self.Vpk = nq.pack_signs(torch.from_numpy(Vt).to(dev))
        self.a_d = torch.from_numpy(self.a.view(np.int16)).to(dev)
        self.b_d = torch.from_numpy(self.b.view(np.int16)).to(dev)
        self.x_d = torch.from_numpy(self.x.view(np.int16)).to(dev)

    def gpu(self, nq):
        y = nq.lowrank_linear_fwd_envelope(self.x_d, self.Upk, self.Vpk, self.a_d, self.b_d, self.m, self.n, self.r)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def oracle(self, orc, rows=None):
        x = self.x if rows is None else np.ascontiguousarray(self.x[rows])
        return orc.lowrank_linear_fwd_envelope(x, self.Upk_o, self.Vpk_o, self.a, self.b, self.m, self.n, self.r)


@pytest.mark.parametrize("batch", [1, 4, 16, 128])
@pytest.mark.parametrize("m,n,r", [(512, 512, 128), (4096, 4096, 1664)])
def test_envelope_rank1_is_the_forward(nq, orc, m, n, r, batch):
    E = Env(orc, nq, m, n, r, 1, batch, seed=5000 + m + batch)
    y = E.gpu(nq)
    plain = nq.lowrank_linear_fwd(E.x_d, E.Upk, E.Vpk, E.a_d[0], E.b_d[0], m, n, r)
    torch.cuda.synchronize()
    assert np.array_equal(y, plain.cpu().numpy())


@pytest.mark.parametrize("l", [2, 4])
@pytest.mark.parametrize("batch", [1, 8, 16, 128])
@pytest.mark.parametrize("m,n,r", [(512, 512, 128), (4096, 4096, 1664), (4096, 11008, 2432), (11008, 4096, 2432)])
def test_envelope_matches_oracle(nq, orc, m, n, r, l, batch):
    E = Env(orc, nq, m, n, r, l, batch, seed=5100 + m + n + l + batch)
    y = E.gpu(nq)
    rows = None if batch <= 16 else np.arange(0, batch, 8)
    ref = E.oracle(orc, rows)
    g, t = errors(y if rows is None else y[rows], ref)
    assert np.all(np.isfinite(y))
    assert g <= TOL and t <= TOL, (g, t)


def test_envelope_repeated_call_and_sixteen_terms(nq, orc):
    """The largest l (16 terms, one decode launch pair) twice in a row: same result both
    times (the terms' scratch is reused) and within the bar."""
    E = Env(orc, nq, 1024, 2048, 256, 16, 3, seed=5200)
    y1 = E.gpu(nq)
    y2 = E.gpu(nq)
    assert np.array_equal(y1, y2)
    g, t = errors(y1, E.oracle(orc))
    assert g <= TOL and t <= TOL


def test_envelope_argument_errors(nq):
    E_m, E_n, E_r = 512, 512, 128
    x = torch.zeros((1, E_n), dtype=torch.int16, device="cuda")
    U = torch.zeros((E_m, E_r // 32), dtype=torch.int32, device="cuda")
    V = torch.zeros((E_r, E_n // 32), dtype=torch.int32, device="cuda")
    a = torch.zeros((17, E_m), dtype=torch.int16, device="cuda")
    b = torch.zeros((17, E_n), dtype=torch.int16, device="cuda")
    y = torch.empty((1, E_m), dtype=torch.float32, device="cuda")
    f = nq.lib().nq_lowrank_linear_fwd_envelope
    h = torch.cuda.current_stream().cuda_stream
    args = (x.data_ptr(), U.data_ptr(), V.data_ptr(), a.data_ptr(), b.data_ptr())
    assert f(*args, 0, E_m, E_n, E_r, 1, y.data_ptr(), h) == nq.NQ_ERR_VALUE
    assert f(*args, 17, E_m, E_n, E_r, 1, y.data_ptr(), h) == nq.NQ_ERR_VALUE
    assert f(*args, 2, E_m, E_n, 100, 1, y.data_ptr(), h) == nq.NQ_ERR_SHAPE
    yh = np.zeros((1, E_m), dtype=np.float32)
    assert f(*args, 2, E_m, E_n, E_r, 1, yh.ctypes.data, h) == nq.NQ_ERR_PTRKIND

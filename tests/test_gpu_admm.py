"""The LB-ADMM initialiser on the GPU (nq_admm_init / nq_admm_iterate / nq_admm_factorize)
against the fp64 oracle (oracle/admm.py), through the C ABI.

Both sides start from the same values: W as bfloat16 (decoded exactly by both), the start
block Omega as fp32, and for the iteration tests the oracle's state rounded to fp32.  The
GPU works in fp32; the tolerance follows from that: the least-squares systems
(F^T F + rho I) have condition numbers below 1 + r / lam (at most ~700 here) and the
Cholesky-QR of the start squares the condition of W Omega, so each step carries relative
errors of ~1e-5..1e-4 of the largest entry; 1e-3 of the largest entry is the bar for every
element.  Signs are a decision taken on such values: they are compared where the entry's
magnitude exceeds that bar, and elsewhere either sign is valid.  Over many iterations the
two trajectories may part at such ties, so long runs are compared by what is unique: the
reconstruction error, within 2 % of the oracle's.
"""
import numpy as np
import pytest

from binary_rank_linear_02_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from binary_rank_linear_02_b200 import nq as mod

    return mod


@pytest.fixture(scope="module")
def adm():
    from oracle import admm

    return admm


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def signs_agree(z_gpu, m_ref, tol=TOL):
    """Signs of z_gpu equal those of m_ref wherever |m_ref| is above tol of its row's max."""
    m_ref = np.asarray(m_ref, np.float64)
    clear = np.abs(m_ref) > tol * np.max(np.abs(m_ref), axis=1, keepdims=True)
    return bool(np.all((np.asarray(z_gpu) >= 0)[clear] == (m_ref >= 0)[clear]))


class Problem:
    def __init__(self, adm, m, n, r, seed, q=1):
        self.m, self.n, self.r, self.q = m, n, r, q
        self.Wbits = synth.weights_bf16(m, n, seed)
        self.W = adm.decode_bf16(self.Wbits)
        self.Om = synth.gaussian_f32(n, r, seed, "omega")
        self.W_d = torch.from_numpy(self.Wbits.view(np.int16)).cuda()
        self.Om_d = torch.from_numpy(self.Om).cuda()


def oracle_start(adm, P):
    A0, B0 = adm.power_iteration_init(P.W, P.Om.astype(np.float64), P.q)
    return adm.start_state(A0, B0)


def gpu_state(nq, P, st):
    """Device state from an oracle state dict (rounded to fp32)."""
    g = nq.AdmmState(P.m, P.n, P.r)
    for name, key in (("A", "A"), ("B", "B"), ("ZA", "ZA"), ("ZB", "ZB"), ("LA", "LA"), ("LB", "LB"),
                      ("sA", "sA"), ("sB", "sB")):
        getattr(g, name).copy_(torch.from_numpy(np.ascontiguousarray(st[key], dtype=np.float32)))
    return g


def host(g):
    return {k: getattr(g, k).cpu().numpy().astype(np.float64) for k in ("A", "B", "ZA", "ZB", "LA", "LB", "sA", "sB")}


@pytest.mark.parametrize("m,n,r,q", [(512, 384, 128, 1), (768, 1024, 256, 0), (1024, 512, 128, 2)])
def test_admm_init_matches_oracle(nq, adm, m, n, r, q):
    P = Problem(adm, m, n, r, seed=11 + m + q, q=q)
    g = host(nq.admm_init(P.W_d, m, n, r, P.Om_d, q))
    torch.cuda.synchronize()
    ref = oracle_start(adm, P)
    for key in ("A", "B", "ZA", "ZB", "sA", "sB"):
        assert rel(g[key], ref[key]) <= TOL, key
    assert np.all(g["LA"] == 0) and np.all(g["LB"] == 0)
    assert signs_agree(g["ZA"], ref["A"]) and signs_agree(g["ZB"], ref["B"])
    # each column pair of the start has equal norms
    assert rel(np.linalg.norm(g["A"], axis=0), np.linalg.norm(g["B"], axis=0)) <= TOL


@pytest.mark.parametrize("m,n,r,lam", [(512, 384, 128, 0.2), (640, 896, 256, 0.05)])
def test_admm_one_iteration_matches_oracle(nq, adm, m, n, r, lam):
    """One iteration from the same fp32 state: the latent factors, projections, duals and
    scales element by element; signs where they are clear."""
    P = Problem(adm, m, n, r, seed=21 + m)
    st = oracle_start(adm, P)
    # two oracle iterations so that the duals are non-zero, then round the state to fp32
    st = adm.admm_step(P.W, adm.admm_step(P.W, st, lam), lam)
    st32 = {k: np.asarray(v, np.float32).astype(np.float64) for k, v in st.items() if k not in ("SA", "SB")}
    g = gpu_state(nq, P, st32)
    nq.admm_iterate(P.W_d, g, 1, lam, 1.0)
    torch.cuda.synchronize()
    out = host(g)
    ref = adm.admm_step(P.W, st32, lam)
    for key in ("A", "B", "ZA", "ZB", "LA", "LB", "sA", "sB"):
        assert rel(out[key], ref[key]) <= TOL, key
    assert signs_agree(out["ZA"], ref["A"] + st32["LA"])
    assert signs_agree(out["ZB"], ref["B"] + st32["LB"])


def test_admm_iterations_track_oracle(nq, adm):
    """Ten iterations with a growing penalty from the same start: the reconstruction error
    of the projected factors within 2 % of the oracle's, and the sign patterns nearly all
    equal (trajectories can part only at near-ties)."""
    m, n, r = 512, 512, 128
    P = Problem(adm, m, n, r, seed=31)
    st = oracle_start(adm, P)
    g = gpu_state(nq, P, {k: v for k, v in st.items() if k not in ("SA", "SB")})
    nq.admm_iterate(P.W_d, g, 10, 0.2, 1.05)
    torch.cuda.synchronize()
    out = host(g)
    lam = 0.2
    for _ in range(10):
        st = adm.admm_step(P.W, st, lam)
        lam *= 1.05
    e_gpu = adm.reconstruction_error(P.W, np.sign(out["ZA"]) + (out["ZA"] == 0), np.sign(out["ZB"]) + (out["ZB"] == 0),
                                     out["sA"], out["sB"])
    e_ref = adm.reconstruction_error(P.W, st["SA"], st["SB"], st["sA"], st["sB"])
    assert abs(e_gpu - e_ref) <= 0.02 * e_ref
    agree = np.mean((out["ZA"] >= 0) == (st["SA"] > 0))
    assert agree >= 0.99


def _unpack(orc, Upk, Vpk, m, n, r):
    U = orc.unpack_signs(Upk.cpu().numpy().view(np.uint32), r)
    Vt = orc.unpack_signs(Vpk.cpu().numpy().view(np.uint32), n)
    return U, np.ascontiguousarray(Vt.T)


@pytest.mark.parametrize("m,n,r", [(512, 512, 128), (1024, 768, 256)])
def test_admm_factorize_against_oracle(nq, adm, orc, m, n, r):
    """The whole initialiser (40 iterations): the stored form reproduces W to within 2 % of
    the oracle's reconstruction error; the reported error equals the one recomputed on
    the host from the stored signs and fp16 scales; the scales are balanced."""
    P = Problem(adm, m, n, r, seed=41 + m)
    Upk, Vpk, s1, s2, err = nq.admm_factorize(P.W_d, m, n, r, P.Om_d, iters=40)
    torch.cuda.synchronize()
    U, V = _unpack(orc, Upk, Vpk, m, n, r)
    f1 = s1.cpu().numpy().view(np.float16).astype(np.float64)
    f2 = s2.cpu().numpy().view(np.float16).astype(np.float64)
    e_host = adm.reconstruction_error(P.W, U, V, f1, f2)
    assert abs(err - e_host) <= 1e-4 * e_host
    Ur, Vr, t1, t2 = adm.factorize(P.W, P.Om.astype(np.float64), 40)
    e_ref = adm.reconstruction_error(P.W, Ur, Vr, t1, t2)
    assert abs(e_host - e_ref) <= 0.02 * e_ref, (e_host, e_ref)
    assert np.all(f1 > 0) and np.all(f2 > 0)
    assert abs(np.sqrt(np.mean(f1 ** 2)) / np.sqrt(np.mean(f2 ** 2)) - 1.0) <= 2e-3


def test_admm_output_drives_the_forward(nq, adm, orc):
    """The stored form feeds nq_lowrank_linear_fwd directly: its output equals the oracle's
    forward of the same packed weights (the forward's 2e-3 bar), and approximates W x as
    well as the factorisation approximates W."""
    m, n, r = 1024, 512, 256
    P = Problem(adm, m, n, r, seed=51)
    Upk, Vpk, s1, s2, err = nq.admm_factorize(P.W_d, m, n, r, P.Om_d, iters=30)
    x = synth.activations_bf16(4, n, 52)
    y = nq.lowrank_linear_fwd(torch.from_numpy(x.view(np.int16)).cuda(), Upk, Vpk, s1, s2, m, n, r)
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)
    ref = orc.lowrank_linear_fwd(x, Upk.cpu().numpy().view(np.uint32), Vpk.cpu().numpy().view(np.uint32),
                                 s1.cpu().numpy().view(np.uint16), s2.cpu().numpy().view(np.uint16), m, n, r)
    assert rel(y, ref) <= 2e-3
    dense = adm.decode_bf16(synth.activations_bf16(4, n, 52)) @ P.W.T
    assert np.linalg.norm(y - dense) / np.linalg.norm(dense) <= 2.0 * err


def test_admm_llama2_7b_q_shape(nq, adm, orc):
    """The Llama-2-7B attention shape, 4096 x 4096 at r = 1664, ten iterations on both
    sides from the same start: reconstruction error within 2 % of the oracle's."""
    m, n, r = 4096, 4096, 1664
    P = Problem(adm, m, n, r, seed=61)
    Upk, Vpk, s1, s2, err = nq.admm_factorize(P.W_d, m, n, r, P.Om_d, iters=10)
    torch.cuda.synchronize()
    Ur, Vr, t1, t2 = adm.factorize(P.W, P.Om.astype(np.float64), 10)
    e_ref = adm.reconstruction_error(P.W, Ur, Vr, t1, t2)
    U, V = _unpack(orc, Upk, Vpk, m, n, r)
    f1 = s1.cpu().numpy().view(np.float16).astype(np.float64)
    f2 = s2.cpu().numpy().view(np.float16).astype(np.float64)
    e_host = adm.reconstruction_error(P.W, U, V, f1, f2)
    assert abs(err - e_host) <= 1e-4 * e_host
    assert abs(e_host - e_ref) <= 0.02 * e_ref, (e_host, e_ref)


def test_admm_zero_matrix_is_reported(nq, adm):
    """W = 0 makes the start block rank 0: the Cholesky pivots are not positive and the
    call returns NQ_ERR_VALUE (no fault, the device stays usable)."""
    m, n, r = 256, 256, 128
    W = torch.zeros((m, n), dtype=torch.int16, device="cuda")
    Om = torch.from_numpy(synth.gaussian_f32(n, r, 71)).cuda()
    st = nq.AdmmState(m, n, r)
    rc = nq.lib().nq_admm_init(W.data_ptr(), m, n, r, Om.data_ptr(), 1, *st.ptrs(),
                                torch.cuda.current_stream().cuda_stream)
    assert rc == nq.NQ_ERR_VALUE
    torch.cuda.synchronize()
    assert torch.zeros(4, device="cuda").sum().item() == 0.0

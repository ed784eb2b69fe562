"""The backward of the layer on the GPU, through the C ABI, against the CPU oracle: the
input gradient (dx = s2 * V U^T (s1 * dy)), the packed-sign transpose it needs, the
gradients with respect to the scale vectors and the straight-through gradients of the factors.

Bar: the transpose bit-exact; dx within max|dx - dx_ref| / max|dx_ref| <= 2e-3, the bar of
the forward pass it is computed with (the same kernels with the factors' roles exchanged).
The oracle computes dx from the forward packings directly, so a transposition mistake on
the device side cannot cancel out.
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


def _words(t):
    return t.cpu().numpy().view(np.uint32)


class Layer:
    """One factorised layer: forward packings made on the device, backward packings by the
    device transpose of them, and the oracle's packings of the same signs."""

    def __init__(self, orc, nq, m, n, r, seed):
        self.m, self.n, self.r = m, n, r
        dev = torch.device("cuda")
        self.U = synth.signs(m, r, seed, "U")
        self.V = synth.signs(n, r, seed, "V")
        self.s1 = synth.scales_f16(m, seed, "s1")
        self.s2 = synth.scales_f16(n, seed, "s2")
        self.Upk_o = orc.pack_signs(self.U)
        self.Vpk_o = orc.pack_signs(np.ascontiguousarray(self.V.T))
        self.Upk = nq.pack_signs(torch.from_numpy(self.U).to(dev))
        self.Vpk = nq.pack_signs(torch.from_numpy(np.ascontiguousarray(self.V.T)).to(dev))
        self.UpkT = nq.transpose_signs(self.Upk, m, r)
        self.VpkT = nq.transpose_signs(self.Vpk, r, n)
        self.s1_d = torch.from_numpy(self.s1.view(np.int16)).to(dev)
        self.s2_d = torch.from_numpy(self.s2.view(np.int16)).to(dev)

    def bwd(self, nq, dy_bits):
        dy = torch.from_numpy(dy_bits.view(np.int16)).cuda()
        dx = nq.lowrank_linear_bwd_input(dy, self.UpkT, self.VpkT, self.s1_d, self.s2_d, self.m, self.n, self.r)
        torch.cuda.synchronize()
        return dx.cpu().numpy()

    def fwd(self, nq, x_bits):
        x = torch.from_numpy(x_bits.view(np.int16)).cuda()
        y = nq.lowrank_linear_fwd(x, self.Upk, self.Vpk, self.s1_d, self.s2_d, self.m, self.n, self.r)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def oracle_bwd(self, orc, dy_bits):
        return orc.lowrank_linear_bwd_input(dy_bits, self.Upk_o, self.Vpk_o, self.s1, self.s2, self.m, self.n, self.r)


@pytest.mark.parametrize("rows,cols", [(70, 45), (1, 100), (129, 3), (128, 2432), (2432, 4096), (4096, 11008)])
def test_transpose_device_bit_exact(nq, orc, rows, cols):
    """Ragged shapes (partial tiles on both axes) and the 7B factor shapes."""
    s = synth.signs(rows, cols, 300 + rows + cols)
    packed = orc.pack_signs(s)
    got = nq.transpose_signs(torch.from_numpy(packed.view(np.int32)).cuda(), rows, cols)
    torch.cuda.synchronize()
    assert np.array_equal(_words(got), orc.transpose_signs(packed, rows, cols))


def test_transpose_twice_is_identity(nq):
    rows, cols = 384, 1664
    p = torch.randint(-(1 << 31), 1 << 31, (rows, cols // 32), dtype=torch.int64, device="cuda").to(torch.int32)
    back = nq.transpose_signs(nq.transpose_signs(p, rows, cols), cols, rows)
    torch.cuda.synchronize()
    assert torch.equal(back, p)


@pytest.mark.parametrize("m,n,r,batch", [
    (512, 512, 128, 1),
    (384, 640, 256, 3),
    (1152, 384, 1664, 8),     # decode path, two token groups
    (4096, 11008, 2432, 1),   # the 7B down projection's shape: dx is 11008 wide
    (11008, 4096, 2432, 2),   # the 7B gate projection's shape
    (640, 384, 256, 16),      # prefill path (tcgen05 GEMMs)
    (1024, 2048, 512, 130),   # prefill with a ragged token tile
])
def test_bwd_input_matches_oracle(nq, orc, m, n, r, batch):
    layer = Layer(orc, nq, m, n, r, seed=400 + m + n + batch)
    dy = synth.activations_bf16(batch, m, 401 + batch, "dy")
    dx = layer.bwd(nq, dy)
    assert dx.shape == (batch, n)
    assert rel_err(dx, layer.oracle_bwd(orc, dy)) <= TOL


def test_bwd_input_adjoint_identity(nq, orc):
    """<y(x), dy> = <x, dx(dy)> holds for the device results to the forward's accuracy."""
    m, n, r, batch = 2048, 1024, 384, 4
    layer = Layer(orc, nq, m, n, r, seed=450)
    x = synth.activations_bf16(batch, n, 451)
    dy = synth.activations_bf16(batch, m, 452, "dy")
    y = layer.fwd(nq, x).astype(np.float64)
    dx = layer.bwd(nq, dy).astype(np.float64)
    lhs = float(np.sum(y * synth.bf16_bits_to_f32(dy)))
    rhs = float(np.sum(synth.bf16_bits_to_f32(x) * dx))
    scale = float(np.sqrt(np.sum(y * y) * np.sum(synth.bf16_bits_to_f32(dy).astype(np.float64) ** 2)))
    assert abs(lhs - rhs) <= TOL * scale


def test_bwd_input_host_buffers(nq, orc):
    """dy and dx in host memory (pinned) take the forward's host-buffer path."""
    m, n, r, batch = 512, 768, 256, 2
    layer = Layer(orc, nq, m, n, r, seed=470)
    dy = synth.activations_bf16(batch, m, 471, "dy")
    dy_h = torch.from_numpy(dy.view(np.int16)).pin_memory()
    dx = nq.lowrank_linear_bwd_input(dy_h, layer.UpkT, layer.VpkT, layer.s1_d, layer.s2_d, m, n, r)
    assert not dx.is_cuda
    assert rel_err(dx.numpy(), layer.oracle_bwd(orc, dy)) <= TOL


ONE_F16 = 0x3C00


@pytest.mark.parametrize("m,n,r,batch", [
    (512, 512, 128, 1),
    (384, 640, 256, 5),       # decode path, two token groups
    (1152, 384, 1664, 8),
    (640, 384, 256, 40),      # prefill path
    (640, 384, 256, 130),     # token sums in three 64-token chunks, the last ragged
    (11008, 4096, 2432, 3),   # the 7B gate projection's shape
])
def test_bwd_scales_match_oracle(nq, orc, m, n, r, batch):
    """ds1 and ds2 against the oracle, within the bound that the accuracy of the layer
    evaluations they are made of gives: |ds1_i - ref| <= 2e-3 sum_b |dy_bi| max|z_b|."""
    layer = Layer(orc, nq, m, n, r, seed=500 + m + batch)
    x = synth.activations_bf16(batch, n, 501 + batch)
    dy = synth.activations_bf16(batch, m, 502 + batch, "dy")
    x_d = torch.from_numpy(x.view(np.int16)).cuda()
    dy_d = torch.from_numpy(dy.view(np.int16)).cuda()
    ds1, ds2 = nq.lowrank_linear_bwd_scales(x_d, dy_d, layer.Upk, layer.Vpk, layer.UpkT, layer.VpkT,
                                            layer.s1_d, layer.s2_d, m, n, r)
    torch.cuda.synchronize()
    ref1, ref2 = orc.lowrank_linear_bwd_scales(x, dy, layer.Upk_o, layer.Vpk_o, layer.s1, layer.s2, m, n, r)
    ones_m = np.full(m, ONE_F16, dtype=np.uint16)
    ones_n = np.full(n, ONE_F16, dtype=np.uint16)
    z = orc.lowrank_linear_fwd(x, layer.Upk_o, layer.Vpk_o, ones_m, layer.s2, m, n, r)
    w = orc.lowrank_linear_bwd_input(dy, layer.Upk_o, layer.Vpk_o, layer.s1, ones_n, m, n, r)
    dyf = np.abs(synth.bf16_bits_to_f32(dy).astype(np.float64))
    xf = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64))
    bound1 = TOL * np.sum(dyf * np.max(np.abs(z), axis=1, keepdims=True), axis=0) + 1e-12
    bound2 = TOL * np.sum(xf * np.max(np.abs(w), axis=1, keepdims=True), axis=0) + 1e-12
    assert np.all(np.abs(ds1.cpu().numpy() - ref1) <= bound1)
    assert np.all(np.abs(ds2.cpu().numpy() - ref2) <= bound2)


@pytest.mark.parametrize("batch", [4, 200])  # one token chunk; four chunks through the prefill GEMMs
def test_bwd_scales_deterministic_and_skippable(nq, orc, batch):
    m, n, r = 512, 768, 256
    layer = Layer(orc, nq, m, n, r, seed=520)
    x_d = torch.from_numpy(synth.activations_bf16(batch, n, 521).view(np.int16)).cuda()
    dy_d = torch.from_numpy(synth.activations_bf16(batch, m, 522, "dy").view(np.int16)).cuda()
    a1, a2 = nq.lowrank_linear_bwd_scales(x_d, dy_d, layer.Upk, layer.Vpk, layer.UpkT, layer.VpkT,
                                          layer.s1_d, layer.s2_d, m, n, r)
    b1, b2 = nq.lowrank_linear_bwd_scales(x_d, dy_d, layer.Upk, layer.Vpk, layer.UpkT, layer.VpkT,
                                          layer.s1_d, layer.s2_d, m, n, r)
    torch.cuda.synchronize()
    assert torch.equal(a1, b1) and torch.equal(a2, b2)
    # ds2 alone (ds1 NULL) gives the same ds2
    only2 = torch.empty((n,), dtype=torch.float32, device="cuda")
    st = nq.nq_lowrank_linear_bwd_scales(x_d.data_ptr(), dy_d.data_ptr(), layer.Upk.data_ptr(), layer.Vpk.data_ptr(),
                                         layer.UpkT.data_ptr(), layer.VpkT.data_ptr(), layer.s1_d.data_ptr(),
                                         layer.s2_d.data_ptr(), m, n, r, batch, 0, only2.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == nq.NQ_OK and torch.equal(only2, a2)



@pytest.mark.parametrize("m,n,r,batch", [
    (512, 512, 128, 1),
    (384, 640, 256, 3),
    (640, 384, 256, 13),      # two launches of the first stage (8 + 5 tokens)
    (1152, 384, 1664, 8),
    (4096, 11008, 2432, 2),   # the 7B down projection's shape
    # calibration-sized batches: t and u from the prefill GEMM, the sums on the tensor cores
    (512, 512, 128, 64),      # the first batch of that route (persistent split-K GEMM for t, u)
    (384, 640, 256, 100),     # tokens padded to 128 in the transposed operands
    (1152, 384, 1664, 257),   # one-tile-per-CTA GEMM for t, u; padded to 320
    (11008, 4096, 2432, 128), # the 7B gate projection's shape
])
def test_bwd_factors_match_oracle(nq, orc, m, n, r, batch):
    """dU and dV against the oracle, within the bound that the accuracy of t and u gives:
    |dU_ik - ref| <= 2e-3 |s1_i| sum_b |dy_bi| max|t_b| (likewise dV)."""
    layer = Layer(orc, nq, m, n, r, seed=600 + m + batch)
    x = synth.activations_bf16(batch, n, 601 + batch)
    dy = synth.activations_bf16(batch, m, 602 + batch, "dy")
    x_d = torch.from_numpy(x.view(np.int16)).cuda()
    dy_d = torch.from_numpy(dy.view(np.int16)).cuda()
    dU, dV = nq.lowrank_linear_bwd_factors(x_d, dy_d, layer.Vpk, layer.UpkT, layer.s1_d, layer.s2_d, m, n, r)
    torch.cuda.synchronize()
    rU, rV = orc.lowrank_linear_bwd_factors(x, dy, layer.Upk_o, layer.Vpk_o, layer.s1, layer.s2, m, n, r)
    t = orc.stage1(x, layer.Vpk_o, layer.s2, n, r)
    u = orc.stage1(dy, orc.transpose_signs(layer.Upk_o, m, r), layer.s1, m, r)
    dyf = np.abs(synth.bf16_bits_to_f32(dy).astype(np.float64))
    xf = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64))
    s1f = np.abs(synth.f16_bits_to_f32(layer.s1).astype(np.float64))
    s2f = np.abs(synth.f16_bits_to_f32(layer.s2).astype(np.float64))
    bU = TOL * s1f * np.sum(dyf * np.max(np.abs(t), axis=1)[:, None], axis=0) + 1e-12
    bV = TOL * s2f * np.sum(xf * np.max(np.abs(u), axis=1)[:, None], axis=0) + 1e-12
    assert np.all(np.abs(dU.cpu().numpy() - rU) <= bU[:, None])
    assert np.all(np.abs(dV.cpu().numpy() - rV) <= bV[:, None])


@pytest.mark.parametrize("batch", [5, 100])  # fp32 token sums; tensor-core token sums
def test_bwd_factors_deterministic_and_skippable(nq, orc, batch):
    m, n, r = 384, 640, 256
    layer = Layer(orc, nq, m, n, r, seed=530)
    x_d = torch.from_numpy(synth.activations_bf16(batch, n, 531).view(np.int16)).cuda()
    dy_d = torch.from_numpy(synth.activations_bf16(batch, m, 532, "dy").view(np.int16)).cuda()
    a1, a2 = nq.lowrank_linear_bwd_factors(x_d, dy_d, layer.Vpk, layer.UpkT, layer.s1_d, layer.s2_d, m, n, r)
    b1, b2 = nq.lowrank_linear_bwd_factors(x_d, dy_d, layer.Vpk, layer.UpkT, layer.s1_d, layer.s2_d, m, n, r)
    torch.cuda.synchronize()
    assert torch.equal(a1, b1) and torch.equal(a2, b2)
    # dV alone (dU NULL) gives the same dV
    only = torch.empty((n, r), dtype=torch.float32, device="cuda")
    st = nq.nq_lowrank_linear_bwd_factors(x_d.data_ptr(), dy_d.data_ptr(), layer.Vpk.data_ptr(),
                                          layer.UpkT.data_ptr(), layer.s1_d.data_ptr(), layer.s2_d.data_ptr(),
                                          m, n, r, batch, 0, only.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == nq.NQ_OK and torch.equal(only, a2)

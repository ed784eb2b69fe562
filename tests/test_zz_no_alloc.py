"""The allocation-free entry point, nq_lowrank_linear_fwd_noalloc, against the regular
nq_lowrank_linear_fwd.

It serves callers that cannot allocate device memory when a layer runs (a memory pool
fixed at start-up, an allocator owned by another framework): its scratch is a fixed
array inside the library.  Two calls in a row with different layers must each match the
regular entry point within the parity tolerance, so the second call is not disturbed by
what the first left in the shared array.  The file is named to be collected last; it
passes alone in a fresh process and after the other tests.
"""
import ctypes

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


def _layer(nq, m, n, r, batch, seed):
    dev = torch.device("cuda")
    U = torch.from_numpy(synth.signs(m, r, seed, "U")).to(dev)
    Vt = torch.from_numpy(np.ascontiguousarray(synth.signs(n, r, seed, "V").T)).to(dev)
    return dict(
        x=torch.from_numpy(synth.activations_bf16(batch, n, seed).view(np.int16)).to(dev),
        Upk=nq.pack_signs(U), Vpk=nq.pack_signs(Vt),
        s1=torch.from_numpy(synth.scales_f16(m, seed, "s1").view(np.int16)).to(dev),
        s2=torch.from_numpy(synth.scales_f16(n, seed, "s2").view(np.int16)).to(dev),
        m=m, n=n, r=r, batch=batch)


def _noalloc(nq, L, y):
    h = torch.cuda.current_stream().cuda_stream
    return nq.nq_lowrank_linear_fwd_noalloc(L["x"].data_ptr(), L["Upk"].data_ptr(), L["Vpk"].data_ptr(),
                                            L["s1"].data_ptr(), L["s2"].data_ptr(), L["m"], L["n"], L["r"],
                                            L["batch"], y.data_ptr(), h)


def test_noalloc_matches_regular_entry_point_on_two_calls(nq):
    layers = [_layer(nq, 4096, 4096, 1664, 1, 71), _layer(nq, 1024, 11008, 2432, 8, 72)]
    outs = []
    for L in layers:
        y = torch.full((L["batch"], L["m"]), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(nq, L, y) == nq.NQ_OK
        outs.append(y)
    torch.cuda.synchronize()
    for L, y in zip(layers, outs):
        ref = nq.lowrank_linear_fwd(L["x"], L["Upk"], L["Vpk"], L["s1"], L["s2"], L["m"], L["n"], L["r"])
        torch.cuda.synchronize()
        a, b = y.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(a))
        assert float(np.max(np.abs(a - b)) / np.max(np.abs(b))) <= TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(nq):
    L = _layer(nq, 512, 512, 128, 1, 73)
    y = torch.empty((9, 512), dtype=torch.float32, device="cuda")
    h = torch.cuda.current_stream().cuda_stream
    args = (L["x"].data_ptr(), L["Upk"].data_ptr(), L["Vpk"].data_ptr(), L["s1"].data_ptr(), L["s2"].data_ptr())
    assert nq.nq_lowrank_linear_fwd_noalloc(*args, 512, 512, 8192, 1, y.data_ptr(), h) == nq.NQ_ERR_NOALLOC_LIMIT
    assert nq.nq_lowrank_linear_fwd_noalloc(*args, 512, 512, 128, 9, y.data_ptr(), h) == nq.NQ_ERR_NOALLOC_LIMIT
    assert "noalloc" in nq.nq_status_string(nq.NQ_ERR_NOALLOC_LIMIT)

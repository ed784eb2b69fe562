"""The allocation-free entry point, nq_lowrank_linear_fwd_noalloc, against the regular
nq_lowrank_linear_fwd and against the CPU oracle.

It serves callers that cannot allocate device memory when a layer runs: an inference
engine that reserved its memory pool at start-up (a later cudaMalloc competes with the
pool and can fail mid-request), or a framework that owns the allocator.  Its scratch is a
fixed array inside the library.  Two calls in a row with different layers must each match
the regular entry point and the oracle within the parity tolerance, so the second call is
not disturbed by what the first left in the shared array; a call at the array's limits
(r = 4096, 8 tokens, the most column splits) must too; and a call must leave the device's
free memory and torch's allocator untouched.  The file is named to be collected last; it
passes alone in a fresh process and after the other tests.
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


def _layer(nq, orc, m, n, r, batch, seed):
    dev = torch.device("cuda")
    U = synth.signs(m, r, seed, "U")
    Vt = np.ascontiguousarray(synth.signs(n, r, seed, "V").T)
    x = synth.activations_bf16(batch, n, seed)
    s1 = synth.scales_f16(m, seed, "s1")
    s2 = synth.scales_f16(n, seed, "s2")
    return dict(
        x=torch.from_numpy(x.view(np.int16)).to(dev),
        Upk=nq.pack_signs(torch.from_numpy(U).to(dev)), Vpk=nq.pack_signs(torch.from_numpy(Vt).to(dev)),
        s1=torch.from_numpy(s1.view(np.int16)).to(dev), s2=torch.from_numpy(s2.view(np.int16)).to(dev),
        m=m, n=n, r=r, batch=batch,
        ref=orc.lowrank_linear_fwd(x, orc.pack_signs(U), orc.pack_signs(Vt), s1, s2, m, n, r))


def _noalloc(nq, L, y):
    h = torch.cuda.current_stream().cuda_stream
    return nq.nq_lowrank_linear_fwd_noalloc(L["x"].data_ptr(), L["Upk"].data_ptr(), L["Vpk"].data_ptr(),
                                            L["s1"].data_ptr(), L["s2"].data_ptr(), L["m"], L["n"], L["r"],
                                            L["batch"], y.data_ptr(), h)


def _rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def _check_two_calls_in_a_row(nq, layers):
    outs = []
    for L in layers:
        y = torch.full((L["batch"], L["m"]), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(nq, L, y) == nq.NQ_OK
        outs.append(y)
    torch.cuda.synchronize()
    for L, y in zip(layers, outs):
        regular = nq.lowrank_linear_fwd(L["x"], L["Upk"], L["Vpk"], L["s1"], L["s2"], L["m"], L["n"], L["r"])
        torch.cuda.synchronize()
        a = y.cpu().numpy()
        assert np.all(np.isfinite(a))
        assert _rel(a, regular.cpu().numpy()) <= TOL
        assert _rel(a, L["ref"]) <= TOL


def test_noalloc_matches_regular_entry_point_on_two_calls(nq, orc):
    _check_two_calls_in_a_row(nq, [_layer(nq, orc, 4096, 4096, 1664, 1, 71),
                                   _layer(nq, orc, 1024, 11008, 2432, 8, 72)])


def test_noalloc_at_its_scratch_limits(nq, orc):
    """r = 4096 and 8 tokens (the array's largest t) on an input wide enough for the
    largest number of column splits the array holds, then a small layer after it."""
    _check_two_calls_in_a_row(nq, [_layer(nq, orc, 1024, 11008, 4096, 8, 74),
                                   _layer(nq, orc, 512, 512, 128, 3, 75)])


def test_noalloc_allocates_nothing(nq, orc):
    """After one warm call, further calls change neither the device's free memory nor
    torch's allocator statistics."""
    L = _layer(nq, orc, 4096, 4096, 1664, 4, 76)
    y = torch.empty((L["batch"], L["m"]), dtype=torch.float32, device="cuda")
    assert _noalloc(nq, L, y) == nq.NQ_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    stats0 = torch.cuda.memory_stats()
    for _ in range(3):
        assert _noalloc(nq, L, y) == nq.NQ_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    stats1 = torch.cuda.memory_stats()
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "allocated_bytes.all.allocated"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    assert _rel(y.cpu().numpy(), L["ref"]) <= TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(nq, orc):
    L = _layer(nq, orc, 512, 512, 128, 1, 73)
    y = torch.empty((9, 512), dtype=torch.float32, device="cuda")
    h = torch.cuda.current_stream().cuda_stream
    args = (L["x"].data_ptr(), L["Upk"].data_ptr(), L["Vpk"].data_ptr(), L["s1"].data_ptr(), L["s2"].data_ptr())
    assert nq.nq_lowrank_linear_fwd_noalloc(*args, 512, 512, 8192, 1, y.data_ptr(), h) == nq.NQ_ERR_NOALLOC_LIMIT
    assert nq.nq_lowrank_linear_fwd_noalloc(*args, 512, 512, 128, 9, y.data_ptr(), h) == nq.NQ_ERR_NOALLOC_LIMIT
    assert "noalloc" in nq.nq_status_string(nq.NQ_ERR_NOALLOC_LIMIT)


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs a second GPU to hold foreign device memory")
def test_noalloc_rejects_another_gpus_memory(nq, orc):
    """Device memory of another GPU is refused on the host, before any launch."""
    L = _layer(nq, orc, 512, 512, 128, 1, 77)
    y_other = torch.empty((1, 512), dtype=torch.float32, device="cuda:1")
    torch.cuda.set_device(0)
    h = torch.cuda.current_stream().cuda_stream
    st = nq.nq_lowrank_linear_fwd_noalloc(L["x"].data_ptr(), L["Upk"].data_ptr(), L["Vpk"].data_ptr(),
                                          L["s1"].data_ptr(), L["s2"].data_ptr(), 512, 512, 128, 1,
                                          y_other.data_ptr(), h)
    assert st == nq.NQ_ERR_PTRKIND

"""The CPU oracle against facts fixed outside it (hand-worked values, closed forms,
invariances, numpy/torch conversions).  CPU only."""
import numpy as np
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, pin):
    pin(orc.default())


def test_bf16_decoder_matches_torch(orc):
    torch = pytest.importorskip("torch")
    bits = np.arange(0, 1 << 16, 3, dtype=np.int64).astype(np.int16)
    vals = torch.from_numpy(bits).view(torch.bfloat16).to(torch.float64).numpy()
    o = orc.default()
    for b, v in zip(bits.view(np.uint16)[::97], vals[::97]):
        if np.isfinite(v):
            assert o.bf16_to_double(int(b)) == v


def test_pack_rejects_out_of_range(orc):
    with pytest.raises(ValueError):
        orc.pack_signs(np.array([[1, 2, -1]], dtype=np.int8))


def test_empty_batch(orc):
    o = orc.default()
    y = o.lowrank_linear_fwd(np.zeros((0, 64), np.uint16), np.zeros((32, 1), np.uint32),
                             np.zeros((32, 2), np.uint32), np.zeros(32, np.uint16),
                             np.zeros(64, np.uint16), 32, 64, 32)
    assert y.shape == (0, 32)

"""Pins for the oracle's gated feed-forward step H = silu(gate) * up.

Checked against what fixes it other than its own formula: the library SiLU (torch, fp64),
the odd-part identity silu(x) - silu(-x) = x, the limits silu(0) = 0 and silu(g) -> g,
fp16 saturation, and one correctly rounded fp16 result.
"""
import numpy as np
import torch


def test_matches_library_silu(orc):
    g = torch.Generator().manual_seed(5)
    GU = (torch.randn(33, 2 * 50, generator=g, dtype=torch.float64) * 6.0)
    H = orc.silu_mul(GU.numpy())
    want = (torch.nn.functional.silu(GU[:, :50]) * GU[:, 50:]).numpy()
    assert H.dtype == np.float16 and H.shape == (33, 50)
    assert np.array_equal(H, want.astype(np.float16))


def test_odd_part_identity(orc):
    x = np.linspace(-30.0, 30.0, 241)
    ones = np.ones_like(x)
    hp = orc.silu_mul(np.stack([np.concatenate([x, ones])]))
    hn = orc.silu_mul(np.stack([np.concatenate([-x, ones])]))
    # silu(x) - silu(-x) = x, up to one fp16 rounding on each side
    d = hp.astype(np.float64) - hn.astype(np.float64)
    assert np.all(np.abs(d - x) <= 2.0 ** -10 * (np.abs(x) + 1.0))


def test_limits_and_saturation(orc):
    GU = np.array([[0.0, 40.0, -40.0, 300.0, 1.0, 2.0, 3.0, 400.0]])
    H = orc.silu_mul(GU).astype(np.float64)[0]
    assert H[0] == 0.0                      # silu(0) = 0
    assert H[1] == 80.0                     # silu(40) = 40 (1 - 4e-18): rounds to 40, times 2
    assert H[2] == 0.0                      # silu(-40) * 3 ~ -5e-16: below fp16's smallest step
    assert H[3] == 65504.0                  # 300 * 400 = 120000 saturates


def test_one_correctly_rounded_value(orc):
    # silu(1) = 1 / (1 + e^-1) = 0.7310585786300049; times 1 -> fp16 0.73095703125
    # (fp16 spacing at 0.73 is 2^-11 = 0.00048828125; 0.7310585786 / 2^-11 = 1497.21 -> 1497)
    H = orc.silu_mul(np.array([[1.0, 1.0]]))
    assert float(H[0, 0]) == 1497 * 2.0 ** -11

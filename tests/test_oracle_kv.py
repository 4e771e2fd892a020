"""Pins of the oracle's KV-cache quantisation (the 4-4-4 setting of the Rotated
Runtime Smooth summary page, "Key results"): each head vector rotated by the
normalised Hadamard transform of its length D, then per-vector symmetric INT4
(scale = max|x| / 7, round half to even).  Checked against a hand-worked vector,
an fp64 rotation from scipy's Hadamard matrix with the quantiser's error bound,
the preservation of attention scores by the rotation, and special cases."""
import numpy as np
import pytest
import scipy.linalg

import oracle


def test_hand_worked_vector():
    # x = [1, 2, 3, 4]: stages h = 1 -> [3, -1, 7, -1]; h = 2 -> [10, -2, -4, 0]; x 1/2 -> [5, -1, -2, 0]
    # amax 5, scale 5/7; codes rint(7 * [5, -1, -2, 0] / 5) = [7, -1, -3, 0] (-1.4 -> -1, -2.8 -> -3)
    codes, q, scale = oracle.kv_quant(np.array([[[1.0, 2.0, 3.0, 4.0]]], np.float32))
    assert codes.tolist() == [[[7, -1, -3, 0]]]
    assert q.tolist() == [[[0xF7, 0x0D]]]          # low nibble = even channel, two's complement
    assert scale.dtype == np.float32 and scale[0, 0] == np.float32(5.0) / np.float32(7.0)
    back = oracle.kv_dequant(q, scale)
    assert np.array_equal(back[0, 0], np.float32([7, -1, -3, 0]) * scale[0, 0])


def _kv(T, H, D, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H, D)).astype(np.float32)
    x[:, :, 3] *= 40.0                              # a channel-wise outlier in every head
    x[T // 2, 1 % H, 7] = 900.0                     # one spike
    return x.astype(np.float16).astype(np.float32)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_error_bound_against_an_fp64_rotation(D):
    x = _kv(24, 4, D, D)
    codes, q, scale = oracle.kv_quant(x)
    Hd = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    rot = x.astype(np.float64) @ Hd.T               # rows of x times H (symmetric)
    amax = np.abs(rot).max(-1)
    # the scale is max|x_rot| / 7 up to the fp32 rounding of the rotation
    assert np.allclose(scale, amax / 7.0, rtol=1e-5, atol=0)
    # every reconstruction error within half a step (plus the fp32 rotation's rounding)
    err = np.abs(rot - codes.astype(np.float64) * scale[..., None])
    assert np.all(err <= scale[..., None] * 0.5 * (1 + 1e-4) + 1e-4 * amax[..., None])
    # the largest element of every vector maps to +-7; -8 is never produced
    assert np.all(np.abs(codes).max(-1) == 7) and codes.min() >= -7


def test_attention_scores_survive_rotation_and_quantisation():
    T, H, D = 32, 2, 128
    k = _kv(T, H, D, 5)
    qv = np.random.default_rng(6).standard_normal((H, D)).astype(np.float32)
    codes, q, scale = oracle.kv_quant(k)
    khat = oracle.kv_dequant(q, scale)               # rotated space
    Hd = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    qrot = qv.astype(np.float64) @ Hd.T
    for h in range(H):
        exact = k[:, h].astype(np.float64) @ qv[h].astype(np.float64)
        approx = khat[:, h].astype(np.float64) @ qrot[h]
        bound = 0.5 * scale[:, h].astype(np.float64) * np.abs(qrot[h]).sum() * (1 + 1e-3) + 1e-3 * np.abs(exact)
        assert np.all(np.abs(approx - exact) <= bound)


def test_zero_vector_and_heads_are_independent():
    x = _kv(5, 3, 128, 9)
    x[2, 1] = 0.0
    codes, q, scale = oracle.kv_quant(x)
    assert scale[2, 1] == 0.0 and not codes[2, 1].any()
    c2, q2, s2 = oracle.kv_quant(x[:, 2:3])
    assert np.array_equal(c2[:, 0], codes[:, 2]) and np.array_equal(s2[:, 0], scale[:, 2])

"""Pins for the CPU oracle against what the pages and mathematics fix.

Every test here checks the oracle against something other than itself: a
closed form (Sylvester Hadamard), a library routine (scipy's Hadamard, numpy
matmul), an identity the pages state (the reorder identity, HH^T = I), a
special case that reduces to a textbook routine (no smoothing = per-token
INT4 RTN), brute force on tiny inputs, or hand-derived values for the readings
the pages leave open (stage order, rounding, packing).
"""
import numpy as np
import pytest
import scipy.linalg

from activation_smoothing_b200 import workloads as wl

F32 = np.float32


def popcount_sign(n):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    bits = np.bitwise_and(i, j)
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


# ---------------------------------------------------------------- Hadamard ---

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_fwht_basis_equals_sylvester_closed_form(orc, n):
    """FWHT(e_i) is row i of H with H[i][j] = (-1)^popcount(i&j), exactly."""
    H = popcount_sign(n)
    for i in range(n):
        e = np.zeros(n, F32)
        e[i] = 1.0
        np.testing.assert_array_equal(orc.fwht(e), H[i].astype(F32))


@pytest.mark.parametrize("n", [2048, 4096, 8192])
def test_fwht_basis_large_sampled(orc, n):
    rng = np.random.default_rng(n)
    for i in list(rng.choice(n, 24, replace=False)) + [0, n - 1]:
        e = np.zeros(n, F32)
        e[i] = 1.0
        j = np.arange(n)
        bits = np.bitwise_and(i, j)
        pc = np.array([bin(b).count("1") for b in bits])
        np.testing.assert_array_equal(orc.fwht(e), np.where(pc % 2 == 0, 1.0, -1.0).astype(F32))


@pytest.mark.parametrize("n", [2, 16, 128, 1024])
def test_fwht_matches_scipy_hadamard(orc, n):
    """The library's Sylvester Hadamard, applied in fp64, agrees within the fp32
    error of log2(n) rounding stages."""
    H = scipy.linalg.hadamard(n).astype(np.float64)
    rng = np.random.default_rng(7)
    x = rng.standard_normal(n).astype(np.float16).astype(F32)
    ref = H @ x.astype(np.float64)
    got = orc.fwht(x).astype(np.float64)
    bound = np.log2(n) * 2.0 ** -24 * np.abs(H) @ np.abs(x.astype(np.float64)) * 2
    assert np.all(np.abs(got - ref) <= bound + 1e-30)


def test_fwht_stage_order_hand_example(orc):
    """Reading R1 fixes the fp32 order: h = 1 stage before h = 2.  For
    x = [1, 2^-24, -1, 2^-24] the h=1 stage rounds 1 + 2^-24 to 1 (tie to even),
    so out[0] = (1 + 2^-24 -> 1) + (-1 + 2^-24) = 2^-24, whereas the exact sum is
    2^-23 and the other stage order gives 2^-23.  out[2] = 1 - (-1 + 2^-24) =
    2 - 2^-24, a tie that rounds to 2."""
    t = F32(2.0 ** -24)
    x = np.array([1.0, t, -1.0, t], F32)
    got = orc.fwht(x)
    want = np.array([2.0 ** -24, -(2.0 ** -24), 2.0, 2.0], F32)
    np.testing.assert_array_equal(got, want)


def test_hadamard_scale_constants(orc):
    assert orc.hadamard_scale(1) == 1.0
    assert orc.hadamard_scale(256) == 2.0 ** -4
    assert orc.hadamard_scale(4096) == 2.0 ** -6
    for n in (2, 2048, 8192):
        assert orc.hadamard_scale(n) == float(F32(1.0 / np.sqrt(np.float64(n))))


@pytest.mark.parametrize("n", [64, 256, 2048])
def test_rotation_orthonormal(orc, n):
    """Normalised Hadamard: R R^T = I within fp32 rounding (HH^T = I)."""
    R = orc.rotate(np.eye(n, dtype=F32), n).astype(np.float64)
    err = np.abs(R @ R.T - np.eye(n)).max()
    assert err <= 4 * 2.0 ** -24


@pytest.mark.parametrize("n", [256, 4096, 8192])
def test_rotation_preserves_norm(orc, n):
    rng = np.random.default_rng(n + 1)
    X = (rng.standard_normal((8, n)) * 3).astype(np.float16)
    R = orc.rotate(X, n).astype(np.float64)
    nx = np.linalg.norm(X.astype(np.float64), axis=1)
    nr = np.linalg.norm(R, axis=1)
    assert np.all(np.abs(nr - nx) <= (np.log2(n) + 2) * 2.0 ** -23 * nx)


def test_block_diagonal_rotation(orc):
    """K = 7 x 2048: each Hadamard block rotates independently and nothing mixes
    across blocks."""
    n, B = 2048, 7
    rng = np.random.default_rng(3)
    X = rng.standard_normal((3, n * B)).astype(np.float16)
    full = orc.rotate(X, n)
    for b in range(B):
        part = orc.rotate(np.ascontiguousarray(X[:, b * n:(b + 1) * n]), n)
        np.testing.assert_array_equal(full[:, b * n:(b + 1) * n], part)
    e = np.zeros((1, n * B), np.float16)
    e[0, 3 * n + 5] = 1
    r = orc.rotate(e, n)
    assert np.all(r[0, :3 * n] == 0) and np.all(r[0, 4 * n:] == 0)
    assert np.all(np.abs(r[0, 3 * n:4 * n]) == F32(orc.hadamard_scale(n)))


def test_no_rotation_is_identity(orc):
    rng = np.random.default_rng(4)
    X = rng.standard_normal((5, 384)).astype(np.float16)
    np.testing.assert_array_equal(orc.rotate(X, 1), X.astype(F32))


def test_rotate_then_reorder_preserves_product(orc):
    """Reorder identity Y = X W^T = sum_i X_i W_i^T with X, W rotated by the same
    orthogonal H and permuted by the same index: the unquantised product is
    unchanged (fp64 product of the fp32 rotated operands)."""
    L = wl.LAYERS["tiny"]
    X = wl.make_activations(L).numpy()
    W = wl.make_weights(L).numpy()
    perm = wl.random_perm(L.K, 11).numpy()
    Xp = orc.reorder(orc.rotate(X, L.had_block), perm).astype(np.float64)
    Wp = orc.reorder(orc.rotate(W, L.had_block), perm).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    got = Xp @ Wp.T
    scale = np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64)).T
    assert np.all(np.abs(got - ref) <= 1e-5 * scale + 1e-12)


def test_reorder_gathers_columns(orc):
    rng = np.random.default_rng(5)
    X = rng.standard_normal((4, 64)).astype(F32)
    perm = rng.permutation(64).astype(np.int32)
    np.testing.assert_array_equal(orc.reorder(X, perm), X[:, perm])
    with pytest.raises(ValueError):
        orc.reorder(X, np.full(64, 64, np.int32))


# ------------------------------------------------------------ group max -----

def test_group_max_brute_force(orc):
    rng = np.random.default_rng(6)
    M, K, G = 5, 24, 8
    Xp = rng.standard_normal((M, K)).astype(F32)
    s = orc.group_max(Xp, G)
    for g in range(K // G):
        m = 0.0
        for t in range(M):
            for j in range(g * G, (g + 1) * G):
                m = max(m, abs(float(Xp[t, j])))
        assert s[g] == F32(m)


def test_group_of_size_K_is_global_max(orc):
    rng = np.random.default_rng(8)
    Xp = rng.standard_normal((7, 256)).astype(F32)
    s = orc.group_max(Xp, 256)
    assert s.shape == (1,) and s[0] == np.abs(Xp).max()


def test_single_token_group_max_is_row_max(orc):
    rng = np.random.default_rng(9)
    Xp = rng.standard_normal((1, 256)).astype(F32)
    s = orc.group_max(Xp, 64)
    np.testing.assert_array_equal(s, np.abs(Xp).reshape(4, 64).max(axis=1))


# -------------------------------------------------- smoothing + quantiser ---

def _xp_tiny(orc, perm=None):
    L = wl.LAYERS["tiny"]
    X = wl.make_activations(L).numpy()
    perm = wl.identity_perm(L.K).numpy() if perm is None else perm
    return orc.reorder(orc.rotate(X, L.had_block), perm), L


def test_smoothed_values_bounded_and_max_token_hits_one(orc):
    Xp, L = _xp_tiny(orc)
    codes, qX, s, st = orc.smooth_quant_from_xp(Xp, L.G)
    d = np.where(s == 0, F32(1), s)
    Xs = (Xp / np.repeat(d, L.G)[None, :]).astype(F32)
    assert np.all(np.abs(Xs) <= 1.0)
    amax = np.abs(Xs).max(axis=1)
    assert amax.max() == F32(1.0)
    np.testing.assert_array_equal(st, (amax / F32(7)).astype(F32))
    assert codes.min() >= -7 and codes.max() <= 7


def test_single_token_scale_is_one_seventh(orc):
    rng = np.random.default_rng(10)
    Xp = rng.standard_normal((1, 256)).astype(F32)
    _, _, _, st = orc.smooth_quant_from_xp(Xp, 128)
    assert st[0] == F32(1.0) / F32(7.0)


def test_unit_scales_is_textbook_per_token_int4_rtn(orc):
    """s = 1 reduces RRS to the A4W4 per-channel (QuaRot-style) scheme: per-token
    symmetric INT4, scale = amax/7, round half to even, clamp [-8, 7]."""
    rng = np.random.default_rng(12)
    Xp = (rng.standard_normal((9, 512)) * rng.uniform(0.1, 30, size=(1, 512))).astype(F32)
    codes, _, s, st = orc.smooth_quant_from_xp(Xp, 128, unit_scales=True)
    assert np.all(s == 1)
    scale = (np.abs(Xp).max(axis=1) / F32(7)).astype(F32)
    ref = np.clip(np.rint((Xp / scale[:, None]).astype(F32)), -8, 7).astype(np.int8)
    np.testing.assert_array_equal(codes, ref)
    np.testing.assert_array_equal(st, scale)


def test_round_half_to_even_and_packing_golden(orc):
    """Hand example for readings R6, R7, R9: with s = 1 the row [7, 2.5, 3.5, -1,
    -2.5, 0, 1, -7] has scale 1 and codes [7, 2, 4, -1, -2, 0, 1, -7];
    packed low nibble first: 0x27, 0xF4, 0x0E, 0x91."""
    Xp = np.array([[7, 2.5, 3.5, -1, -2.5, 0, 1, -7]], F32)
    codes, qX, _, st = orc.smooth_quant_from_xp(Xp, 8, unit_scales=True)
    assert st[0] == 1.0
    np.testing.assert_array_equal(codes[0], np.array([7, 2, 4, -1, -2, 0, 1, -7], np.int8))
    np.testing.assert_array_equal(qX[0], np.array([0x27, 0xF4, 0x0E, 0x91], np.uint8))
    np.testing.assert_array_equal(orc.unpack(qX, 8), codes)


def test_zero_group_and_zero_token(orc):
    rng = np.random.default_rng(13)
    Xp = rng.standard_normal((4, 256)).astype(F32)
    Xp[:, 128:] = 0          # a group that is zero for every token
    Xp[2, :] = 0             # a token that is zero everywhere
    codes, qX, s, st = orc.smooth_quant_from_xp(Xp, 128)
    assert s[1] == 0 and st[2] == 0
    assert np.all(codes[:, 128:] == 0) and np.all(codes[2] == 0)
    assert np.all(qX[2] == 0)


def test_victim_effect_of_channel_wise_smoothing(orc):
    """Channel-wise smoothing (G = 1, no rotation) zeroes the small elements of a
    channel that holds a spike (rebuttal, Figure 1(c)); the rotation spreads the
    spike and the same elements survive."""
    rng = np.random.default_rng(14)
    M, K = 16, 256
    X = rng.standard_normal((M, K)).astype(np.float16)
    X[3, 40] = 1000.0
    ident = np.arange(K, dtype=np.int32)
    codes_rs, _, _, _ = orc.smooth_quant(X, 1, 1, ident)
    small = [t for t in range(M) if t != 3]
    assert np.all(codes_rs[small, 40] == 0)
    codes_rrs, _, _, _ = orc.smooth_quant(X, 1, 256, ident)
    assert np.count_nonzero(codes_rrs[small]) > 0.5 * len(small) * K


# ----------------------------------------------------------------- GEMM -----

def test_group_partials_brute_force(orc):
    rng = np.random.default_rng(15)
    M, N, K, G = 6, 5, 64, 16
    cx = rng.integers(-8, 8, size=(M, K)).astype(np.int8)
    cw = rng.integers(-8, 8, size=(N, K)).astype(np.int8)

    def pack(c):
        u = (c.astype(np.int16) & 0xF).astype(np.uint8)
        return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)

    qX, qW = pack(cx), pack(cw)
    np.testing.assert_array_equal(orc.unpack(qX, K), cx)
    P = orc.group_partials(qX, qW, G)
    for g in range(K // G):
        ref = cx[:, g * G:(g + 1) * G].astype(np.int64) @ cw[:, g * G:(g + 1) * G].astype(np.int64).T
        np.testing.assert_array_equal(P[g], ref)
    rows = [4, 1]
    Pr = orc.group_partials(qX, qW, G, rows=rows)
    np.testing.assert_array_equal(Pr, P[:, rows, :])


def test_linear_equals_group_scaled_sum(orc):
    rng = np.random.default_rng(16)
    M, N, K, G = 4, 6, 256, 64
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = rng.uniform(0.1, 50, K // G).astype(F32)
    st = rng.uniform(1e-3, 1, M).astype(F32)
    sw = rng.uniform(1e-3, 1, N).astype(F32)
    Y, B = orc.linear_rows(qX, s, st, qW, sw, G)
    cx = orc.unpack(qX, K).astype(np.float64).reshape(M, K // G, G)
    cw = orc.unpack(qW, K).astype(np.float64).reshape(N, K // G, G)
    P = np.einsum("mgk,ngk->gmn", cx, cw)
    ref = np.einsum("g,gmn->mn", s.astype(np.float64), P) * st[:, None] * sw[None, :]
    np.testing.assert_allclose(Y, ref.astype(F32), rtol=1e-6)
    assert np.all(B >= np.abs(ref) - 1e-9)


def test_end_to_end_tracks_unquantised_product(orc):
    """RRS W4A4 output stays close to the fp64 X W^T on the tiny workload."""
    L = wl.LAYERS["tiny"]
    X = wl.make_activations(L).numpy()
    W = wl.make_weights(L).numpy()
    perm = orc.calibrate_perm(wl.make_activations(L, sample=1).numpy(), L.had_block)
    _, qX, s, st = orc.smooth_quant(X, L.G, L.had_block, perm)
    _, qW, sw = orc.prepare_weights(W, L.had_block, perm)
    Y, _ = orc.linear_rows(qX, s, st, qW, sw, L.G)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert rel < 0.25


def test_rotation_beats_plain_runtime_smooth_on_spikes(orc):
    """Summary page, 'Surprising findings': with G = 128 and spike outliers, plain
    Runtime Smooth degrades while RRS does not (output error, synthetic data)."""
    L = wl.Layer("spiky", 64, 1024, 128, 128, 1024, seed=77)
    X = wl.make_activations(L).numpy()
    X[5, :] *= 1  # keep shape
    X[5, 17] = 3000.0
    X[40, 900] = -2500.0
    W = wl.make_weights(L).numpy()
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    errs = {}
    for n in (1, 1024):
        perm = orc.calibrate_perm(X, n)
        _, qX, s, st = orc.smooth_quant(X, L.G, n, perm)
        _, qW, sw = orc.prepare_weights(W, n, perm)
        Y, _ = orc.linear_rows(qX, s, st, qW, sw, L.G)
        errs[n] = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert errs[1024] < errs[1]


def test_calibrate_perm_sorts_descending_stable(orc):
    rng = np.random.default_rng(17)
    X = rng.standard_normal((32, 256)).astype(np.float16)
    perm = orc.calibrate_perm(X, 256)
    c = orc.channel_absmax(X, 256)
    assert sorted(perm.tolist()) == list(range(256))
    assert np.all(np.diff(c[perm]) <= 0)
    np.testing.assert_array_equal(c, np.abs(orc.rotate(X, 256)).max(axis=0))
    Xz = np.zeros((4, 64), np.float16)
    np.testing.assert_array_equal(orc.calibrate_perm(Xz, 1), np.arange(64))


def test_weights_use_same_path_as_tokens(orc):
    """Weights: rotation + reorder as activations, per-row scale amax/7, no s."""
    L = wl.LAYERS["tiny"]
    W = wl.make_weights(L).numpy()
    perm = wl.random_perm(L.K, 3).numpy()
    codes, qW, sw = orc.prepare_weights(W, L.had_block, perm)
    Wp = orc.reorder(orc.rotate(W, L.had_block), perm)
    scale = (np.abs(Wp).max(axis=1) / F32(7)).astype(F32)
    np.testing.assert_array_equal(sw, scale)
    ref = np.clip(np.rint((Wp / scale[:, None]).astype(F32)), -8, 7).astype(np.int8)
    np.testing.assert_array_equal(codes, ref)
    np.testing.assert_array_equal(orc.unpack(qW, L.K), codes)

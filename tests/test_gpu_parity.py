"""Parity of the CUDA path with the CPU oracle (needs a B200).

Integer stages (codes/bytes of qX and qW, s, scale_t, scale_w, per-group
int32 partials) must match bit for bit; Y must satisfy, per element,
|dY| <= 1e-3 |Y_oracle| + 2^-20 sum_g |s_g P_g| scale_t scale_w.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_smoothing_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def rrs():
    import activation_smoothing_b200 as m
    m.lib()
    return m


def bits(t):
    a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_bits_equal(gpu, orc, what):
    g = bits(gpu)
    o = bits(orc)
    assert g.shape == o.shape, what
    bad = np.nonzero(g != o)
    assert bad[0].size == 0, f"{what}: {bad[0].size} mismatches, first at {[b[0] for b in bad]}"


def min_workspace(M, K):
    """The smallest workspace rrs_w4a4_gemm accepts: header + int8 operand, no room to split k."""
    return torch.zeros(256 + (M * K + 255) // 256 * 256, dtype=torch.uint8, device=DEV)


def run_layer(rrs, X, W, perm, G, n, flags=0, rows=None, check_y=True, pool=False):
    """Runs the CUDA path and the oracle on the same inputs and compares (Y on the
    listed rows, or every row; pool=True computes the oracle's rows in worker processes)."""
    K = X.shape[1]
    unit = bool(flags & rrs.FORCE_UNIT_SCALES)
    n_eff = 1 if flags & rrs.NO_ROTATE else n
    Xd, Wd, pd = X.to(DEV), W.to(DEV), perm.to(DEV)
    qW, sw = rrs.prepare_weights(Wd, pd, n, flags)
    qX, s, st = rrs.smooth_quant(Xd, pd, G, n, flags)
    ws = rrs.make_workspace(X.shape[0], W.shape[0], K, G, n, flags)
    Y = rrs.w4a4_gemm(qX, s, st, qW, sw, G, ws=ws)
    # the expanded-weight (fp8) kernel computes the same exact partials and the same
    # fp32 promotion in the same order as the packed kernel when that one does not
    # split k (a workspace with no room for partial sums): its Y must be bit-identical
    qW8 = rrs.expand_weights(qW)
    Y8 = rrs.w4a4_gemm(qX, s, st, qW8, sw, G, ws=ws, flags=rrs.W_EXPANDED)
    Y1 = rrs.w4a4_gemm(qX, s, st, qW, sw, G, ws=min_workspace(X.shape[0], K))
    rrs.check_workspace(ws)
    torch.cuda.synchronize()
    assert_bits_equal(Y8, Y1, "Y (expanded weights) vs Y (packed weights, unsplit)")

    _, oqX, os_, ost = oracle.smooth_quant(X, G, n_eff, perm.numpy(), unit_scales=unit)
    assert_bits_equal(s, os_, "s")
    assert_bits_equal(st, ost, "scale_t")
    assert_bits_equal(qX, oqX, "qX")
    _, oqW, osw = oracle.prepare_weights(W, n_eff, perm.numpy())
    assert_bits_equal(sw, osw, "scale_w")
    assert_bits_equal(qW, oqW, "qW")
    if check_y:
        if pool and rows is None:
            from _oracle_pool import linear_rows_all
            Yo, B = linear_rows_all(oqX, os_, ost, oqW, osw, G)
        else:
            Yo, B = oracle.linear_rows(oqX, os_, ost, oqW, osw, G, rows=rows)
        for Yt, what in ((Y, "Y"), (Y8, "Y (expanded weights)")):
            Yg = Yt.cpu().numpy() if rows is None else Yt.cpu().numpy()[rows]
            ok = oracle.y_tolerance_ok(Yg, Yo, B)
            assert ok.all(), f"{what}: {np.count_nonzero(~ok)} of {ok.size} outside tolerance"
            rel = np.linalg.norm(Yg - Yo) / max(np.linalg.norm(Yo), 1e-30)
            assert rel < 1e-5
    return dict(qX=qX, s=s, st=st, qW=qW, sw=sw, Y=Y)


# ------------------------------------------------------------------ tiny ---

@pytest.mark.parametrize("perm_kind", ["identity", "calibrated", "random"])
def test_tiny_full_parity(rrs, perm_kind):
    L = wl.LAYERS["tiny"]
    X, W = wl.make_activations(L), wl.make_weights(L)
    if perm_kind == "identity":
        perm = wl.identity_perm(L.K)
    elif perm_kind == "random":
        perm = wl.random_perm(L.K, 5)
    else:
        perm = torch.from_numpy(oracle.calibrate_perm(wl.make_activations(L, sample=1), L.had_block))
    run_layer(rrs, X, W, perm, L.G, L.had_block)


def test_tiny_partials_bit_exact(rrs):
    L = wl.LAYERS["tiny"]
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = wl.random_perm(L.K, 9)
    _, oqX, _, _ = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    _, oqW, _ = oracle.prepare_weights(W, L.had_block, perm.numpy())
    P = rrs.w4a4_gemm_debug_partials(torch.from_numpy(oqX).to(DEV), torch.from_numpy(oqW).to(DEV), L.G)
    assert_bits_equal(P, oracle.group_partials(oqX, oqW, L.G), "P_g")


# e4m3 bytes of the codes -8..7: sign, 4 exponent bits (bias 7), 3 mantissa bits
# (OCP FP8 e4m3 format), written out by hand from the format's definition.
E4M3_OF_CODE = {-8: 0xD0, -7: 0xCE, -6: 0xCC, -5: 0xCA, -4: 0xC8, -3: 0xC4, -2: 0xC0, -1: 0xB8,
                0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48, 5: 0x4A, 6: 0x4C, 7: 0x4E}


def expanded_operand(q_packed: np.ndarray) -> np.ndarray:
    """The codes one per byte as e4m3, natural k order (from the oracle's packed codes)."""
    N, K2 = q_packed.shape
    codes = oracle.unpack(q_packed, 2 * K2).astype(np.int32)          # [N, K] natural k order
    lut = np.array([E4M3_OF_CODE[c] for c in range(-8, 8)], dtype=np.uint8)
    return lut[codes + 8]


def test_e4m3_table_decodes_to_the_codes():
    """The hand-written e4m3 table decodes (by torch's fp8 type) to the integer codes."""
    b = torch.tensor([E4M3_OF_CODE[c] for c in range(-8, 8)], dtype=torch.uint8)
    assert b.view(torch.float8_e4m3fn).float().tolist() == [float(c) for c in range(-8, 8)]


def test_expand_weights_operand_bit_exact(rrs):
    L = wl.LAYERS["tiny"]
    W = wl.make_weights(L)
    perm = wl.random_perm(L.K, 3)
    _, oqW, _ = oracle.prepare_weights(W, L.had_block, perm.numpy())
    qW8 = rrs.expand_weights(torch.from_numpy(oqW).to(DEV))
    assert_bits_equal(qW8.view(torch.uint8), expanded_operand(oqW), "qW8")
    # every code pattern: all 256 packed bytes in one row
    allb = np.tile(np.arange(256, dtype=np.uint8), (4, 1))
    assert_bits_equal(rrs.expand_weights(torch.from_numpy(allb).to(DEV)).view(torch.uint8),
                      expanded_operand(allb), "qW8 (all byte values)")


@pytest.mark.parametrize("M,N,K,G", [(130, 520, 1024, 128), (257, 136, 512, 256)])
def test_partials_bit_exact_expanded_weights(rrs, M, N, K, G):
    rng = np.random.default_rng(M + N)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    qW8 = rrs.expand_weights(torch.from_numpy(qW).to(DEV))
    P = rrs.w4a4_gemm_debug_partials(torch.from_numpy(qX).to(DEV), qW8, G, flags=rrs.W_EXPANDED)
    assert_bits_equal(P, oracle.group_partials(qX, qW, G), "P_g (expanded weights)")


# Shapes with at least 74 tiles of 256 x 256 take the CTA-pair kernel of the fp8
# GEMM; ragged M and N (not multiples of 256) exercise its edge tiles.
# 256 x 256 CTA-pair tiles (the first three) and 256 x 128 pair tiles (the last three,
# narrow N: k/v-like), with ragged edges
PAIR_SHAPES = [(300, 19016, 384, 128), (512, 18944, 512, 256), (260, 20480, 256, 256),
               (2048, 1024, 512, 128), (1900, 1000, 384, 128), (2100, 1200, 256, 256)]


@pytest.mark.parametrize("M,N,K,G", PAIR_SHAPES)
def test_pair_tiles_partials_bit_exact(rrs, M, N, K, G):
    rng = np.random.default_rng(M * 3 + N)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    qW8 = rrs.expand_weights(torch.from_numpy(qW).to(DEV))
    P = rrs.w4a4_gemm_debug_partials(torch.from_numpy(qX).to(DEV), qW8, G, flags=rrs.W_EXPANDED)
    assert_bits_equal(P, oracle.group_partials(qX, qW, G), "P_g (CTA-pair tiles)")


@pytest.mark.parametrize("M,N,K,G", PAIR_SHAPES)
def test_pair_tiles_y_matches_oracle_and_packed_kernel(rrs, M, N, K, G):
    rng = np.random.default_rng(M + 7 * N)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = (rng.random(K // G, dtype=np.float32) + 0.5).astype(np.float32)
    st = rng.random(M, dtype=np.float32)
    sw = rng.random(N, dtype=np.float32)
    qXd, sd, std, qWd, swd = (torch.from_numpy(a).to(DEV) for a in (qX, s, st, qW, sw))
    Y8 = rrs.w4a4_gemm(qXd, sd, std, rrs.expand_weights(qWd), swd, G, flags=rrs.W_EXPANDED)
    Y = rrs.w4a4_gemm(qXd, sd, std, qWd, swd, G)
    Yb = rrs.w4a4_gemm(qXd, sd, std, rrs.expand_weights(qWd), swd, G, flags=rrs.W_EXPANDED,
                       Y=torch.empty((M, N), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert_bits_equal(Y8, Y, "Y (CTA-pair fp8 tiles) vs Y (packed kernel)")
    assert torch.equal(Yb, Y8.to(torch.bfloat16)), "bf16 Y is the fp32 Y rounded"
    rows = np.unique(np.concatenate([np.arange(4), np.arange(M - 4, M), rng.integers(0, M, 8)]))
    Yo, B = oracle.linear_rows(qX, s, st, qW, sw, G, rows=rows)
    ok = oracle.y_tolerance_ok(Y8.cpu().numpy()[rows], Yo, B)
    assert ok.all(), f"{np.count_nonzero(~ok)} outside tolerance"


@pytest.mark.parametrize("M,N", [(130, 520), (67, 200)])
def test_y_not_32_byte_aligned_matches(rrs, M, N):
    """A Y that is 16- but not 32-byte aligned takes the scalar store path: same values."""
    K, G = 512, 128
    rng = np.random.default_rng(M)
    qX = torch.from_numpy(rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)).to(DEV)
    qW = torch.from_numpy(rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)).to(DEV)
    s = torch.rand(K // G, device=DEV) + 0.5
    st = torch.rand(M, device=DEV)
    sw = torch.rand(N, device=DEV)
    Y = rrs.w4a4_gemm(qX, s, st, qW, sw, G)
    big = torch.zeros(M * N + 8, dtype=torch.float32, device=DEV)
    Yoff = big[4:4 + M * N].view(M, N)
    assert Yoff.data_ptr() % 32 == 16
    rrs.w4a4_gemm(qX, s, st, qW, sw, G, Y=Yoff)
    torch.cuda.synchronize()
    assert_bits_equal(Yoff, Y, "Y at a 16-byte offset")
    assert torch.all(big[:4] == 0) and torch.all(big[4 + M * N:] == 0)


@pytest.mark.parametrize("M,N,K", [(1, 8192, 8192), (16, 2048, 28672), (8, 1000, 4096)])
def test_split_k_for_small_m(rrs, M, N, K):
    """Token counts up to 16 split k across CTAs when the workspace has room: Y within the
    tolerance of the oracle and of the unsplit kernel (a workspace sized without room)."""
    G = 128
    rng = np.random.default_rng(M * 7 + K)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = (rng.random(K // G, dtype=np.float32) + 0.5).astype(np.float32)
    st = rng.random(M, dtype=np.float32)
    sw = rng.random(N, dtype=np.float32)
    args = [torch.from_numpy(a).to(DEV) for a in (qX, s, st, qW, sw)]
    big = rrs.workspace_size(M, N, K, G, 1)
    small = rrs.workspace_size(M, 0, K, G, 1)
    assert big > small
    Y_split = rrs.w4a4_gemm(*args, G, ws=rrs.make_workspace(M, N, K, G, 1))
    Y_one = rrs.w4a4_gemm(*args, G, ws=rrs.make_workspace(M, 0, K, G, 1))
    torch.cuda.synchronize()
    Yo, B = oracle.linear_rows(qX, s, st, qW, sw, G)
    for Y in (Y_split, Y_one):
        ok = oracle.y_tolerance_ok(Y.cpu().numpy(), Yo, B)
        assert ok.all(), f"{np.count_nonzero(~ok)} outside tolerance"
    d = (Y_split - Y_one).abs().max().item()
    assert d <= 1e-5 * Y_one.abs().max().item()


@pytest.mark.parametrize("M,N,K,G", [(4, 3000, 8192, 512), (16, 1536, 4096, 1024), (2, 704, 16384, 8192)])
def test_split_k_group_sizes_and_expanded_weights(rrs, M, N, K, G):
    """Split k with groups wider than one k-block (and G > 4096, promoted in 4096-wide
    pieces), for packed and expanded weights: both within the oracle's tolerance and
    bit-identical to each other (same kernels, same split)."""
    rng = np.random.default_rng(M + N + G)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = (rng.random(K // G, dtype=np.float32) + 0.5).astype(np.float32)
    st = rng.random(M, dtype=np.float32)
    sw = rng.random(N, dtype=np.float32)
    qXd, sd, std, qWd, swd = (torch.from_numpy(a).to(DEV) for a in (qX, s, st, qW, sw))
    ws = rrs.make_workspace(M, N, K, G, 1)
    Y = rrs.w4a4_gemm(qXd, sd, std, qWd, swd, G, ws=ws)
    Y1 = rrs.w4a4_gemm(qXd, sd, std, qWd, swd, G, ws=min_workspace(M, K))   # no split
    Y8 = rrs.w4a4_gemm(qXd, sd, std, rrs.expand_weights(qWd), swd, G, ws=ws, flags=rrs.W_EXPANDED)
    torch.cuda.synchronize()
    # the fp8 kernel does not split k: same promotion order as the unsplit packed kernel
    assert_bits_equal(Y8, Y1, "Y (expanded) vs Y (packed, unsplit)")
    Yo, B = oracle.linear_rows(qX, s, st, qW, sw, G)
    for Yg in (Y, Y8):
        ok = oracle.y_tolerance_ok(Yg.cpu().numpy(), Yo, B)
        assert ok.all(), f"{np.count_nonzero(~ok)} outside tolerance"


@pytest.mark.parametrize("M,K,G,n,flags", [(1, 2048, 128, 2048, 0), (3, 4096, 256, 4096, 0), (16, 8192, 128, 8192, 0),
                                            (5, 14336, 128, 2048, 0), (2, 4096, 128, 4096, 1), (4, 2048, 512, 1024, 2),
                                            (16, 2048, 2048, 2048, 0)])
def test_activation_path_small_m_repeated_calls(rrs, M, K, G, n, flags):
    """Decode-sized token counts on the fast activation path: codes, s and scale_t
    bit-exact with the oracle, over repeated calls on one workspace with different M."""
    L = wl.Layer("small", M, K, 256, G, n, seed=M * 31 + K)
    unit = bool(flags & rrs.FORCE_UNIT_SCALES)
    n_eff = 1 if flags & rrs.NO_ROTATE else n
    perm = wl.random_perm(K, M)
    ws = rrs.make_workspace(16, 256, K, G, n, flags)
    for rep, m in enumerate((M, max(1, M // 2), M)):
        X = wl.make_activations(L, sample=rep, M=m)
        qX, s, st = rrs.smooth_quant(X.to(DEV), perm.to(DEV), G, n, flags, ws=ws)
        rrs.check_workspace(ws)
        _, oqX, os_, ost = oracle.smooth_quant(X, G, n_eff, perm.numpy(), unit_scales=unit)
        assert_bits_equal(s, os_, f"s (call {rep}, M={m})")
        assert_bits_equal(st, ost, f"scale_t (call {rep}, M={m})")
        assert_bits_equal(qX, oqX, f"qX (call {rep}, M={m})")


@pytest.mark.parametrize("M,N,K", [(2048, 4096, 4096), (130, 520, 1024), (8, 2048, 8192), (33, 200, 512), (17, 203, 1024)])
def test_bf16_output_is_rounded_fp32(rrs, M, N, K):
    """RRS_Y_BF16: Y in bf16 equals the fp32 Y rounded to nearest even, bit for bit, on the
    prefill kernel, the split-k path (M <= 16), ragged N and through rrs_linear."""
    G = 128
    L = wl.Layer("bf16", M, K, N, G, K if K <= 8192 else 2048, seed=M + N)
    X, W = wl.make_activations(L).to(DEV), wl.make_weights(L).to(DEV)
    perm = wl.random_perm(K, 3).to(DEV)
    qW, sw = rrs.prepare_weights(W, perm, L.had_block)
    ws = rrs.make_workspace(M, N, K, G, L.had_block)
    Y32 = rrs.linear(X, qW, sw, perm, G, L.had_block, ws=ws)
    Y16 = rrs.linear(X, qW, sw, perm, G, L.had_block, ws=ws,
                     Y=torch.empty((M, N), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert Y16.dtype == torch.bfloat16
    assert_bits_equal(Y16.view(torch.int16), Y32.to(torch.bfloat16).view(torch.int16), "bf16 Y")


def test_partials_extreme_codes(rrs):
    """All codes -8 or 7 (|P_g| at its maximum 64 G) stay exact."""
    rng = np.random.default_rng(1)
    M, N, K, G = 130, 136, 512, 256
    qX = rng.choice(np.array([0x88, 0x77, 0x87, 0x78], np.uint8), size=(M, K // 2))
    qW = rng.choice(np.array([0x88, 0x77], np.uint8), size=(N, K // 2))
    qX[3, :] = 0x88
    qW[5, :] = 0x88
    P = rrs.w4a4_gemm_debug_partials(torch.from_numpy(qX).to(DEV), torch.from_numpy(qW).to(DEV), G)
    Po = oracle.group_partials(qX, qW, G)
    assert Po[0, 3, 5] == 64 * G
    assert_bits_equal(P, Po, "P_g extreme")


def test_tiny_plain_runtime_smooth_and_unit_scales(rrs):
    L = wl.LAYERS["tiny"]
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = wl.random_perm(L.K, 2)
    run_layer(rrs, X, W, perm, L.G, L.had_block, flags=rrs.NO_ROTATE)
    run_layer(rrs, X, W, perm, L.G, 1)
    r = run_layer(rrs, X, W, perm, L.G, L.had_block, flags=rrs.FORCE_UNIT_SCALES)
    assert torch.all(r["s"] == 1)


# ------------------------------------------------------------ edge cases ---

@pytest.mark.parametrize("M,N,K,G,n", [
    (1, 256, 256, 128, 256),
    (17, 136, 512, 128, 64),
    (130, 200, 1024, 256, 1024),
    (257, 384, 2048, 2048, 2048),       # one group (G = K)
    (64, 128, 384, 128, 128),           # K not a power of two, 3 Hadamard blocks
    (33, 520, 4096, 512, 1),            # no rotation, ragged N
])
def test_edge_shapes(rrs, M, N, K, G, n):
    L = wl.Layer("edge", M, K, N, G, n, seed=M * 7 + N)
    X, W = wl.make_activations(L), wl.make_weights(L)
    run_layer(rrs, X, W, wl.random_perm(K, M + N), G, n)


@pytest.mark.parametrize("M,K", [(700, 6144), (400, 10240), (9, 10240)])
def test_activation_kernel_team_layouts(rrs, M, K):
    """K values whose row teams fill the activation kernel's CTA differently: K = 6144
    (three teams of 96 threads) and K = 10240 (two teams of 160, 320 threads), with more
    rows than teams (the rotation recomputed in pass B) and with one row per team (the
    rotated row kept on chip); Hadamard blocks of 2048."""
    L = wl.Layer("teams", M, K, 256, 128, 2048, seed=M + K)
    X, W = wl.make_activations(L), wl.make_weights(L)
    run_layer(rrs, X, W, wl.random_perm(K, M), 128, 2048, rows=np.unique(np.r_[0:4, M - 4:M, M // 2]))


@pytest.mark.parametrize("misaligned", ["qX", "ws"])
def test_activation_outputs_at_16_byte_offsets(rrs, misaligned):
    """qX, or the workspace that holds the GEMM operand, 16- but not 32-byte aligned: the
    activation kernel then writes with 16-byte stores instead of 32-byte ones; codes,
    scales and the fp8 GEMM's Y are bit-identical to the aligned run."""
    L = wl.LAYERS["llama3_8b_kv"]
    M = 300
    X = wl.make_activations(L, M=M).to(DEV)
    perm = wl.random_perm(L.K, 5).to(DEV)
    W = wl.make_weights(L).to(DEV)
    qW, sw = rrs.prepare_weights(W, perm, L.had_block)
    qW8 = rrs.expand_weights(qW)
    flags = rrs.W_EXPANDED
    n_ws = rrs.workspace_size(M, L.N, L.K, L.G, L.had_block, flags)

    def run(qX_buf, ws_buf):
        qX, s, st = rrs.smooth_quant(X, perm, L.G, L.had_block, flags=flags, qX=qX_buf, ws=ws_buf)
        Y = rrs.w4a4_gemm(qX, s, st, qW8, sw, L.G, ws=ws_buf, flags=flags | rrs.WS_HOLDS_A8)
        return qX.clone(), s.clone(), st.clone(), Y

    ref = run(torch.empty((M, L.K // 2), dtype=torch.uint8, device=DEV),
              torch.zeros(n_ws, dtype=torch.uint8, device=DEV))
    qbuf = torch.empty(M * (L.K // 2) + 32, dtype=torch.uint8, device=DEV)
    wbuf = torch.zeros(n_ws + 32, dtype=torch.uint8, device=DEV)
    assert qbuf.data_ptr() % 32 == 0 and wbuf.data_ptr() % 32 == 0
    qX_u = qbuf[16:16 + M * (L.K // 2)].view(M, L.K // 2) if misaligned == "qX" else qbuf[:M * (L.K // 2)].view(M, L.K // 2)
    ws_u = wbuf[16:16 + n_ws] if misaligned == "ws" else wbuf[:n_ws]
    got = run(qX_u, ws_u)
    torch.cuda.synchronize()
    for a, b, what in zip(got, ref, ("qX", "s", "scale_t", "Y")):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.uint8 else a.view(torch.int32),
                           b.view(torch.uint8) if b.dtype == torch.uint8 else b.view(torch.int32)), what


def test_zero_group_and_zero_token(rrs):
    L = wl.Layer("zeros", 40, 512, 256, 128, 512, seed=3)
    X, W = wl.make_activations(L), wl.make_weights(L)
    X[7, :] = 0                      # a token that is zero everywhere
    perm = wl.identity_perm(L.K)
    # rotated group 2 is zero for all tokens only if the input is zero in a
    # whole Hadamard block; with no rotation zero channels 256..383 instead
    X[:, 256:384] = 0
    r = run_layer(rrs, X, W, perm, L.G, 1)
    assert r["s"][2].item() == 0 and r["st"][7].item() == 0
    run_layer(rrs, X, W, perm, L.G, L.had_block)


def test_channel_absmax_and_calibrated_perm(rrs):
    for name in ("tiny", "llama3_8b_qo", "llama3_8b_down"):
        L = wl.LAYERS[name]
        Xc = wl.make_activations(L, sample=1, M=min(L.M, 512))
        cm = rrs.channel_absmax(Xc.to(DEV), L.had_block)
        assert_bits_equal(cm, oracle.channel_absmax(Xc, L.had_block), f"cmax {name}")
        perm = rrs.calibrate_perm(Xc.to(DEV), L.had_block)
        np.testing.assert_array_equal(perm.cpu().numpy(), oracle.calibrate_perm(Xc, L.had_block))


# ------------------------------------------------------- full-size layers ---

def _sample_rows(M, st, k=48, seed=0):
    rng = np.random.default_rng(seed)
    top = list(np.argsort(-st)[:8])
    rest = list(rng.choice(M, size=min(M, k), replace=False))
    return sorted(set(top + rest + [0, M - 1]))


@pytest.mark.parametrize("name", ["llama3_8b_kv", "llama3_8b_qo", "llama3_8b_gateup", "llama3_8b_down"])
def test_llama3_8b_layers(rrs, name):
    """Every code and scale, and Y on every row (the oracle's rows in worker
    processes), at the full LLaMA-3-8B projection sizes."""
    L = wl.LAYERS[name]
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = torch.from_numpy(oracle.calibrate_perm(wl.make_activations(L, sample=1, M=512), L.had_block))
    run_layer(rrs, X, W, perm, L.G, L.had_block, rows=None, pool=True)


@pytest.mark.parametrize("name,N", [("llama3_70b_qo_decode_m1", 8192), ("llama3_70b_gateup_decode_m8", 4096),
                                    ("llama3_70b_down_decode_m16", 2048)])
def test_llama3_70b_decode(rrs, name, N):
    """Decode token counts at the 70B K and Hadamard sizes (N cut to keep the
    oracle's weight path short; N is a plain GEMM dimension)."""
    L = wl.LAYERS[name]
    X, W = wl.make_activations(L), wl.make_weights(L, N=N)
    perm = wl.random_perm(L.K, 1)
    run_layer(rrs, X, W, perm, L.G, L.had_block, rows=None)


def test_llama3_70b_prefill_prep(rrs):
    """70B q/o prep at full size (M=4096, K=8192, n=8192): codes and scales."""
    L = wl.LAYERS["llama3_70b_qo"]
    X = wl.make_activations(L)
    perm = wl.random_perm(L.K, 4)
    qX, s, st = rrs.smooth_quant(X.to(DEV), perm.to(DEV), L.G, L.had_block)
    _, oqX, os_, ost = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    assert_bits_equal(s, os_, "s")
    assert_bits_equal(st, ost, "scale_t")
    assert_bits_equal(qX, oqX, "qX")


@pytest.mark.parametrize("G,n", [(256, 4096), (512, 1), (4096, 4096)])
def test_group_sweep_shapes(rrs, G, n):
    L = wl.Layer("sweep", 2048, 4096, 1024, G, n, seed=G + n)
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = torch.from_numpy(oracle.calibrate_perm(wl.make_activations(L, sample=1, M=256), n))
    _, _, _, ost = oracle.smooth_quant(X, G, n, perm.numpy())
    run_layer(rrs, X, W, perm, G, n, rows=_sample_rows(L.M, ost, 16))


# ----------------------------------------------------------- API surface ---

def test_linear_equals_two_calls_and_host_path(rrs):
    L = wl.LAYERS["llama3_8b_kv"]
    X, W = wl.make_activations(L, M=256), wl.make_weights(L)
    perm = wl.random_perm(L.K, 8).to(DEV)
    Xd = X.to(DEV)
    qW, sw = rrs.prepare_weights(W.to(DEV), perm, L.had_block)
    qX, s, st = rrs.smooth_quant(Xd, perm, L.G, L.had_block)
    Y1 = rrs.w4a4_gemm(qX, s, st, qW, sw, L.G)
    Y2 = rrs.linear(Xd, qW, sw, perm, L.G, L.had_block)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    M, N, K = 256, L.N, L.K
    Xh = X.pin_memory()
    Yh = torch.empty((M, N), dtype=torch.float32).pin_memory()
    ws = rrs.make_workspace(M, N, K, L.G, L.had_block)
    rrs.linear_from_host(Xh, torch.empty_like(Xd), qW, sw, perm, L.G, L.had_block,
                         torch.empty_like(qX), torch.empty_like(s), torch.empty_like(st),
                         torch.empty((M, N), dtype=torch.float32, device=DEV), Yh, ws)
    assert torch.equal(Yh, Y1.cpu())
    qW8 = rrs.expand_weights(qW)
    Y3 = rrs.linear(Xd, qW8, sw, perm, L.G, L.had_block, flags=rrs.W_EXPANDED)
    rrs.linear_from_host(Xh, torch.empty_like(Xd), qW8, sw, perm, L.G, L.had_block,
                         torch.empty_like(qX), torch.empty_like(s), torch.empty_like(st),
                         torch.empty((M, N), dtype=torch.float32, device=DEV), Yh, ws, flags=rrs.W_EXPANDED)
    torch.cuda.synchronize()
    assert torch.equal(Y3, Y1)
    assert torch.equal(Yh, Y1.cpu())


def test_invalid_arguments_raise(rrs):
    X = torch.zeros(4, 200, dtype=torch.float16, device=DEV)
    with pytest.raises(rrs.RRSError) as e:
        rrs.smooth_quant(X, torch.arange(200, dtype=torch.int32, device=DEV), 100, 8)
    assert e.value.status_name in ("RRS_ERR_UNSUPPORTED", "RRS_ERR_INVALID_ARG")
    X = torch.zeros(4, 256, dtype=torch.float16, device=DEV)
    with pytest.raises(rrs.RRSError) as e:
        rrs.smooth_quant(X, torch.arange(256, dtype=torch.int32, device=DEV), 64, 256)
    assert e.value.status_name == "RRS_ERR_UNSUPPORTED"


def test_bounded_wait_reports_timeout_and_context_survives(rrs):
    ws = rrs.make_workspace(16, 16, 256, 128, 256)
    rrs.debug_wait_timeout(2000, ws)            # 2 ms limit, nothing releases the wait
    with pytest.raises(rrs.RRSError) as e:
        rrs.check_workspace(ws)
    assert e.value.status_name == "RRS_ERR_TIMEOUT"
    rrs.check_workspace(ws)                     # cleared
    test_tiny_full_parity(rrs, "identity")      # the context still works


def test_markstein_division_matches_ieee(rrs):
    """The activation kernels divide with Markstein's correction from RN(1/b);
    over the divisions they perform (|a| <= 8 b, b > 0) it must equal the IEEE
    quotient.  Hard cases: every divisor mantissa pattern class, quotients next
    to representable ties, exact multiples, tiny numerators."""
    rng = np.random.default_rng(123)
    n = 1 << 22
    e = rng.integers(-40, 40, size=n)
    mant = rng.integers(0, 1 << 23, size=n)
    mant[: n // 16] = (1 << 23) - 1                      # all-ones mantissas
    mant[n // 16: n // 8] = 0                            # powers of two
    mant[n // 8: n // 8 + n // 16] = rng.integers((1 << 23) - 64, 1 << 23, size=n // 16)
    b = np.ldexp(1.0 + mant / 2.0 ** 23, e).astype(np.float32)
    k = rng.uniform(-8.0, 8.0, size=n)
    a = (k * b.astype(np.float64)).astype(np.float32)
    q = rng.integers(-8, 8, size=n).astype(np.float32)     # exact multiples and their neighbours
    sel = slice(n // 4, n // 2)
    a[sel] = (q[sel] * b[sel]).astype(np.float32)
    ulp_steps = rng.integers(-3, 4, size=n).astype(np.int32)
    sel2 = slice(n // 2, 3 * n // 4)
    a[sel2] = (a[sel2].view(np.int32) + ulp_steps[sel2]).view(np.float32)
    a[3 * n // 4: 3 * n // 4 + 1024] = 0.0
    tiny = slice(7 * n // 8, n)
    a[tiny] = (b[tiny].astype(np.float64) * rng.uniform(-1, 1, size=n // 8) * 2.0 ** -30).astype(np.float32)
    ad = torch.from_numpy(a).to(DEV)
    bd = torch.from_numpy(b).to(DEV)
    qf, qi = rrs.debug_divide(ad, bd)
    qf, qi = qf.cpu().numpy(), qi.cpu().numpy()
    same = (qf.view(np.uint32) == qi.view(np.uint32)) | ((qf == 0) & (qi == 0))
    assert same.all(), f"{np.count_nonzero(~same)} quotients differ, e.g. a={a[~same][:3]} b={b[~same][:3]}"
    # and the IEEE division itself is the correctly rounded quotient (checked in double)
    ref = (a.astype(np.float64) / b.astype(np.float64)).astype(np.float32)
    assert np.array_equal(qi, ref)


@pytest.mark.parametrize("name", ["llama3_70b_qo", "llama3_70b_gateup", "llama3_70b_down"])
def test_llama3_70b_prefill_layers(rrs, name):
    """70B prefill layers at full size (M=4096; K, N and the Hadamard blocks as defined):
    every code and scale bit-exact, Y on sampled rows (the largest token scales, the first
    and last rows, and random ones) within tolerance, packed and expanded weights
    bit-identical."""
    L = wl.LAYERS[name]
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = wl.random_perm(L.K, 5)
    _, _, _, ost = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    run_layer(rrs, X, W, perm, L.G, L.had_block, rows=_sample_rows(L.M, ost, k=8))


def test_one_hadamard_size_at_two_row_lengths_in_sequence(rrs):
    """The activation kernel for one Hadamard size serves row lengths that need
    different shared memory (K = 14336 with 7 blocks of 2048, then K = 2048 with 8
    rows per CTA): the second launch must get its own shared-memory limit."""
    L = wl.LAYERS["llama3_8b_down"]
    X1 = wl.make_activations(L, M=64)
    p1 = wl.random_perm(L.K, 31)
    rrs.smooth_quant(X1.to(DEV), p1.to(DEV), L.G, L.had_block)
    g = torch.Generator().manual_seed(32)
    X2 = (torch.randn(256, 2048, generator=g) * 2).to(torch.float16)
    p2 = wl.random_perm(2048, 32)
    qX, s, st = rrs.smooth_quant(X2.to(DEV), p2.to(DEV), 128, 2048)
    torch.cuda.synchronize()
    _, oqX, os_, ost = oracle.smooth_quant(X2, 128, 2048, p2.numpy())
    assert_bits_equal(s, os_, "s")
    assert_bits_equal(st, ost, "scale_t")
    assert_bits_equal(qX, oqX, "qX")


@pytest.mark.parametrize("flags", [0, "expanded"])
def test_group_larger_than_a_promotion_block(rrs, flags):
    """G = 6144 (K = 12288): the GEMM promotes in blocks of 3072 channels (the largest
    multiple of 128 that divides G and is at most 4096); every group's P_g must still be
    the oracle's, on the packed and the fp8 kernel, and Y within the tolerance."""
    M, N, K, G = 64, 256, 12288, 6144
    rng = np.random.default_rng(6144)
    qX = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    qWd = torch.from_numpy(qW).to(DEV)
    fl = rrs.W_EXPANDED if flags == "expanded" else 0
    qWg = rrs.expand_weights(qWd) if fl else qWd
    P = rrs.w4a4_gemm_debug_partials(torch.from_numpy(qX).to(DEV), qWg, G, flags=fl)
    assert_bits_equal(P, oracle.group_partials(qX, qW, G), "P_g (G = 6144)")
    s = (rng.random(K // G, dtype=np.float32) + 0.5).astype(np.float32)
    st = rng.random(M, dtype=np.float32)
    sw = rng.random(N, dtype=np.float32)
    Y = rrs.w4a4_gemm(torch.from_numpy(qX).to(DEV), torch.from_numpy(s).to(DEV), torch.from_numpy(st).to(DEV),
                      qWg, torch.from_numpy(sw).to(DEV), G, flags=fl)
    torch.cuda.synchronize()
    Yo, B = oracle.linear_rows(qX, s, st, qW, sw, G)
    assert oracle.y_tolerance_ok(Y.cpu().numpy(), Yo, B).all()


def test_largest_k(rrs):
    """K = 32768 (four Hadamard blocks of 8192): the one-launch activation kernel's
    shared memory would not fit, so the general kernels take it; codes and scales
    bit-exact, and the layer's Y within the tolerance."""
    M, N, K, G, n = 8, 128, 32768, 128, 8192
    L = wl.Layer("k32768", M, K, N, G, n, seed=32768)
    X, W = wl.make_activations(L), wl.make_weights(L)
    perm = wl.random_perm(K, 5)
    run_layer(rrs, X, W, perm, G, n, rows=None)

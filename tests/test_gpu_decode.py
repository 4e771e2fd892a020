"""GPU: the single-launch linear layer for few tokens (M <= 16) that rrs_linear
takes with packed weights.  Codes, s and scale_t must match the oracle bit for
bit and Y must meet the per-element tolerance, at the 70B decode sizes (Hadamard
blocks of 8192 and 7 x 4096), over the edge cases of the launch: one token, a
token count that is not a multiple of 8, 9..16 tokens (two MMA column tiles),
one output tile, groups of 256 and 1024 channels, no rotation, unit scales,
all-zero tokens and groups, bf16 Y, and consecutive calls through one
workspace.  The rotated activations the kernel leaves in the workspace are
compared with the oracle's rotation, which also shows the single launch ran."""
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


def _bits(t):
    a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def _same(gpu, orc, what):
    g, o = _bits(gpu), _bits(orc)
    assert g.shape == o.shape, what
    bad = np.nonzero(g != o)
    assert bad[0].size == 0, f"{what}: {bad[0].size} mismatches, first at {[b[0] for b in bad]}"


def _single_launch(rrs, X, qW, sw, perm, G, n, flags=0, ws=None, Y=None):
    M, K = X.shape
    N = qW.shape[0]
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
    s = torch.empty(K // G, dtype=torch.float32, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV)
    ws = rrs.make_workspace(M, N, K, G, n, flags) if ws is None else ws
    Y = rrs.linear(X, qW, sw, perm, G, n, flags=flags | rrs.ONE_LAUNCH, qX=qX, s=s, scale_t=st, ws=ws, Y=Y)
    rrs.check_workspace(ws)
    return Y, qX, s, st, ws


def _check(rrs, X, W, perm, G, n, flags=0, check_rot=True):
    """Single launch vs the oracle (codes, scales, Y) and vs the two-launch path (Y)."""
    M, K = X.shape
    unit = bool(flags & rrs.FORCE_UNIT_SCALES)
    n_eff = 1 if flags & rrs.NO_ROTATE else n
    Xd, Wd, pd = X.to(DEV), W.to(DEV), perm.to(DEV)
    qW, sw = rrs.prepare_weights(Wd, pd, n, flags)
    Y, qX, s, st, ws = _single_launch(rrs, Xd, qW, sw, pd, G, n, flags)
    _, oqX, os_, ost = oracle.smooth_quant(X, G, n_eff, perm.numpy(), unit_scales=unit)
    _same(s, os_, "s")
    _same(st, ost, "scale_t")
    _same(qX, oqX, "qX")
    if check_rot:
        rot = ws[256:256 + M * K * 4].view(torch.float32).view(M, K)
        _same(rot, oracle.rotate(X, n_eff), "X_rot left in the workspace")
    _, oqW, osw = oracle.prepare_weights(W, n_eff, perm.numpy())
    _same(qW, oqW, "qW")
    Yo, B = oracle.linear_rows(oqX, os_, ost, oqW, osw, G)
    Yg = Y.cpu().numpy()
    ok = oracle.y_tolerance_ok(Yg, Yo, B)
    assert ok.all(), f"Y: {np.count_nonzero(~ok)} of {ok.size} outside tolerance"
    assert np.linalg.norm(Yg - Yo) / max(np.linalg.norm(Yo), 1e-30) < 1e-5
    # the two-launch path (activation kernel, then the GEMM) on the same inputs
    qX2, s2, st2 = rrs.smooth_quant(Xd, pd, G, n, flags)
    Y2 = rrs.w4a4_gemm(qX2, s2, st2, qW, sw, G)
    torch.cuda.synchronize()
    _same(qX2, qX, "qX (two launches)")
    ok2 = oracle.y_tolerance_ok(Y2.cpu().numpy(), Yo, B)
    assert ok2.all()
    return Y


@pytest.mark.parametrize("name,N,M", [
    ("llama3_70b_qo_decode_m1", 1024, 1),
    ("llama3_70b_qo_decode_m8", 512, 8),
    ("llama3_70b_gateup_decode_m16", 1024, 16),
    ("llama3_70b_down_decode_m1", 512, 1),
    ("llama3_70b_down_decode_m16", 1024, 16),
])
def test_decode_shapes_against_the_oracle(rrs, name, N, M):
    """70B K and Hadamard sizes (8192 full, 7 x 4096 block-diagonal); N cut for the oracle."""
    L = wl.LAYERS[name]
    X, W = wl.make_activations(L, M=M), wl.make_weights(L, N=N)
    _check(rrs, X, W, wl.random_perm(L.K, 2), L.G, L.had_block)


@pytest.mark.parametrize("M", [2, 3, 7, 9, 13])
def test_ragged_token_counts(rrs, M):
    L = wl.LAYERS["llama3_8b_qo"]
    X, W = wl.make_activations(L, sample=M, M=M), wl.make_weights(L, N=256)
    _check(rrs, X, W, wl.random_perm(L.K, M), L.G, L.had_block)


@pytest.mark.parametrize("N", [16, 48])
def test_few_output_tiles(rrs, N):
    L = wl.LAYERS["llama3_8b_down"]              # K = 14336 = 14 chunks, 7 x 2048 blocks
    X, W = wl.make_activations(L, M=5), wl.make_weights(L, N=N)
    _check(rrs, X, W, wl.random_perm(L.K, 7), L.G, L.had_block)


@pytest.mark.parametrize("G", [256, 1024])
def test_larger_groups(rrs, G):
    L = wl.LAYERS["llama3_8b_gateup"]
    X, W = wl.make_activations(L, M=6), wl.make_weights(L, N=512)
    _check(rrs, X, W, wl.random_perm(L.K, G), G, L.had_block)


@pytest.mark.parametrize("flag", ["no_rotate", "unit_scales"])
def test_flags(rrs, flag):
    f = {"no_rotate": rrs.NO_ROTATE, "unit_scales": rrs.FORCE_UNIT_SCALES}[flag]
    L = wl.LAYERS["llama3_8b_qo"]
    X, W = wl.make_activations(L, sample=4, M=11), wl.make_weights(L, N=256)
    _check(rrs, X, W, wl.random_perm(L.K, 4), L.G, L.had_block, flags=f)


def test_small_hadamard_blocks_and_one_chunk(rrs):
    # K = 1024 (a single chunk) with Hadamard blocks of 256: several blocks per rotation item
    K, M, N = 1024, 4, 64
    g = torch.Generator().manual_seed(12)
    X = (torch.randn(M, K, generator=g) * 3).to(torch.float16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.float16)
    _check(rrs, X, W, wl.random_perm(K, 12), 128, 256)


def test_zero_tokens_and_zero_groups(rrs):
    L = wl.LAYERS["llama3_8b_qo"]
    X = wl.make_activations(L, sample=9, M=10)
    X[3] = 0                                     # amax_t = 0: scale 0, codes 0
    W = wl.make_weights(L, N=128)
    # a group that is zero for every token: with no rotation and the identity
    # reorder, zero channels 128..255 make group 1 all zero (s_1 = 0)
    X[:, 128:256] = 0
    _check(rrs, X, W, wl.identity_perm(L.K), L.G, L.had_block, flags=rrs.NO_ROTATE)


def test_bf16_y_is_the_fp32_y_rounded(rrs):
    L = wl.LAYERS["llama3_70b_qo_decode_m16"]
    X, W = wl.make_activations(L), wl.make_weights(L, N=512)
    perm = wl.random_perm(L.K, 3).to(DEV)
    qW, sw = rrs.prepare_weights(W.to(DEV), perm, L.had_block)
    Y32, *_ = _single_launch(rrs, X.to(DEV), qW, sw, perm, L.G, L.had_block)
    Yb = torch.empty((X.shape[0], 512), dtype=torch.bfloat16, device=DEV)
    Y16, *_ = _single_launch(rrs, X.to(DEV), qW, sw, perm, L.G, L.had_block, flags=rrs.Y_BF16, Y=Yb)
    torch.cuda.synchronize()
    _same(Y16.view(torch.int16), Y32.to(torch.bfloat16).view(torch.int16), "bf16 Y")


def test_consecutive_calls_through_one_workspace(rrs):
    """The grid barrier state is left ready for the next call, whatever the shape."""
    big = wl.LAYERS["llama3_70b_down_decode_m16"]
    ws = rrs.make_workspace(16, 8192, big.K, big.G, big.had_block)
    outs = []
    for name, N, M, seed in [("llama3_70b_qo_decode_m8", 8192, 8, 1), ("llama3_70b_down_decode_m16", 2048, 16, 2),
                             ("llama3_70b_qo_decode_m8", 8192, 3, 3), ("llama3_70b_qo_decode_m8", 8192, 8, 1)]:
        L = wl.LAYERS[name]
        X, W = wl.make_activations(L, sample=seed, M=M).to(DEV), wl.make_weights(L, N=N).to(DEV)
        perm = wl.random_perm(L.K, seed).to(DEV)
        qW, sw = rrs.prepare_weights(W, perm, L.had_block)
        Y, qX, s, st, _ = _single_launch(rrs, X, qW, sw, perm, L.G, L.had_block, ws=ws)
        Y2 = rrs.w4a4_gemm(*rrs.smooth_quant(X, perm, L.G, L.had_block), qW, sw, L.G)
        torch.cuda.synchronize()
        rel = (torch.linalg.norm(Y - Y2) / torch.linalg.norm(Y2)).item()
        assert rel < 1e-5, (name, rel)
        outs.append(Y.clone())
    _same(outs[3], outs[0], "the same call repeated")


@pytest.mark.parametrize("name", ["llama3_70b_qo_decode_m16", "llama3_70b_gateup_decode_m1",
                                  "llama3_70b_down_decode_m8"])
def test_full_70b_decode_sizes(rrs, name):
    """Full N (8192 / 28672): codes and scales against the oracle; Y against the
    two-launch path (whose Y is checked against the oracle at cut N above)."""
    L = wl.LAYERS[name]
    X = wl.make_activations(L)
    perm = wl.random_perm(L.K, 6)
    Xd, pd = X.to(DEV), perm.to(DEV)
    qW, sw = rrs.prepare_weights(wl.make_weights(L).to(DEV), pd, L.had_block)
    Y, qX, s, st, ws = _single_launch(rrs, Xd, qW, sw, pd, L.G, L.had_block)
    _, oqX, os_, ost = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    _same(s, os_, "s")
    _same(st, ost, "scale_t")
    _same(qX, oqX, "qX")
    Y2 = rrs.w4a4_gemm(*rrs.smooth_quant(Xd, pd, L.G, L.had_block), qW, sw, L.G)
    torch.cuda.synchronize()
    d = (Y - Y2).abs()
    assert (d <= 1e-3 * Y2.abs() + 1e-6 * Y2.abs().max()).all()
    assert (torch.linalg.norm(Y - Y2) / torch.linalg.norm(Y2)).item() < 1e-5


@pytest.mark.parametrize("M,one_launch", [(1, True), (6, True), (12, False)])
def test_default_choice_of_form(rrs, M, one_launch):
    """Without RRS_ONE_LAUNCH, rrs_linear takes the single launch for M <= 6 (or a
    large weight stream) and the two launches otherwise; the rotated rows left in
    the workspace show which ran.  Both give the oracle's codes and Y."""
    L = wl.LAYERS["llama3_8b_qo"]
    X, W = wl.make_activations(L, sample=M, M=M), wl.make_weights(L, N=256)
    perm = wl.random_perm(L.K, M)
    Xd, pd = X.to(DEV), perm.to(DEV)
    qW, sw = rrs.prepare_weights(W.to(DEV), pd, L.had_block)
    ws = rrs.make_workspace(M, 256, L.K, L.G, L.had_block)
    qX = torch.empty((M, L.K // 2), dtype=torch.uint8, device=DEV)
    s = torch.empty(L.K // L.G, dtype=torch.float32, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV)
    Y = rrs.linear(Xd, qW, sw, pd, L.G, L.had_block, qX=qX, s=s, scale_t=st, ws=ws)
    rrs.check_workspace(ws)
    torch.cuda.synchronize()
    rot = ws[256:256 + M * L.K * 4].view(torch.float32).view(M, L.K).cpu().numpy()
    same_rot = np.array_equal(rot.view(np.uint32), oracle.rotate(X, L.had_block).view(np.uint32))
    assert same_rot == one_launch
    _, oqX, os_, ost = oracle.smooth_quant(X, L.G, L.had_block, perm.numpy())
    _same(qX, oqX, "qX")
    _same(s, os_, "s")
    _same(st, ost, "scale_t")
    _, oqW, osw = oracle.prepare_weights(W, L.had_block, perm.numpy())
    Yo, B = oracle.linear_rows(oqX, os_, ost, oqW, osw, L.G)
    assert oracle.y_tolerance_ok(Y.cpu().numpy(), Yo, B).all()

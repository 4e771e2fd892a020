"""rrs_smooth_quant_noalloc: the activation path for callers that cannot
allocate device memory at call time (no workspace argument; a fixed scratch
array inside the library instead).

It must give exactly what rrs_smooth_quant gives with a caller workspace: the
same packed codes, group scales and per-token scales, bit for bit.  Two calls
in a row with different inputs check that the shared scratch carries nothing
from one call into the next.  This file is named so that pytest collects it
last.
"""
import ctypes

import numpy as np
import pytest
import torch

from activation_smoothing_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")


def _noalloc_fn():
    import activation_smoothing_b200 as rrs
    f = rrs.lib().rrs_smooth_quant_noalloc
    P, I, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    f.argtypes = [P, I, I, I, I, P, P, P, P, U, P]
    f.restype = I
    return rrs, f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _run_noalloc(rrs, f, X, perm, G, n, flags=0):
    M, K = X.shape
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
    s = torch.empty(K // G, dtype=torch.float32, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = f(_ptr(X), M, K, G, n, _ptr(perm), _ptr(qX), _ptr(s), _ptr(st), flags, stream)
    assert rc == 0, rrs.lib().rrs_last_error_string()
    return qX, s, st


@pytest.mark.parametrize("calls", [[("llama3_8b_qo", 128, 11), ("llama3_8b_down", 64, 12)]])
def test_noalloc_matches_workspace_path_on_consecutive_calls(calls):
    rrs, f = _noalloc_fn()
    for name, M, seed in calls:
        L = wl.LAYERS[name]
        X = wl.make_activations(L, sample=seed, M=M).to(DEV)
        perm = wl.random_perm(L.K, seed).to(DEV)
        ref = rrs.smooth_quant(X, perm, L.G, L.had_block)
        got = _run_noalloc(rrs, f, X, perm, L.G, L.had_block)
        torch.cuda.synchronize()
        for a, b, what in zip(got, ref, ("qX", "s", "scale_t")):
            a_np, b_np = a.cpu().numpy(), b.cpu().numpy()
            assert np.array_equal(a_np.view(np.uint8), b_np.view(np.uint8)), f"{name}: {what} differs"


def _flag(name):
    import activation_smoothing_b200 as rrs
    return {"none": 0, "no_rotate": rrs.NO_ROTATE, "unit_scales": rrs.FORCE_UNIT_SCALES}[name]


# K = 256 takes the general two-kernel path, K = 4096 the single activation kernel;
# each under plain RRS, without the rotation (Runtime Smooth) and with s forced to 1.
@pytest.mark.parametrize("flag", ["none", "no_rotate", "unit_scales"])
@pytest.mark.parametrize("name,M", [("tiny", 16), ("llama3_8b_qo", 96)])
def test_noalloc_matches_workspace_path_per_path_and_flag(name, M, flag):
    rrs, f = _noalloc_fn()
    flags = _flag(flag)
    L = wl.LAYERS[name]
    for seed in (21, 22):                    # two calls in a row through the shared scratch
        X = wl.make_activations(L, sample=seed, M=M).to(DEV)
        perm = wl.random_perm(L.K, seed).to(DEV)
        ref = rrs.smooth_quant(X, perm, L.G, L.had_block, flags=flags)
        got = _run_noalloc(rrs, f, X, perm, L.G, L.had_block, flags)
        torch.cuda.synchronize()
        for a, b, what in zip(got, ref, ("qX", "s", "scale_t")):
            a_np, b_np = a.cpu().numpy(), b.cpu().numpy()
            assert np.array_equal(a_np.view(np.uint8), b_np.view(np.uint8)), f"{name}/{flag}: {what} differs"
        if flag == "unit_scales":
            assert torch.all(got[1] == 1.0)


def test_noalloc_rejects_sizes_beyond_its_limit():
    rrs, f = _noalloc_fn()
    M, K = 512, 4096                       # 2M elements > the 1M limit
    X = torch.zeros((M, K), dtype=torch.float16, device=DEV)
    perm = torch.arange(K, dtype=torch.int32, device=DEV)
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
    s = torch.empty(K // 128, dtype=torch.float32, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV)
    rc = f(_ptr(X), M, K, 128, K, _ptr(perm), _ptr(qX), _ptr(s), _ptr(st), 0, None)
    assert rc == 2                          # RRS_ERR_UNSUPPORTED
    assert b"limit" in rrs.lib().rrs_last_error_string()

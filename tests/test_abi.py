"""The C-ABI library builds, loads and exports every symbol the header declares;
host-side argument checks and the host sort work without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rrs.h")


@pytest.fixture(scope="module")
def L():
    from activation_smoothing_b200 import build
    build.build()
    from activation_smoothing_b200 import _binding
    return _binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rrs_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_core_calls():
    names = declared_functions()
    for n in ("rrs_prepare_weights", "rrs_smooth_quant", "rrs_w4a4_gemm", "rrs_linear"):
        assert n in names


def test_binding_constants_match_the_header():
    from activation_smoothing_b200 import _binding as b
    defs = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define RRS_(\w+) (\d+)u", open(HEADER).read())}
    for name in ("NO_ROTATE", "FORCE_UNIT_SCALES", "WS_HOLDS_A8", "W_EXPANDED", "Y_BF16", "Y_SILU_MUL", "ONE_LAUNCH"):
        assert getattr(b, name) == defs[name], name


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/rrs.h but not exported"


def test_library_is_sm100a_build():
    from activation_smoothing_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)
    assert "--use_fast_math" not in build.FLAGS


def test_workspace_size(L):
    # header + the GEMM operand (M*K bytes) + one row of K/128 group maxima per CTA of
    # the activation kernel; nothing of size M*K*4 (the rotation is recomputed, not stored)
    need = L.rrs_workspace_size(2048, 4096, 4096, 128, 4096, 0)
    assert 256 + 2048 * 4096 <= need < 256 + 2048 * 4096 + 2048 * 4096 // 4
    # decode sizes keep room for the split-k partial sums of the GEMM
    assert L.rrs_workspace_size(16, 8192, 8192, 128, 8192, 0) >= 256 + 16 * 8192 + 16 * 16 * 8192 * 4


def test_perm_from_channel_max_host(L):
    rng = np.random.default_rng(0)
    c = rng.standard_normal(1000).astype(np.float32)
    c[10] = c[20] = c[30] = 5.0          # ties keep the lower index first
    perm = np.empty(1000, np.int32)
    rc = L.rrs_perm_from_channel_max(c.ctypes.data_as(ctypes.c_void_p), 1000,
                                     perm.ctypes.data_as(ctypes.c_void_p))
    assert rc == 0
    np.testing.assert_array_equal(perm, np.argsort(-c, kind="stable"))
    assert list(perm[:3]) == [10, 20, 30]


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_argument_checks_fail_before_any_launch(L):
    ok = _fake(0x10000)
    mis = _fake(0x10008)
    # null pointer
    assert L.rrs_prepare_weights(None, 16, 256, 256, ok, ok, ok, 0, None) == 1
    # misaligned pointer
    assert L.rrs_prepare_weights(mis, 16, 256, 256, ok, ok, ok, 0, None) == 1
    assert b"aligned" in L.rrs_last_error_string()
    # K not a multiple of 128 -> unsupported on the CUDA path
    assert L.rrs_prepare_weights(ok, 16, 200, 8, ok, ok, ok, 0, None) == 2
    # Hadamard block not a power of two
    assert L.rrs_prepare_weights(ok, 16, 256, 96, ok, ok, ok, 0, None) == 1
    # Hadamard block not dividing K
    assert L.rrs_prepare_weights(ok, 16, 384, 256, ok, ok, ok, 0, None) == 1
    ws = ok
    # G not dividing K -> invalid; G not a multiple of 128 -> unsupported
    assert L.rrs_smooth_quant(ok, 16, 256, 100, 256, ok, ok, ok, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_smooth_quant(ok, 16, 256, 64, 256, ok, ok, ok, ok, ws, 1 << 20, 0, None) == 2
    # workspace too small
    assert L.rrs_smooth_quant(ok, 16, 256, 128, 256, ok, ok, ok, ok, ws, 8, 0, None) == 5
    need = L.rrs_workspace_size(16, 16, 4096, 128, 4096, 0)
    assert need >= 256 + 16 * 4096 + 16 * 16 * 16 * 4      # header, operand, split-k room
    need_sq = L.rrs_workspace_size(16, 0, 4096, 128, 4096, 0)     # N = 0: no GEMM split-k room
    assert 256 + 16 * 4096 <= need_sq <= need
    assert L.rrs_smooth_quant(ok, 16, 4096, 128, 4096, ok, ok, ok, ok, ws, need_sq - 1, 0, None) == 5
    # pass A / pass B of the token-sharded path: same checks
    assert L.rrs_group_max(None, 16, 256, 128, 256, ok, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_group_max(ok, 0, 256, 128, 256, ok, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_group_max(ok, 16, 256, 64, 256, ok, ok, ws, 1 << 20, 0, None) == 2
    assert L.rrs_group_max(ok, 16, 4096, 128, 4096, ok, ok, ws, need_sq - 1, 0, None) == 5
    assert L.rrs_smooth_quant_scaled(ok, 16, 256, 128, 256, ok, None, ok, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_smooth_quant_scaled(ok, 16, 256, 100, 256, ok, ok, ok, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_smooth_quant_scaled(ok, 16, 4096, 128, 4096, ok, ok, ok, ok, ws, need_sq - 1, 0, None) == 5
    # the scales come from s: unit scales do not apply to pass B
    assert L.rrs_smooth_quant_scaled(ok, 16, 256, 128, 256, ok, ok, ok, ok, ws, 1 << 20, 2, None) == 1
    assert b"s filled with 1" in L.rrs_last_error_string()
    # KV cache: null pointers, bad sizes, flags
    assert L.rrs_kv_quant(None, 4, 2, 128, ok, ok, 0, None) == 1
    assert L.rrs_kv_quant(ok, 0, 2, 128, ok, ok, 0, None) == 1
    assert L.rrs_kv_quant(ok, 4, 2, 96, ok, ok, 0, None) == 1        # not a power of two
    assert L.rrs_kv_quant(ok, 4, 2, 64, ok, ok, 0, None) == 2        # below the CUDA path's head size
    assert L.rrs_kv_quant(ok, 4, 2, 128, ok, ok, 1, None) == 1       # no flags
    assert L.rrs_kv_dequant(ok, ok, 4, 2, 12, ok, None) == 1
    assert L.rrs_kv_dequant(ok, None, 4, 2, 128, ok, None) == 1
    # M < 1
    assert L.rrs_w4a4_gemm(ok, ok, ok, ok, ok, 0, 16, 256, 128, ok, ws, 1 << 20, 0, None) == 1
    assert L.rrs_debug_wait_timeout(0, ws, 256, None) == 1
    assert len(L.rrs_last_error_string()) > 0


def test_next_row_entry_points_check_arguments_before_any_launch(L):
    ok = _fake(0x10000)
    mis = _fake(0x10004)
    # rrs_silu_mul(GU, M, F, H, stream)
    assert L.rrs_silu_mul(None, 4, 8, ok, None) == 1
    assert L.rrs_silu_mul(ok, 4, 8, None, None) == 1
    assert L.rrs_silu_mul(mis, 4, 8, ok, None) == 1
    assert b"aligned" in L.rrs_last_error_string()
    assert L.rrs_silu_mul(ok, 0, 8, ok, None) == 1
    assert L.rrs_silu_mul(ok, 4, 0, ok, None) == 1
    # rrs_expand_weights(qW, N, K, qW8, stream)
    assert L.rrs_expand_weights(None, 16, 256, ok, None) == 1
    assert L.rrs_expand_weights(ok, 16, 256, mis, None) == 1
    assert L.rrs_expand_weights(ok, 0, 256, ok, None) == 1
    assert L.rrs_expand_weights(ok, 16, 200, ok, None) == 2     # K % 128 != 0: unsupported


def test_check_perm_checks_arguments_before_any_launch(L):
    ok = _fake(0x10000)
    mis = _fake(0x10004)
    K = 4096
    need = 256 + 16 + 4 * ((K + 31) // 32)
    # rrs_check_perm(perm, K, ws, ws_bytes, stream)
    assert L.rrs_check_perm(None, K, ok, need, None) == 1
    assert b"perm" in L.rrs_last_error_string()
    assert L.rrs_check_perm(mis, K, ok, need, None) == 1
    assert L.rrs_check_perm(ok, 0, ok, need, None) == 1
    assert L.rrs_check_perm(ok, K, None, need, None) == 5           # workspace missing
    assert L.rrs_check_perm(ok, K, ok, need - 4, None) == 5         # one bitmap word short
    assert b"need" in L.rrs_last_error_string()
    # any workspace rrs_workspace_size gives for this K is large enough
    assert L.rrs_workspace_size(1, 0, K, 128, K, 0) >= need


def test_binding_shape_checks_without_gpu():
    import torch
    import activation_smoothing_b200 as rrs
    X = torch.zeros(4, 256, dtype=torch.float16)
    with pytest.raises(ValueError):
        rrs.smooth_quant(X, torch.arange(256, dtype=torch.int32), 128, 256)   # host tensors rejected


def test_binding_flag_and_dtype_inference_without_gpu():
    import torch
    from activation_smoothing_b200 import _binding as b
    assert b._y_flags(None, 0) == 0
    assert b._y_flags(torch.empty(2, 2, dtype=torch.float32), b.WS_HOLDS_A8) == b.WS_HOLDS_A8
    assert b._y_flags(torch.empty(2, 2, dtype=torch.bfloat16), 0) == b.Y_BF16
    assert b._y_dtype(b.Y_BF16 | b.W_EXPANDED) == torch.bfloat16
    assert b._y_dtype(b.W_EXPANDED) == torch.float32
    # packed weights are uint8 [N, K/2]; expanded ones e4m3 [N, K]; host tensors are refused
    with pytest.raises(TypeError):
        b._need_weights(torch.zeros(4, 64, dtype=torch.int8), 4, 128, 0)
    with pytest.raises(TypeError):
        b._need_weights(torch.zeros(4, 128, dtype=torch.uint8), 4, 128, b.W_EXPANDED)
    with pytest.raises(ValueError):
        b._need_weights(torch.zeros(4, 64, dtype=torch.uint8), 4, 128, 0)
    with pytest.raises(ValueError):
        b._need_weights(torch.zeros(4, 128, dtype=torch.float8_e4m3fn), 4, 128, b.W_EXPANDED)


def test_next_row_bindings_refuse_host_tensors():
    import torch
    import activation_smoothing_b200 as rrs
    with pytest.raises((TypeError, ValueError)):
        rrs.silu_mul(torch.zeros(4, 16, dtype=torch.float32))
    with pytest.raises((TypeError, ValueError)):
        rrs.expand_weights(torch.zeros(4, 64, dtype=torch.uint8))


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "activation_smoothing_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "rrs_oracle" not in src, f


def test_interleave_gate_up_rows_without_gpu():
    import torch
    from activation_smoothing_b200 import _binding as b
    Wg = torch.arange(12, dtype=torch.float32).reshape(3, 4)
    Wu = -Wg
    W = b.interleave_gate_up(Wg, Wu)
    assert W.shape == (6, 4)
    assert torch.equal(W[0::2], Wg) and torch.equal(W[1::2], Wu)
    assert b._y_shape(8, 10, b.Y_SILU_MUL) == (8, 5) and b._y_dtype(b.Y_SILU_MUL) == torch.float16

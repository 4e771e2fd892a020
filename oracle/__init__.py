"""CPU oracle for the Rotated Runtime Smooth W4A4 linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package; the product (``activation_smoothing_b200``) never does.  It shares no
code with the CUDA path.  The arithmetic lives in ``rrs_oracle.c`` (plain C
loops, one IEEE fp32 operation per source operator); this module only
marshals numpy arrays through ctypes.  Each function cites the page passage it
follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # RRS_ORACLE_LIB lets the mutation test load a deliberately broken build.
        path = os.environ.get("RRS_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        L.orc_fwht.argtypes = [P, i32]
        L.orc_fwht.restype = None
        L.orc_hadamard_scale.argtypes = [i32]
        L.orc_hadamard_scale.restype = ctypes.c_float
        L.orc_rotate.argtypes = [P, i64, i32, i32, P]
        L.orc_reorder.argtypes = [P, i64, i32, P, P]
        L.orc_group_max.argtypes = [P, i64, i32, i32, P]
        L.orc_smooth_quant_from_xp.argtypes = [P, i64, i32, i32, i32, P, P, P, P]
        L.orc_smooth_quant.argtypes = [P, i64, i32, i32, i32, P, i32, P, P, P, P]
        L.orc_prepare_weights.argtypes = [P, i64, i32, i32, P, P, P, P]
        L.orc_group_partials.argtypes = [P, P, i64, i64, i32, i32, P, i64, P]
        L.orc_linear_rows.argtypes = [P, P, P, P, P, i64, i64, i32, i32, P, i64, P, P]
        L.orc_channel_absmax.argtypes = [P, i64, i32, i32, P]
        L.orc_kv_quant.argtypes = [P, i64, i32, P, P, P]
        L.orc_kv_dequant.argtypes = [P, i64, i32, P, P]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    """fp16 (or fp32) array-like -> contiguous fp32 numpy (fp16 -> fp32 is exact)."""
    if hasattr(x, "numpy"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x).astype(np.float32))


def _i32(x) -> np.ndarray:
    if hasattr(x, "numpy"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x).astype(np.int32))


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def fwht(v) -> np.ndarray:
    """Unnormalised canonical-order FWHT of a 1-D vector (fp32)."""
    a = _f32(v).copy()
    n = a.shape[0]
    lib().orc_fwht(_p(a), n)
    return a


def hadamard_scale(n: int) -> float:
    return float(np.float32(lib().orc_hadamard_scale(n)))


def rotate(X, n: int) -> np.ndarray:
    x = _f32(X)
    rows, K = x.shape
    out = np.empty_like(x)
    _check(lib().orc_rotate(_p(x), rows, K, n, _p(out)), "rotate")
    return out


def reorder(Xrot: np.ndarray, perm) -> np.ndarray:
    x = _f32(Xrot)
    p = _i32(perm)
    out = np.empty_like(x)
    _check(lib().orc_reorder(_p(x), x.shape[0], x.shape[1], _p(p), _p(out)), "reorder")
    return out


def group_max(Xp: np.ndarray, G: int) -> np.ndarray:
    x = _f32(Xp)
    s = np.empty(x.shape[1] // G, np.float32)
    _check(lib().orc_group_max(_p(x), x.shape[0], x.shape[1], G, _p(s)), "group_max")
    return s


def smooth_quant_from_xp(Xp: np.ndarray, G: int, unit_scales: bool = False):
    """-> (codes int8 [M,K], qX uint8 [M,K/2], s fp32 [K/G], scale_t fp32 [M])."""
    x = _f32(Xp)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    qX = np.empty((M, K // 2), np.uint8)
    s = np.empty(K // G, np.float32)
    st = np.empty(M, np.float32)
    _check(lib().orc_smooth_quant_from_xp(_p(x), M, K, G, int(unit_scales), _p(codes), _p(qX),
                                          _p(s), _p(st)), "smooth_quant_from_xp")
    return codes, qX, s, st


def smooth_quant(X, G: int, n: int, perm, unit_scales: bool = False):
    """Online path on fp16 X [M,K] -> (codes, qX, s, scale_t)."""
    x = _f32(X)
    p = _i32(perm)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    qX = np.empty((M, K // 2), np.uint8)
    s = np.empty(K // G, np.float32)
    st = np.empty(M, np.float32)
    _check(lib().orc_smooth_quant(_p(x), M, K, G, n, _p(p), int(unit_scales), _p(codes), _p(qX),
                                  _p(s), _p(st)), "smooth_quant")
    return codes, qX, s, st


def prepare_weights(W, n: int, perm):
    """Offline path on fp16 W [N,K] -> (codes int8 [N,K], qW uint8 [N,K/2], scale_w fp32 [N])."""
    w = _f32(W)
    p = _i32(perm)
    N, K = w.shape
    codes = np.empty((N, K), np.int8)
    qW = np.empty((N, K // 2), np.uint8)
    sw = np.empty(N, np.float32)
    _check(lib().orc_prepare_weights(_p(w), N, K, n, _p(p), _p(codes), _p(qW), _p(sw)),
           "prepare_weights")
    return codes, qW, sw


def group_partials(qX: np.ndarray, qW: np.ndarray, G: int, rows: Optional[Sequence[int]] = None):
    """Exact per-group int32 partial sums -> int32 [K/G, R, N]."""
    qX = np.ascontiguousarray(qX, np.uint8)
    qW = np.ascontiguousarray(qW, np.uint8)
    M, K2 = qX.shape
    N = qW.shape[0]
    K = 2 * K2
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, np.int64))
    R = M if r is None else r.shape[0]
    P = np.empty((K // G, R, N), np.int32)
    _check(lib().orc_group_partials(_p(qX), _p(qW), M, N, K, G, _p(r), 0 if r is None else R, _p(P)),
           "group_partials")
    return P


def linear_rows(qX, s, scale_t, qW, scale_w, G: int, rows: Optional[Sequence[int]] = None
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Y (fp32) and the per-element summation bound for the listed rows."""
    qX = np.ascontiguousarray(qX, np.uint8)
    qW = np.ascontiguousarray(qW, np.uint8)
    s = _f32(s)
    st = _f32(scale_t)
    sw = _f32(scale_w)
    M, K2 = qX.shape
    N = qW.shape[0]
    K = 2 * K2
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, np.int64))
    R = M if r is None else r.shape[0]
    Y = np.empty((R, N), np.float32)
    B = np.empty((R, N), np.float64)
    _check(lib().orc_linear_rows(_p(qX), _p(s), _p(st), _p(qW), _p(sw), M, N, K, G, _p(r),
                                 0 if r is None else R, _p(Y), _p(B)), "linear_rows")
    return Y, B


def channel_absmax(X, n: int) -> np.ndarray:
    x = _f32(X)
    M, K = x.shape
    c = np.empty(K, np.float32)
    _check(lib().orc_channel_absmax(_p(x), M, K, n, _p(c)), "channel_absmax")
    return c


def calibrate_perm(X_cal, n: int) -> np.ndarray:
    """Reorder index from a calibration draw: channels sorted by descending
    max |X_rot|, ties by lower channel index (stable)."""
    c = channel_absmax(X_cal, n)
    return np.argsort(-c, kind="stable").astype(np.int32)


def unpack(q: np.ndarray, K: int) -> np.ndarray:
    """Packed nibbles -> int8 codes (inverse of the packing reading)."""
    q = np.asarray(q, np.uint8)
    lo = (q & 0x0F).astype(np.int16)
    hi = (q >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(q.shape[:-1] + (K,), np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def y_tolerance_ok(Y_gpu: np.ndarray, Y_orc: np.ndarray, bound: np.ndarray,
                   rel: float = 1e-3) -> np.ndarray:
    """Per-element acceptance of an fp32 Y against the oracle:
    |dY| <= rel*|Y| + 2^-20 * sum_g |s_g P_g| scale_t scale_w."""
    d = np.abs(Y_gpu.astype(np.float64) - Y_orc.astype(np.float64))
    return d <= rel * np.abs(Y_orc.astype(np.float64)) + (2.0 ** -20) * bound


def silu_mul(GU) -> np.ndarray:
    """The step between the two linears of a gated feed-forward block:
    H = silu(gate) * up, with gate = GU[:, :F] and up = GU[:, F:] of the fused gate/up
    projection's output, and silu(g) = g / (1 + exp(-g)).

    The block is the feed-forward block of the LLaMA models the pages evaluate
    (Rotated Runtime Smooth summary page, "Key results").  Its down projection takes an
    online Hadamard rotation of its input ("Understanding LLM Quantization through
    Activation-Guided Compensation and Orthogonal Residuals", Sec. 4.6).  Computed
    in fp64, saturated to the fp16 range +-65504, and rounded once to fp16 (round half
    to even): the down projection's fp16 activations.
    """
    gu = np.asarray(GU.detach().cpu().numpy() if hasattr(GU, "numpy") else GU, np.float64)
    F = gu.shape[1] // 2
    g, u = gu[:, :F], gu[:, F:]
    h = g / (1.0 + np.exp(-g)) * u
    return np.clip(h, -65504.0, 65504.0).astype(np.float16)


def kv_quant(KV):
    """KV-cache quantisation (the 4-4-4 setting) of fp16/fp32 KV [..., D]: every head
    vector rotated by the normalised Hadamard transform of size D, then per-vector
    symmetric INT4.  -> (codes int8 [..., D], q uint8 [..., D/2], scale fp32 [...])."""
    x = _f32(KV)
    lead = x.shape[:-1]
    D = x.shape[-1]
    x2 = np.ascontiguousarray(x.reshape(-1, D))
    rows = x2.shape[0]
    codes = np.empty((rows, D), np.int8)
    q = np.empty((rows, D // 2), np.uint8)
    scale = np.empty(rows, np.float32)
    _check(lib().orc_kv_quant(_p(x2), rows, D, _p(codes), _p(q), _p(scale)), "kv_quant")
    return codes.reshape(*lead, D), q.reshape(*lead, D // 2), scale.reshape(lead)


def kv_dequant(q, scale) -> np.ndarray:
    """code * scale in fp32, in the rotated space: q uint8 [..., D/2], scale [...] -> [..., D]."""
    qq = np.ascontiguousarray(np.asarray(q, np.uint8))
    lead = qq.shape[:-1]
    D = 2 * qq.shape[-1]
    q2 = qq.reshape(-1, D // 2)
    sc = np.ascontiguousarray(np.asarray(scale, np.float32).reshape(-1))
    out = np.empty((q2.shape[0], D), np.float32)
    _check(lib().orc_kv_dequant(_p(q2), q2.shape[0], D, _p(sc), _p(out)), "kv_dequant")
    return out.reshape(*lead, D)

"""ctypes binding of ``librrs.so`` (the C ABI in ``include/rrs.h``).

Argument marshalling only: shape/dtype/device checks, output allocation with
torch (device memory is the only thing torch provides here) and the call into
the library on torch's current CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no fallback.  If the library is
missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librrs.so")

NO_ROTATE = 1
FORCE_UNIT_SCALES = 2
WS_HOLDS_A8 = 4
W_EXPANDED = 8
Y_BF16 = 16
Y_SILU_MUL = 32
ONE_LAUNCH = 64

_STATUS = {
    0: "RRS_OK",
    1: "RRS_ERR_INVALID_ARG",
    2: "RRS_ERR_UNSUPPORTED",
    3: "RRS_ERR_CUDA",
    4: "RRS_ERR_TIMEOUT",
    5: "RRS_ERR_WORKSPACE",
}


class RRSError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status
        self.status_name = _STATUS.get(status, str(status))


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load librrs.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m activation_smoothing_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, U, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
    sigs = {
        "rrs_workspace_size": ([I, I, I, I, I, U], Z),
        "rrs_prepare_weights": ([P, I, I, I, P, P, P, U, P], I),
        "rrs_smooth_quant": ([P, I, I, I, I, P, P, P, P, P, Z, U, P], I),
        "rrs_group_max": ([P, I, I, I, I, P, P, P, Z, U, P], I),
        "rrs_smooth_quant_scaled": ([P, I, I, I, I, P, P, P, P, P, Z, U, P], I),
        "rrs_w4a4_gemm": ([P, P, P, P, P, I, I, I, I, P, P, Z, U, P], I),
        "rrs_linear": ([P, P, P, P, I, I, I, I, I, P, P, P, P, P, Z, U, P], I),
        "rrs_linear_from_host": ([P, P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, Z, U, P], I),
        "rrs_w4a4_gemm_debug_partials": ([P, P, I, I, I, I, P, P, Z, U, P], I),
        "rrs_expand_weights": ([P, I, I, P, P], I),
        "rrs_silu_mul": ([P, I, I, P, P], I),
        "rrs_channel_absmax": ([P, I, I, I, P, U, P], I),
        "rrs_kv_quant": ([P, I, I, I, P, P, U, P], I),
        "rrs_kv_dequant": ([P, P, I, I, I, P, P], I),
        "rrs_perm_from_channel_max": ([P, I, P], I),
        "rrs_check_workspace": ([P, P], I),
        "rrs_check_perm": ([P, I, P, Z, P], I),
        "rrs_debug_wait_timeout": ([I, P, Z, P], I),
        "rrs_debug_divide": ([P, P, I, P, P, P], I),
        "rrs_last_error_string": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sigs.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(status: int) -> None:
    if status != 0:
        msg = lib().rrs_last_error_string()
        raise RRSError(status, msg.decode() if msg else "")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Tuple[int, ...]) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(M: int, N: int, K: int, G: int, had_block: int, flags: int = 0) -> int:
    return int(lib().rrs_workspace_size(M, N, K, G, had_block, flags))


def make_workspace(M: int, N: int, K: int, G: int, had_block: int, flags: int = 0,
                   device: Optional[torch.device] = None) -> torch.Tensor:
    """A zero-filled workspace of the size the library asks for."""
    n = workspace_size(M, N, K, G, had_block, flags)
    return torch.zeros(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def prepare_weights(W: torch.Tensor, perm: torch.Tensor, had_block: int, flags: int = 0,
                    qW: Optional[torch.Tensor] = None, scale_w: Optional[torch.Tensor] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Offline weight path: fp16 W [N, K] -> (qW uint8 [N, K/2], scale_w fp32 [N])."""
    N, K = W.shape
    _need(W, "W", torch.float16, (N, K))
    _need(perm, "perm", torch.int32, (K,))
    qW = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device) if qW is None else qW
    scale_w = torch.empty(N, dtype=torch.float32, device=W.device) if scale_w is None else scale_w
    _need(qW, "qW", torch.uint8, (N, K // 2))
    _need(scale_w, "scale_w", torch.float32, (N,))
    _check(lib().rrs_prepare_weights(_ptr(W), N, K, had_block, _ptr(perm), _ptr(qW), _ptr(scale_w), flags,
                                     _stream(stream)))
    return qW, scale_w


def smooth_quant(X: torch.Tensor, perm: torch.Tensor, G: int, had_block: int, flags: int = 0,
                 qX: Optional[torch.Tensor] = None, s: Optional[torch.Tensor] = None,
                 scale_t: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Online activation path: fp16 X [M, K] -> (qX uint8 [M, K/2], s fp32 [K/G], scale_t fp32 [M])."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    _need(perm, "perm", torch.int32, (K,))
    dev = X.device
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if qX is None else qX
    s = torch.empty(max(K // G, 1), dtype=torch.float32, device=dev) if s is None else s
    scale_t = torch.empty(M, dtype=torch.float32, device=dev) if scale_t is None else scale_t
    ws = make_workspace(M, 1, K, G, had_block, flags, dev) if ws is None else ws
    _check(lib().rrs_smooth_quant(_ptr(X), M, K, G, had_block, _ptr(perm), _ptr(qX), _ptr(s), _ptr(scale_t),
                                  _ptr(ws), ws.numel(), flags, _stream(stream)))
    return qX, s, scale_t


def group_max(X: torch.Tensor, perm: torch.Tensor, G: int, had_block: int, flags: int = 0,
              s: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pass A of the activation path: s fp32 [K/G] = per-group max |X'| over these tokens."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    _need(perm, "perm", torch.int32, (K,))
    s = torch.empty(max(K // G, 1), dtype=torch.float32, device=X.device) if s is None else s
    ws = make_workspace(M, 0, K, G, had_block, flags, X.device) if ws is None else ws
    _check(lib().rrs_group_max(_ptr(X), M, K, G, had_block, _ptr(perm), _ptr(s), _ptr(ws), ws.numel(), flags,
                               _stream(stream)))
    return s


def smooth_quant_scaled(X: torch.Tensor, perm: torch.Tensor, s: torch.Tensor, G: int, had_block: int,
                        flags: int = 0, qX: Optional[torch.Tensor] = None, scale_t: Optional[torch.Tensor] = None,
                        ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Pass B: (qX uint8 [M, K/2], scale_t fp32 [M]) with the given group scales s [K/G]."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    _need(perm, "perm", torch.int32, (K,))
    _need(s, "s", torch.float32, (K // G,))
    dev = X.device
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if qX is None else qX
    scale_t = torch.empty(M, dtype=torch.float32, device=dev) if scale_t is None else scale_t
    ws = make_workspace(M, 0, K, G, had_block, flags, dev) if ws is None else ws
    _check(lib().rrs_smooth_quant_scaled(_ptr(X), M, K, G, had_block, _ptr(perm), _ptr(s), _ptr(qX), _ptr(scale_t),
                                         _ptr(ws), ws.numel(), flags, _stream(stream)))
    return qX, scale_t


def _y_flags(Y: Optional[torch.Tensor], flags: int) -> int:
    """A bf16 Y selects the bf16 output (RRS_Y_BF16)."""
    if Y is not None and Y.dtype == torch.bfloat16:
        return flags | Y_BF16
    return flags


def _y_dtype(flags: int) -> torch.dtype:
    if flags & Y_SILU_MUL:
        return torch.float16
    return torch.bfloat16 if flags & Y_BF16 else torch.float32


def _y_shape(M: int, N: int, flags: int) -> Tuple[int, int]:
    return (M, N // 2) if flags & Y_SILU_MUL else (M, N)


def interleave_gate_up(W_gate: torch.Tensor, W_up: torch.Tensor) -> torch.Tensor:
    """Weight rows of a gated MLP's fused gate/up projection in the order RRS_Y_SILU_MUL
    reads: row 2f = W_gate[f], row 2f + 1 = W_up[f]."""
    if W_gate.shape != W_up.shape:
        raise ValueError("gate and up weights must have the same shape")
    return torch.stack([W_gate, W_up], dim=1).reshape(2 * W_gate.shape[0], W_gate.shape[1]).contiguous()


def _need_weights(qW: torch.Tensor, N: int, K: int, flags: int):
    if flags & W_EXPANDED:
        _need(qW, "qW", torch.float8_e4m3fn, (N, K))
    else:
        _need(qW, "qW", torch.uint8, (N, K // 2))


def w4a4_gemm(qX: torch.Tensor, s: torch.Tensor, scale_t: torch.Tensor, qW: torch.Tensor,
              scale_w: torch.Tensor, G: int, Y: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, flags: int = 0, stream=None) -> torch.Tensor:
    """Group-scaled W4A4 GEMM -> Y fp32 [M, N].  flags=WS_HOLDS_A8 when ``ws`` is the
    workspace the preceding smooth_quant of this qX wrote (with the same W_EXPANDED bit;
    skips re-expanding qX); W_EXPANDED when ``qW`` is the e4m3 operand from expand_weights."""
    M, K2 = qX.shape
    N = qW.shape[0]
    K = 2 * K2
    _need(qX, "qX", torch.uint8, (M, K2))
    _need_weights(qW, N, K, flags)
    _need(s, "s", torch.float32, (K // G,))
    _need(scale_t, "scale_t", torch.float32, (M,))
    _need(scale_w, "scale_w", torch.float32, (N,))
    flags = _y_flags(Y, flags)
    Y = torch.empty(_y_shape(M, N, flags), dtype=_y_dtype(flags), device=qX.device) if Y is None else Y
    _need(Y, "Y", _y_dtype(flags), _y_shape(M, N, flags))
    ws = make_workspace(M, N, K, G, 1, 0, qX.device) if ws is None else ws
    _check(lib().rrs_w4a4_gemm(_ptr(qX), _ptr(s), _ptr(scale_t), _ptr(qW), _ptr(scale_w), M, N, K, G, _ptr(Y),
                               _ptr(ws), ws.numel(), flags, _stream(stream)))
    return Y


def linear(X: torch.Tensor, qW: torch.Tensor, scale_w: torch.Tensor, perm: torch.Tensor, G: int,
           had_block: int, flags: int = 0, Y: Optional[torch.Tensor] = None,
           qX: Optional[torch.Tensor] = None, s: Optional[torch.Tensor] = None,
           scale_t: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """RRS W4A4 linear: Y fp32 [M, N] from fp16 X [M, K] and prepared weights."""
    M, K = X.shape
    N = qW.shape[0]
    dev = X.device
    _need(X, "X", torch.float16, (M, K))
    _need_weights(qW, N, K, flags)
    _need(scale_w, "scale_w", torch.float32, (N,))
    _need(perm, "perm", torch.int32, (K,))
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if qX is None else qX
    s = torch.empty(max(K // G, 1), dtype=torch.float32, device=dev) if s is None else s
    scale_t = torch.empty(M, dtype=torch.float32, device=dev) if scale_t is None else scale_t
    flags = _y_flags(Y, flags)
    Y = torch.empty(_y_shape(M, N, flags), dtype=_y_dtype(flags), device=dev) if Y is None else Y
    _need(Y, "Y", _y_dtype(flags), _y_shape(M, N, flags))
    ws = make_workspace(M, N, K, G, had_block, flags, dev) if ws is None else ws
    _check(lib().rrs_linear(_ptr(X), _ptr(qW), _ptr(scale_w), _ptr(perm), M, N, K, G, had_block, _ptr(qX),
                            _ptr(s), _ptr(scale_t), _ptr(Y), _ptr(ws), ws.numel(), flags, _stream(stream)))
    return Y


def linear_from_host(X_host: torch.Tensor, X_dev: torch.Tensor, qW: torch.Tensor, scale_w: torch.Tensor,
                     perm: torch.Tensor, G: int, had_block: int, qX: torch.Tensor, s: torch.Tensor,
                     scale_t: torch.Tensor, Y_dev: torch.Tensor, Y_host: torch.Tensor, ws: torch.Tensor,
                     flags: int = 0, stream=None) -> torch.Tensor:
    """End to end from host memory: copies X_host in, runs the layer, copies Y out, syncs."""
    M, K = X_host.shape
    N = qW.shape[0]
    if X_host.device.type != "cpu" or Y_host.device.type != "cpu":
        raise ValueError("X_host and Y_host must be host tensors")
    flags = _y_flags(Y_dev, flags)
    if X_host.dtype != torch.float16 or Y_host.dtype != _y_dtype(flags):
        raise TypeError("X_host must be fp16 and Y_host of Y_dev's type (fp32 or bf16)")
    if tuple(Y_host.shape) != (M, N) or not X_host.is_contiguous() or not Y_host.is_contiguous():
        raise ValueError("host buffers must be contiguous with shapes [M, K] and [M, N]")
    _need(X_dev, "X_dev", torch.float16, (M, K))
    _need(Y_dev, "Y_dev", _y_dtype(flags), (M, N))
    _check(lib().rrs_linear_from_host(_ptr(X_host), _ptr(X_dev), _ptr(qW), _ptr(scale_w), _ptr(perm), M, N, K,
                                      G, had_block, _ptr(qX), _ptr(s), _ptr(scale_t), _ptr(Y_dev), _ptr(Y_host),
                                      _ptr(ws), ws.numel(), flags, _stream(stream)))
    return Y_host


def w4a4_gemm_debug_partials(qX: torch.Tensor, qW: torch.Tensor, G: int, P: Optional[torch.Tensor] = None,
                             ws: Optional[torch.Tensor] = None, flags: int = 0, stream=None) -> torch.Tensor:
    """Exact per-group int32 partial sums P [K/G, M, N] (debug, small problems)."""
    M, K2 = qX.shape
    N = qW.shape[0]
    K = 2 * K2
    _need(qX, "qX", torch.uint8, (M, K2))
    _need_weights(qW, N, K, flags)
    P = torch.empty((K // G, M, N), dtype=torch.int32, device=qX.device) if P is None else P
    _need(P, "P", torch.int32, (K // G, M, N))
    ws = make_workspace(M, N, K, G, 1, 0, qX.device) if ws is None else ws
    _check(lib().rrs_w4a4_gemm_debug_partials(_ptr(qX), _ptr(qW), M, N, K, G, _ptr(P), _ptr(ws), ws.numel(),
                                              flags & W_EXPANDED, _stream(stream)))
    return P


def silu_mul(GU: torch.Tensor, H: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fp16 H [M, F] = silu(GU[:, :F]) * GU[:, F:] from the fused gate/up output GU fp32 [M, 2F]."""
    M, F2 = GU.shape
    if F2 % 2:
        raise ValueError("GU must have an even number of columns [gate | up]")
    F = F2 // 2
    _need(GU, "GU", torch.float32, (M, F2))
    H = torch.empty((M, F), dtype=torch.float16, device=GU.device) if H is None else H
    _need(H, "H", torch.float16, (M, F))
    _check(lib().rrs_silu_mul(_ptr(GU), M, F, _ptr(H), _stream(stream)))
    return H


def expand_weights(qW: torch.Tensor, qW8: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The INT4 weight codes one per byte as e4m3 numbers [N, K] (natural k order; every
    code is exact in e4m3) from packed INT4 weights [N, K/2]; pass it with flags=W_EXPANDED."""
    N, K2 = qW.shape
    K = 2 * K2
    _need(qW, "qW", torch.uint8, (N, K2))
    qW8 = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=qW.device) if qW8 is None else qW8
    _need(qW8, "qW8", torch.float8_e4m3fn, (N, K))
    _check(lib().rrs_expand_weights(_ptr(qW), N, K, _ptr(qW8), _stream(stream)))
    return qW8


def kv_quant(KV: torch.Tensor, q: Optional[torch.Tensor] = None, scale: Optional[torch.Tensor] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """KV cache (4-4-4 setting): fp16 KV [T, H, D] -> (q uint8 [T, H, D/2], scale fp32 [T, H]),
    every head vector rotated by the normalised Hadamard transform of size D."""
    T, H, D = KV.shape
    _need(KV, "KV", torch.float16, (T, H, D))
    q = torch.empty((T, H, D // 2), dtype=torch.uint8, device=KV.device) if q is None else q
    scale = torch.empty((T, H), dtype=torch.float32, device=KV.device) if scale is None else scale
    _need(q, "q", torch.uint8, (T, H, D // 2))
    _need(scale, "scale", torch.float32, (T, H))
    _check(lib().rrs_kv_quant(_ptr(KV), T, H, D, _ptr(q), _ptr(scale), 0, _stream(stream)))
    return q, scale


def kv_dequant(q: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """fp16 [T, H, D] = code * scale, in the rotated space."""
    T, H, D2 = q.shape
    D = 2 * D2
    _need(q, "q", torch.uint8, (T, H, D2))
    _need(scale, "scale", torch.float32, (T, H))
    out = torch.empty((T, H, D), dtype=torch.float16, device=q.device) if out is None else out
    _need(out, "out", torch.float16, (T, H, D))
    _check(lib().rrs_kv_dequant(_ptr(q), _ptr(scale), T, H, D, _ptr(out), _stream(stream)))
    return out


def channel_absmax(X: torch.Tensor, had_block: int, flags: int = 0, cmax: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """cmax[k] = max over tokens of |X_rot[:, k]| (fp32 [K])."""
    M, K = X.shape
    _need(X, "X", torch.float16, (M, K))
    cmax = torch.empty(K, dtype=torch.float32, device=X.device) if cmax is None else cmax
    _need(cmax, "cmax", torch.float32, (K,))
    _check(lib().rrs_channel_absmax(_ptr(X), M, K, had_block, _ptr(cmax), flags, _stream(stream)))
    return cmax


def perm_from_channel_max(cmax_host: torch.Tensor) -> torch.Tensor:
    """Host: channels by descending statistic, ties by lower index -> int32 [K] (CPU)."""
    c = cmax_host.detach().to("cpu", torch.float32).contiguous()
    K = c.numel()
    perm = torch.empty(K, dtype=torch.int32)
    _check(lib().rrs_perm_from_channel_max(_ptr(c), K, _ptr(perm)))
    return perm


def calibrate_perm(X_cal: torch.Tensor, had_block: int, flags: int = 0) -> torch.Tensor:
    """Reorder index from a calibration batch (device int32 [K])."""
    cmax = channel_absmax(X_cal, had_block, flags)
    return perm_from_channel_max(cmax.cpu()).to(X_cal.device)


def check_workspace(ws: torch.Tensor, stream=None) -> None:
    """Synchronise and raise RRSError(RRS_ERR_TIMEOUT) if a kernel gave up on a wait."""
    _check(lib().rrs_check_workspace(_ptr(ws), _stream(stream)))


def check_perm(perm: torch.Tensor, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    """Raise RRSError(RRS_ERR_INVALID_ARG) unless the device int32 index perm [K] is a
    permutation of 0..K-1 (synchronises the stream)."""
    K = perm.numel()
    _need(perm, "perm", torch.int32, (K,))
    if ws is None:
        ws = torch.empty(256 + 16 + 4 * ((K + 31) // 32), dtype=torch.uint8, device=perm.device)
    _check(lib().rrs_check_perm(_ptr(perm), K, _ptr(ws), ws.numel(), _stream(stream)))


def debug_wait_timeout(limit_us: int, ws: torch.Tensor, stream=None) -> None:
    """Launch the fault-injection kernel (a wait that nothing releases, bounded by limit_us)."""
    _check(lib().rrs_debug_wait_timeout(limit_us, _ptr(ws), ws.numel(), _stream(stream)))


def debug_divide(a: torch.Tensor, b: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(division as the activation kernels compute it, IEEE division) for fp32 device vectors."""
    n = a.numel()
    _need(a, "a", torch.float32, (n,))
    _need(b, "b", torch.float32, (n,))
    qf = torch.empty_like(a)
    qi = torch.empty_like(a)
    _check(lib().rrs_debug_divide(_ptr(a), _ptr(b), n, _ptr(qf), _ptr(qi), _stream(stream)))
    return qf, qi

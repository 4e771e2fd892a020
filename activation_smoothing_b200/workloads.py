"""Seeded synthetic inputs for the RRS W4A4 linear layer.

This module only draws random tensors (activations X, weights W, reorder
indices).  It holds none of the method's arithmetic: no rotation, no
smoothing, no quantisation.  Both the CUDA path (through the benchmark) and
the CPU oracle (through the tests) consume what it returns.

The pages evaluate on real LLaMA activations from WikiText-2; neither data
set nor weights exist here, so these tensors stand in for them.  They carry
the two outlier kinds the method targets (Rotated Runtime Smooth summary
page, "Problem" and "Approach"): channel-wise outliers (a fixed set of
channels scaled up for every token) and spike outliers (a few very large
elements on a few tokens).

Recipe (all draws on the CPU with ``torch.Generator``, fp32, then cast to
fp16 with saturation to +-65504):

* X ~ N(0, 1) per element, times a per-channel magnitude (1, or LogNormal(0,
  sigma) for down projections), with round(1% of K) seeded channels x50 and
  round(0.01% of M*K) spikes x500 placed uniformly over the non-outlier
  channels of min(M, 4) seeded token rows.
* W ~ N(0, 0.02^2) per element.
* The outlier channel set and channel magnitudes depend on the layer seed
  only; the noise and the spike positions also depend on the sample index,
  so a calibration draw (sample=1) shares the layer's channel structure.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

FP16_MAX = 65504.0


@dataclasses.dataclass(frozen=True)
class Layer:
    """One linear layer workload: Y[M, N] = X[M, K] . W[N, K]^T."""

    name: str
    M: int
    K: int
    N: int
    G: int
    had_block: int          # Hadamard block size n (1 = no rotation, plain Runtime Smooth)
    seed: int
    lognormal_sigma: Optional[float] = None
    tiny: bool = False

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


def _tiny_activations(M: int, K: int, seed: int, sample: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed + 7919 * sample)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    x[:, 3] *= 50.0
    x[:, 77 % K] *= 50.0
    if M > 5 and K > 10:
        x[5, 10] = 400.0
    return x.to(torch.float16)


def make_activations(layer: Layer, sample: int = 0, M: Optional[int] = None) -> torch.Tensor:
    """fp16 [M, K] activations for ``layer`` (row-major, CPU)."""
    M = layer.M if M is None else M
    K = layer.K
    if layer.tiny:
        return _tiny_activations(M, K, layer.seed, sample)
    gs = torch.Generator().manual_seed(layer.seed)
    n_out = int(round(0.01 * K))
    out_ch = torch.randperm(K, generator=gs)[:n_out]
    colscale = torch.ones(K, dtype=torch.float32)
    if layer.lognormal_sigma:
        colscale = torch.exp(layer.lognormal_sigma * torch.randn(K, generator=gs))
    colscale[out_ch] *= 50.0

    gx = torch.Generator().manual_seed(layer.seed * 1009 + 104729 * (sample + 1))
    x = torch.randn(M, K, generator=gx, dtype=torch.float32) * colscale

    n_spike_rows = min(M, 4)
    spike_rows = torch.randperm(M, generator=gx)[:n_spike_rows]
    normal = torch.ones(K, dtype=torch.bool)
    normal[out_ch] = False
    normal_ch = torch.nonzero(normal).flatten()
    n_spikes = max(1, int(round(1e-4 * M * K)))
    cand = n_spike_rows * normal_ch.numel()
    pick = torch.randperm(cand, generator=gx)[:n_spikes]
    r = spike_rows[pick // normal_ch.numel()]
    c = normal_ch[pick % normal_ch.numel()]
    x[r, c] *= 500.0
    return x.clamp_(-FP16_MAX, FP16_MAX).to(torch.float16)


def make_weights(layer: Layer, N: Optional[int] = None) -> torch.Tensor:
    """fp16 [N, K] weights, N(0, 0.02^2) per element."""
    N = layer.N if N is None else N
    g = torch.Generator().manual_seed(layer.seed + 500_000)
    w = torch.randn(N, layer.K, generator=g, dtype=torch.float32) * 0.02
    return w.to(torch.float16)


def identity_perm(K: int) -> torch.Tensor:
    return torch.arange(K, dtype=torch.int32)


def random_perm(K: int, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(K, generator=g).to(torch.int32)


def saturated_count(x32: torch.Tensor) -> int:
    return int((x32.abs() >= FP16_MAX).sum())


def _layers() -> Dict[str, Layer]:
    L: Dict[str, Layer] = {}

    def add(layer: Layer) -> None:
        L[layer.name] = layer

    # Tiny case: channels 3 and 77 x50, one spike of 400 at (token 5, channel 10).
    add(Layer("tiny", 16, 256, 256, 128, 256, seed=0, tiny=True))
    # LLaMA-3-8B attention and MLP input projections.
    add(Layer("llama3_8b_qo", 2048, 4096, 4096, 128, 4096, seed=1000))
    add(Layer("llama3_8b_kv", 2048, 4096, 1024, 128, 4096, seed=1001))
    add(Layer("llama3_8b_gateup", 2048, 4096, 14336, 128, 4096, seed=1002))
    # LLaMA-3-8B down projection: 7 Hadamard blocks of 2048, log-normal channel magnitudes.
    add(Layer("llama3_8b_down", 2048, 14336, 4096, 128, 2048, seed=2000, lognormal_sigma=1.5))
    # LLaMA-3-70B.
    add(Layer("llama3_70b_qo", 4096, 8192, 8192, 128, 8192, seed=3000))
    add(Layer("llama3_70b_gateup", 4096, 8192, 28672, 128, 8192, seed=3001))
    add(Layer("llama3_70b_down", 4096, 28672, 8192, 128, 4096, seed=3002, lognormal_sigma=1.5))
    for m in (1, 8, 16):
        add(Layer(f"llama3_70b_qo_decode_m{m}", m, 8192, 8192, 128, 8192, seed=3100 + m))
        add(Layer(f"llama3_70b_gateup_decode_m{m}", m, 8192, 28672, 128, 8192, seed=3200 + m))
        add(Layer(f"llama3_70b_down_decode_m{m}", m, 28672, 8192, 128, 4096, seed=3300 + m,
                  lognormal_sigma=1.5))
    # Group-size sweep on the gate/up shape, with (RRS) and without (RS) rotation.
    for G in (128, 256, 512, 4096):
        add(Layer(f"sweep_g{G}_rrs", 2048, 4096, 14336, G, 4096, seed=4000 + G))
        add(Layer(f"sweep_g{G}_rs", 2048, 4096, 14336, G, 1, seed=4000 + G))
    return L


LAYERS: Dict[str, Layer] = _layers()

# The three LLaMA-3-8B projection shapes the headline metric is quoted on.
HEADLINE: List[str] = ["llama3_8b_qo", "llama3_8b_kv", "llama3_8b_gateup"]

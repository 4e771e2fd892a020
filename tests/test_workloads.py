"""The seeded synthetic inputs follow the stated recipe (CPU only).

The inputs stand in for the pages' real LLaMA activations, which carry channel-wise
outliers and spike outliers (Rotated Runtime Smooth summary page, "Problem").  These
tests check the recipe the inputs are documented with: 1% of channels x50, shared by
every draw of a layer; 0.01% spikes x500 confined to min(M, 4) token rows; W ~ N(0, 0.02^2);
fp16 saturation; determinism by seed; the tiny case's fixed outliers.
"""
import numpy as np
import torch

from activation_smoothing_b200 import workloads as wl


def _outlier_channels(X: np.ndarray) -> np.ndarray:
    # channel-wise x50 outliers stand far above N(0, 1) in their median magnitude
    return np.nonzero(np.median(np.abs(X), axis=0) > 10.0)[0]


def test_channel_outliers_one_percent_and_shared_by_draws():
    L = wl.LAYERS["llama3_8b_qo"]
    X0 = wl.make_activations(L, M=256).float().numpy()
    X1 = wl.make_activations(L, sample=1, M=256).float().numpy()
    ch0, ch1 = _outlier_channels(X0), _outlier_channels(X1)
    assert ch0.size == round(0.01 * L.K)
    assert np.array_equal(ch0, ch1)                      # the calibration draw shares them
    assert not np.array_equal(X0, X1)                    # but its noise differs


def test_spikes_confined_to_four_rows():
    L = wl.LAYERS["llama3_8b_qo"]
    M = 512
    X = wl.make_activations(L, M=M).float().numpy()
    normal = np.setdiff1d(np.arange(L.K), _outlier_channels(X))
    big = np.abs(X[:, normal]) > 50.0                    # N(0, 1) never reaches 50 here
    rows = np.unique(np.nonzero(big)[0])
    n_spikes = round(1e-4 * M * L.K)
    assert 1 <= rows.size <= min(M, 4)
    assert 0.7 * n_spikes <= big.sum() <= n_spikes       # a spike of a small base value stays below 50


def test_weights_scale_and_determinism():
    L = wl.LAYERS["llama3_8b_kv"]
    W = wl.make_weights(L, N=128).float().numpy()
    assert abs(W.std() - 0.02) < 0.001 and abs(W.mean()) < 0.001
    assert np.array_equal(W, wl.make_weights(L, N=128).float().numpy())
    X = wl.make_activations(L, M=64)
    assert torch.equal(X, wl.make_activations(L, M=64))


def test_fp16_saturation_keeps_values_finite():
    L = wl.LAYERS["llama3_8b_down"]                      # log-normal channel magnitudes
    X = wl.make_activations(L, M=64)
    assert X.dtype == torch.float16
    assert torch.isfinite(X).all()
    assert float(X.abs().max()) <= wl.FP16_MAX


def test_tiny_case_fixed_outliers():
    L = wl.LAYERS["tiny"]
    X = wl.make_activations(L).float().numpy()
    assert X.shape == (16, 256)
    assert X[5, 10] == 400.0
    med = np.median(np.abs(X), axis=0)
    assert set(np.nonzero(med > 10.0)[0]) == {3, 77}


def test_headline_shapes():
    shapes = [(wl.LAYERS[n].M, wl.LAYERS[n].K, wl.LAYERS[n].N, wl.LAYERS[n].G, wl.LAYERS[n].had_block)
              for n in wl.HEADLINE]
    assert shapes == [(2048, 4096, 4096, 128, 4096), (2048, 4096, 1024, 128, 4096),
                      (2048, 4096, 14336, 128, 4096)]

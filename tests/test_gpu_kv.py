"""KV cache of the 4-4-4 setting on the CUDA path (needs a GPU): codes and scales
bit-exact with the oracle, the reconstruction equal to the oracle's rounded to
fp16, on outlier-laden head vectors, ragged token counts and several head sizes."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def rrs():
    import activation_smoothing_b200 as m
    m.lib()
    return m


def _kv(T, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, D, generator=g)
    x[:, :, 5] *= 50.0                    # a channel-wise outlier in every head
    x[T // 3, H - 1, 17] = 3000.0         # a spike
    if T > 4:
        x[4, 0] = 0.0                     # an all-zero head vector: scale 0, codes 0
    return x.clamp(-65504, 65504).to(torch.float16)


# D = 128, 256, 512 take the warp-per-vector kernel (with vector counts that are not a
# multiple of its per-warp batch), D = 1024 the general activation kernels
@pytest.mark.parametrize("T,H,D", [(64, 8, 128), (33, 4, 256), (1, 1, 128), (517, 8, 128), (7, 2, 512),
                                   (3, 3, 128), (5, 2, 1024)])
def test_kv_quant_bit_exact(rrs, T, H, D):
    x = _kv(T, H, D, T * 7 + D)
    q, sc = rrs.kv_quant(x.to(DEV))
    back = rrs.kv_dequant(q, sc)
    torch.cuda.synchronize()
    _, oq, osc = oracle.kv_quant(x)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), osc.view(np.uint32))
    ref = oracle.kv_dequant(oq, osc).astype(np.float16)
    assert np.array_equal(back.cpu().numpy().view(np.uint16), ref.view(np.uint16))


def test_kv_quant_rejects_bad_sizes(rrs):
    x = torch.zeros(4, 2, 64, dtype=torch.float16, device=DEV)
    with pytest.raises(rrs.RRSError) as e:
        rrs.kv_quant(x)
    assert e.value.status_name == "RRS_ERR_UNSUPPORTED"


@pytest.mark.parametrize("T,H,D", [(9, 3, 40), (4, 2, 32), (130, 1, 64)])
def test_kv_dequant_of_any_codes(rrs, T, H, D):
    """The way back for head sizes the quantiser does not take (D a multiple of 8,
    or a power of two below 128): fp16(code * scale) against the oracle's fp32
    reconstruction rounded to fp16."""
    rng = np.random.default_rng(T * H + D)
    q = rng.integers(0, 256, size=(T, H, D // 2), dtype=np.uint8)
    sc = (rng.random((T, H), dtype=np.float32) * 3).astype(np.float32)
    sc[0, 0] = 0.0
    back = rrs.kv_dequant(torch.from_numpy(q).to(DEV), torch.from_numpy(sc).to(DEV))
    torch.cuda.synchronize()
    ref = oracle.kv_dequant(q, sc).astype(np.float16)
    assert np.array_equal(back.cpu().numpy().view(np.uint16), ref.view(np.uint16))

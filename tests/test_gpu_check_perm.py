"""GPU: the debug check of the reorder index (a valid permutation of 0..K-1)."""
import pytest
import torch

import activation_smoothing_b200 as rrs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K", [1, 100, 4096, 28672])
def test_valid_permutations_pass(K):
    g = torch.Generator().manual_seed(K)
    rrs.check_perm(torch.arange(K, dtype=torch.int32, device="cuda"))
    rrs.check_perm(torch.randperm(K, generator=g).to(torch.int32).cuda())


def test_repeated_value_names_the_missing_one():
    K = 4096
    p = torch.randperm(K, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    where = int((p == 777).nonzero()[0, 0])
    p[where] = 12                                   # 12 twice, 777 nowhere
    with pytest.raises(rrs.RRSError) as e:
        rrs.check_perm(p.cuda())
    assert e.value.status == 1 and "no position holds 777" in str(e.value)


@pytest.mark.parametrize("bad", [-1, 4096, 1 << 30])
def test_out_of_range_value_names_the_first_position(bad):
    K = 4096
    p = torch.arange(K, dtype=torch.int32)
    p[3000] = bad
    p[3500] = bad
    with pytest.raises(rrs.RRSError) as e:
        rrs.check_perm(p.cuda())
    assert e.value.status == 1 and "perm[3000]" in str(e.value)


def test_ragged_tail_word_is_checked():
    K = 100                                         # the last bitmap word holds 4 values
    p = torch.arange(K, dtype=torch.int32)
    p[99] = 98
    with pytest.raises(rrs.RRSError) as e:
        rrs.check_perm(p.cuda())
    assert "no position holds 99" in str(e.value)


def test_workspace_error_word_is_left_alone():
    K = 4096
    ws = rrs.make_workspace(1, 0, K, 128, K)
    ws[:4] = 0
    rrs.check_perm(torch.arange(K, dtype=torch.int32, device="cuda"), ws=ws)
    rrs.check_workspace(ws)

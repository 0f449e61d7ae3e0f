"""GPU: the allocation-free grouping call against the workspace one.

moe_group_tokens_static serves callers that cannot allocate device memory
where they call the library; its scratch is a fixed array inside the
library.  It must give exactly the results of moe_group_tokens, call after
call (the array keeps the previous call's contents), and refuse sizes
beyond its fixed maximum.  This file is named to run last.
"""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import dev, run_group

pytestmark = pytest.mark.gpu


def _static_group(idx, E, err=None):
    T, k = idx.shape
    d_idx = dev(idx.astype(np.int32))
    off = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    pairs = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    act = torch.full((E,), -9, dtype=torch.int32, device="cuda")
    na = torch.full((1,), -9, dtype=torch.int32, device="cuda")
    moe.moe_group_tokens_static(d_idx, T, k, E, off, pairs, act, na, err)
    torch.cuda.synchronize()
    n = int(na.item())
    return off.cpu().numpy(), pairs.cpu().numpy(), act.cpu().numpy()[:n]


@pytest.mark.parametrize("T,k,E", [(3, 10, 512), (2000, 10, 512),
                                   (9536, 10, 512), (700, 8, 1024)])
def test_static_grouping_matches_workspace_grouping(T, k, E):
    rng = np.random.default_rng(T + E)
    p = synth.zipf_popularity(E)[rng.permutation(E)]
    a = np.array([rng.choice(E, k, replace=False, p=p) for _ in range(T)])
    b = np.array([rng.choice(E, k, replace=False) for _ in range(T)])
    for idx in (a, b):        # two calls in a row on different inputs
        off, pairs, act, err, _ = run_group(idx, E)
        assert err == 0
        s_off, s_pairs, s_act = _static_group(idx, E)
        assert np.array_equal(s_off, off)
        assert np.array_equal(s_pairs, pairs)
        assert np.array_equal(s_act, act)
        r_off, r_pairs, r_act = o.group_pairs(idx, E)
        assert np.array_equal(s_pairs, r_pairs)


def test_static_grouping_at_capacity_allocates_nothing():
    """The largest sizes the fixed array holds (T*k = 262144 pairs over
    E = 1024 experts fill every per-chunk histogram row), against the
    workspace call; and the device's free memory is the same before and
    after a call (the call itself allocates nothing)."""
    T, k, E = 32768, 8, 1024
    rng = np.random.default_rng(5)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    off, pairs, act, err, _ = run_group(idx, E)
    assert err == 0
    d_idx = dev(idx)
    s_off = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    s_pairs = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    s_act = torch.full((E,), -9, dtype=torch.int32, device="cuda")
    na = torch.full((1,), -9, dtype=torch.int32, device="cuda")
    for _ in range(2):      # the first call has looked the array up
        moe.moe_group_tokens_static(d_idx, T, k, E, s_off, s_pairs, s_act,
                                    na, None)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        used0 = torch.cuda.memory_allocated()
        s_pairs.fill_(-9)
        moe.moe_group_tokens_static(d_idx, T, k, E, s_off, s_pairs, s_act,
                                    na, None)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        assert torch.cuda.memory_allocated() == used0
        assert np.array_equal(s_off.cpu().numpy(), off)
        assert np.array_equal(s_pairs.cpu().numpy(), pairs)
        assert np.array_equal(s_act.cpu().numpy()[:int(na.item())], act)


def test_static_grouping_reports_bad_ids_and_rejects_large_sizes():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = np.array([[0, 3], [99, 1]], np.int32)
    off, pairs, act = _static_group(idx, 8, err)
    assert int(err.item()) == moe.MOE_ERR_DEVICE
    assert act.tolist() == [0, 1, 3]
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_group_tokens_static(z, 262145, 1, 8, z, z, z, z, None)
    assert ei.value.code == moe.MOE_ERR_SHAPE
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_group_tokens_static(z, 4, 2, 1025, z, z, z, z, None)
    assert ei.value.code == moe.MOE_ERR_SHAPE

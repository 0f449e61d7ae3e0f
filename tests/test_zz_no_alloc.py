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

"""Plan parity (block partition and window lists): the GPU block partition and window lists are bit-exact with the
oracle's, through the C ABI (ssa_plan / ssa_plan_varlen / ssa_plan_export)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import coords_of, make_plan

pytestmark = pytest.mark.gpu


def _compare(coords, cu, grids, r):
    plan = make_plan(coords, cu, grids, r)
    got = {k: v.cpu().numpy() for k, v in plan.export().items()}
    ref = oracle.plan(coords, cu, 8, r)
    for key in ("perm", "tok_blk", "blk_off", "blk_coord", "blk_seq", "nbr_off", "nbr_idx"):
        assert np.array_equal(got[key], ref[key].astype(got[key].dtype)), key
    assert plan.num_blocks == len(ref["blk_coord"]) and plan.nnz == len(ref["nbr_idx"])
    return plan


@pytest.mark.parametrize("name", ["tiny", "small", "pass1", "pass3", "varlen"])
def test_plan_bit_exact(name):
    c, cu, g = coords_of(name)
    _compare(c, cu, g, workloads.CONFIGS[name].radius)


@pytest.mark.parametrize("r", [0, 1, 4, 8])
def test_plan_radii_and_shuffled_order(r):
    c, cu, g = coords_of("small")
    p = np.random.default_rng(r).permutation(len(c))
    _compare(c[p], cu, g, r)


def test_plan_varlen_with_empty_and_single_token_sequences():
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    _compare(c, cu, grids, 2)


def test_plan_grid_not_multiple_of_block():
    rng = np.random.default_rng(5)
    cells = rng.choice(13 * 21 * 30, 900, replace=False)
    c = np.stack([cells // (21 * 30), (cells // 30) % 21, cells % 30], 1).astype(np.int32)
    _compare(c, np.array([0, len(c)]), np.array([[13, 21, 30]], np.int32), 3)


def test_plan_errors():
    import spatial_sparse_attention_b200 as ssa
    dup = torch.tensor([[1, 2, 3], [4, 5, 6], [1, 2, 3]], dtype=torch.int32, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        ssa.Plan(dup, grid=(8, 8, 8), r=1)
    assert e.value.name == "SSA_ERR_DUPLICATE_COORD"
    bad = torch.tensor([[1, 2, 3], [4, 5, 8]], dtype=torch.int32, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        ssa.Plan(bad, grid=(8, 8, 8), r=1)
    assert e.value.name == "SSA_ERR_COORD_RANGE"
    neg = torch.tensor([[1, -2, 3]], dtype=torch.int32, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        ssa.Plan(neg, grid=(8, 8, 8), r=1)
    assert e.value.name == "SSA_ERR_COORD_RANGE"
    ok = torch.tensor([[1, 2, 3]], dtype=torch.int32, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        ssa.Plan(ok, grid=(8, 8, 8), r=1, block=4)
    assert e.value.name == "SSA_ERR_UNSUPPORTED"
    # a plan built after the errors works
    p = ssa.Plan(ok, grid=(8, 8, 8), r=1)
    assert p.num_blocks == 1 and p.nnz == 1

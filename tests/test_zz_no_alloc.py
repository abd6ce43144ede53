"""The no-allocation entry point ssa_block_offsets_noalloc against the plan's block offsets.

Collected last (file name): it shares a fixed device scratch array inside the library, and must
give the plan's result on two calls in a row (the second call starts from the first one's leftover
counters, which it has to clear itself), whether it runs alone or after the other tests.
"""
import numpy as np
import pytest
import torch

import workloads
from ssa_testlib import coords_of, make_plan

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "small", "pass3"])
def test_noalloc_block_offsets_match_plan_twice(name):
    import spatial_sparse_attention_b200 as ssa
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    plan = make_plan(c, cu, g, cfg.radius)
    ref = plan.export()["blk_off"].cpu().numpy()
    cd = torch.from_numpy(np.ascontiguousarray(c, dtype=np.int32)).cuda()
    for _ in range(2):
        blk_off, nb = ssa.block_offsets_noalloc(cd, tuple(int(x) for x in g[0]))
        torch.cuda.synchronize()
        assert nb == len(ref) - 1
        np.testing.assert_array_equal(blk_off.cpu().numpy(), ref)


def test_noalloc_rejects_and_flags():
    import spatial_sparse_attention_b200 as ssa
    c, cu, g = coords_of("small")
    cd = torch.from_numpy(np.ascontiguousarray(c, dtype=np.int32)).cuda()
    # more grid blocks than the fixed scratch holds (2^21): rejected before any device work
    with pytest.raises(ssa.SSAError, match="UNSUPPORTED"):
        ssa.block_offsets_noalloc(cd, (2048, 2048, 1024))
    # a coordinate outside the grid is reported through n_blocks = -1
    bad = cd.clone()
    bad[5, 0] = int(g[0][0])
    _, nb = ssa.block_offsets_noalloc(bad, tuple(int(x) for x in g[0]))
    assert nb == -1
    # and the next call with good coordinates is unaffected
    blk_off, nb = ssa.block_offsets_noalloc(cd, tuple(int(x) for x in g[0]))
    assert nb > 0 and int(blk_off[-1]) == len(c)

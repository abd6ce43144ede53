"""Parity of ssa_forward_prologue (Hi3D v1.0 pipeline page, "Stage 3: sparse flow sampling": RMS
normalisation and rotary position embedding of the self-attention queries and keys, applied
before SSA) against the fp64 oracle with the same prologue, through the C ABI.

The GPU rounds the transformed queries and keys to the input type before the tensor cores use
them; the oracle keeps them unrounded. Every compared row is compared on every element, with the
oracle evaluated on the GPU's validated selection.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import (check_close, coords_of, make_plan, oracle_on_gpu_selection, tensors_of,
                         tile_rows, to_gpu)

pytestmark = pytest.mark.gpu


def _weights(D, seed):
    rng = np.random.default_rng(seed)
    return {"q_gamma": torch.from_numpy(rng.random(D).astype(np.float32) + 0.5),
            "k_gamma": torch.from_numpy(rng.random(D).astype(np.float32) + 0.5)}


def run_and_compare(name, c, cu, grids, t, topk, r, dtype, theta, rows=None, seed=0):
    D = t["Q"].shape[2]
    w = _weights(D, seed)
    plan = make_plan(c, cu, grids, r)
    g = to_gpu(t)
    out, sel = plan.forward_prologue(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], topk,
                                     w["q_gamma"].cuda(), w["k_gamma"].cuda(), rope_theta=theta,
                                     eps=1e-6, return_sel=True)
    torch.cuda.synchronize()
    assert plan.status() == 0
    pro = dict(q_gamma=w["q_gamma"], k_gamma=w["k_gamma"], eps=1e-6, theta=theta)
    bs = plan.export()["blk_seq"].cpu().numpy()
    ref, _ = oracle_on_gpu_selection(c, cu, t, topk, r, sel.cpu().numpy(), bs, dtype, rows=rows,
                                     prologue=pro)
    R = ref["rows"]
    got = out[torch.from_numpy(R).cuda()].double().cpu().numpy()
    check_close(got, ref["out"], dtype, f"{name} prologue out")
    # the prologue is applied: the result differs from the plain forward
    plain = plan.forward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], topk)
    assert (plain - out).abs().max().item() > 1e-2


@pytest.mark.parametrize("name,dtype", [("tiny", "f32"), ("small", "bf16"), ("small", "f16")])
@pytest.mark.parametrize("theta", [10000.0, 100.0])
def test_prologue_full_output(name, dtype, theta):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = dict(tensors_of(name))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    for key in ("Q", "K", "V"):
        t[key] = t[key].float().to(tdt)
    run_and_compare(name, c, cu, g, t, cfg.topk, cfg.radius, dtype, theta, seed=cfg.index)


def test_prologue_head_dims_and_ragged_varlen():
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:1333]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    for D, dtype in ((32, "f16"), (64, "bf16"), (128, "f16"), (64, "f32")):
        cfg = workloads.WorkloadConfig("pro", 12, (), H=3, D=D, dtype=dtype, topk=5, radius=2)
        t = workloads.make_tensors(cfg, len(c))
        run_and_compare(f"D={D} {dtype}", c, cu, grids, t, 5, 2, dtype, 1000.0, seed=D)


@pytest.mark.slow
def test_prologue_full_size_every_query_tile():
    """The headline workload (110k tokens, 22 heads, fp16) with the prologue: every head of rows
    from every 128-token query tile."""
    cfg = workloads.CONFIGS["pass3"]
    c, cu, g = coords_of("pass3")
    perm = oracle.plan(c, cu, 8, cfg.radius)["perm"]
    rows = tile_rows(perm, cu, seed=cfg.index * 1000 + 97)
    run_and_compare("pass3", c, cu, g, tensors_of("pass3"), cfg.topk, cfg.radius, cfg.dtype,
                    10000.0, rows=rows, seed=4)

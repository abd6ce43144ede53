"""Backward parity of the CUDA path against the fp64 oracle, through the C ABI.

The oracle holds the GPU's selection (validated against its own: equal sets or near ties within
the stated gap), so every element is compared. Small configurations: every element of dQ, dK, dV.
The varlen batch (4 shapes, 340k tokens, H=22, D=96, fp16): dQ on 512 sampled rows per shape for
every head (dQ of a row depends only on that row), dQ, dK and dV on every row of one seeded head
(the oracle's full backward on that head alone: heads are independent), and the sums over all
tokens of dK and dV, which hold at any size: sum_j dK_j = 0 per head, and
sum_j dV_j = sum_i (g0_i dO_i Wc^T + (g1_i + g2_i) dO_i) per head.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import (check_grad_close, coords_of, head_slice, make_plan, rel_l2, tensors_of,
                         to_gpu, validate_gpu_selection)

pytestmark = pytest.mark.gpu


def gpu_backward(plan, t, topk):
    """GPU gradients (CUDA tensors) and the GPU's selection ([N, H, k] numpy)."""
    g = to_gpu(t)
    dq, dk, dv = plan.backward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], g["dO"], topk)
    _, sel = plan.forward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], topk, return_sel=True)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return dq, dk, dv, sel.cpu().numpy()


def _np(x, rows=None, heads=None):
    if rows is not None:
        x = x[torch.from_numpy(np.asarray(rows)).to(x.device)]
    if heads is not None:
        x = x[:, list(heads)]
    return x.double().cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_backward_full(name):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = tensors_of(name, with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    dq, dk, dv, sel = gpu_backward(plan, t, cfg.topk)
    bs = plan.export()["blk_seq"].cpu().numpy()
    validate_gpu_selection(c, cu, t, cfg.topk, cfg.radius, sel, bs, cfg.dtype)
    ref = oracle.backward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"], cfg.topk,
                          cfg.radius, sel=sel)
    check_grad_close(_np(dq), ref[0], cfg.dtype, "dQ")
    check_grad_close(_np(dk), ref[1], cfg.dtype, "dK")
    check_grad_close(_np(dv), ref[2], cfg.dtype, "dV")


@pytest.mark.slow
def test_backward_varlen_rows_one_head_in_full_and_sums():
    cfg = workloads.CONFIGS["varlen"]
    c, cu, g = coords_of("varlen")
    t = tensors_of("varlen", with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    dq, dk, dv, sel = gpu_backward(plan, t, cfg.topk)
    bs = plan.export()["blk_seq"].cpu().numpy()
    # dQ of 512 sampled rows per shape, every head
    rows = np.concatenate(workloads.stratified_rows(cu, 512, seed=5099))
    gs, _ = validate_gpu_selection(c, cu, t, cfg.topk, cfg.radius, sel, bs, cfg.dtype, rows=rows)
    ref = oracle.backward_dq_rows(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"],
                                  cfg.topk, cfg.radius, rows, sel_in=gs)
    check_grad_close(_np(dq, rows), ref, cfg.dtype, "dQ rows")
    # dQ, dK, dV of every row of one head
    h = int(np.random.default_rng(5098).integers(cfg.H))
    gs, _ = validate_gpu_selection(c, cu, t, cfg.topk, cfg.radius, sel, bs, cfg.dtype, heads=[h])
    th = head_slice(t, [h])
    full = oracle.backward(c, cu, th["Q"], th["K"], th["V"], th["gates"], th["Wc"], th["dO"],
                           cfg.topk, cfg.radius, sel=gs)
    for x, r, nm in zip((dq, dk, dv), full, ("dQ", "dK", "dV")):
        check_grad_close(_np(x, heads=[h]), r, cfg.dtype, f"{nm} head {h}")
    # sums over all tokens, every head
    dk, dv = _np(dk), _np(dv)
    gates = t["gates"].double().numpy()
    dO = t["dO"].double().numpy()
    Wc = t["Wc"].double().numpy()
    for s in range(len(cu) - 1):
        lo, hi = cu[s], cu[s + 1]
        sk = dk[lo:hi].sum(0)
        # exact sum is zero; allow the rounding of N fp16 gradients (relative to sum |dK_j|)
        assert np.abs(sk).max() <= 1e-3 * np.abs(dk[lo:hi]).sum(0).max()
        exp = (np.einsum("nh,nhd->hd", gates[lo:hi, :, 0], dO[lo:hi]) @ Wc.T
               + np.einsum("nh,nhd->hd", gates[lo:hi, :, 1] + gates[lo:hi, :, 2], dO[lo:hi]))
        assert rel_l2(dv[lo:hi].sum(0), exp) <= 5e-3


def test_backward_head_dims_and_ragged_varlen():
    """Every element of dQ, dK, dV on a ragged batch (an empty and a one-token sequence among two
    shells) for head dims 32-128 in each input type: the compressed branch's GEMMs meet sequences
    of one row and one block, and batches of heads of every size."""
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:1333]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    for D, dtype, k in ((128, "f16", 5), (96, "bf16", 3), (32, "f32", 4)):
        cfg = workloads.WorkloadConfig("bwd", 19, (), H=3, D=D, dtype=dtype, topk=k, radius=2)
        t = workloads.make_tensors(cfg, len(c), with_grad_out=True)
        plan = make_plan(c, cu, grids, 2)
        dq, dk, dv, sel = gpu_backward(plan, t, k)
        bs = plan.export()["blk_seq"].cpu().numpy()
        gs, _ = validate_gpu_selection(c, cu, t, k, 2, sel, bs, dtype)
        ref = oracle.backward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"], k, 2, sel=gs)
        for x, r, nm in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            check_grad_close(_np(x), r, dtype, f"D={D} {dtype} {nm}")

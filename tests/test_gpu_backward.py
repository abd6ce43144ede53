"""Backward parity (row a9) of the CUDA path against the fp64 oracle, through the C ABI.

Small configurations: every element of dQ, dK, dV. The varlen batch (4 shapes, 340k tokens,
H=22, D=96, fp16): dQ on 512 sampled rows per shape (dQ of a row depends only on that row), and
for dK, dV the sums over all tokens, which hold at any size: sum_j dK_j = 0 per head, and
sum_j dV_j = sum_i (g0_i dO_i Wc^T + (g1_i + g2_i) dO_i) per head.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import check_grad_close, coords_of, make_plan, rel_l2, tensors_of, to_gpu

pytestmark = pytest.mark.gpu


def gpu_backward(plan, t, topk):
    """GPU gradients and the GPU's selection ([N, H, k])."""
    g = to_gpu(t)
    dq, dk, dv = plan.backward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], g["dO"], topk)
    _, sel = plan.forward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], topk, return_sel=True)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return [x.double().cpu().numpy() for x in (dq, dk, dv)] + [sel.cpu().numpy()]


def swapped_keys(gpu_sel, ora_sel, blk_off, perm, H):
    """[N, H] mask of (key, head) pairs whose gradient receives a contribution that differs between
    the two selections. The selected branch is one softmax over all tokens of a row's selected
    blocks, so a swapped block changes the normaliser and with it the weight of every selected
    token: the mask covers the tokens of every block in the union of the pair's two block sets."""
    mask = np.zeros((len(perm), H), bool)
    diff = np.nonzero(~same_selection(gpu_sel, ora_sel))
    for i, h in zip(*diff):
        for b in set(gpu_sel[i, h].tolist()) | set(ora_sel[i, h].tolist()):
            if b >= 0:
                mask[perm[blk_off[b]:blk_off[b + 1]], h] = True
    return mask


def same_selection(gpu_sel, ora_sel):
    """[R, H] mask of (row, head) pairs whose selected block sets agree. Rows that differ (near
    ties, validated by the forward tests) attend to different keys, so their dQ is not comparable."""
    return np.all(np.sort(gpu_sel, axis=2) == np.sort(ora_sel, axis=2), axis=2)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_backward_full(name):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = tensors_of(name, with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    dq, dk, dv, sel = gpu_backward(plan, t, cfg.topk)
    ref = oracle.backward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"], cfg.topk,
                          cfg.radius)
    ora_sel = oracle.forward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], cfg.topk,
                             cfg.radius)["sel"]
    keep = same_selection(sel, ora_sel)
    assert keep.mean() >= 0.99
    check_grad_close(dq[keep], ref[0][keep], cfg.dtype, "dQ")
    pl = oracle.plan(c, cu, 8, cfg.radius)
    kk = ~swapped_keys(sel, ora_sel, pl["blk_off"], pl["perm"], cfg.H)
    assert kk.mean() >= 0.9, kk.mean()
    check_grad_close(dk[kk], ref[1][kk], cfg.dtype, "dK")
    check_grad_close(dv[kk], ref[2][kk], cfg.dtype, "dV")


@pytest.mark.slow
def test_backward_varlen_sampled_rows_and_sums():
    cfg = workloads.CONFIGS["varlen"]
    c, cu, g = coords_of("varlen")
    t = tensors_of("varlen", with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    dq, dk, dv, sel = gpu_backward(plan, t, cfg.topk)
    rows = np.concatenate(workloads.stratified_rows(cu, 512, seed=5099))
    ref, ora_sel = oracle.backward_dq_rows(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"],
                                           t["dO"], cfg.topk, cfg.radius, rows, return_sel=True)
    keep = same_selection(sel[rows], ora_sel)
    assert keep.mean() >= 0.99
    check_grad_close(dq[rows][keep], ref[keep], cfg.dtype, "dQ rows")
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

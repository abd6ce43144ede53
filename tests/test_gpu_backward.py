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
from ssa_testlib import check_close, coords_of, make_plan, rel_l2, tensors_of, to_gpu

pytestmark = pytest.mark.gpu


def gpu_backward(plan, t, topk):
    g = to_gpu(t)
    dq, dk, dv = plan.backward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], g["dO"], topk)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return [x.double().cpu().numpy() for x in (dq, dk, dv)]


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_backward_full(name):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = tensors_of(name, with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    got = gpu_backward(plan, t, cfg.topk)
    ref = oracle.backward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"], cfg.topk,
                          cfg.radius)
    for a, b, what in zip(got, ref, ("dQ", "dK", "dV")):
        check_close(a, b, cfg.dtype, what)


@pytest.mark.slow
def test_backward_varlen_sampled_rows_and_sums():
    cfg = workloads.CONFIGS["varlen"]
    c, cu, g = coords_of("varlen")
    t = tensors_of("varlen", with_grad_out=True)
    plan = make_plan(c, cu, g, cfg.radius)
    dq, dk, dv = gpu_backward(plan, t, cfg.topk)
    rows = np.concatenate(workloads.stratified_rows(cu, 512, seed=5099))
    ref = oracle.backward_dq_rows(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], t["dO"],
                                  cfg.topk, cfg.radius, rows)
    check_close(dq[rows], ref, cfg.dtype, "dQ rows")
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

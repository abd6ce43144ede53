"""Parity of ssa_forward_ex against the fp64 oracle, through the C ABI: compression by sparse 3D
convolution over the block grid and gates predicted from the queries (Direct3D-S2 summary page,
"Technical principles of Direct3D-S2", SSA item: blocks become block-level tokens by sparse 3D
convolution and pooling; the branches are aggregated with predicted gating scores), alone and
together with the attention prologue.

Every compared row is compared on every element, with the oracle evaluated on the GPU's validated
selection.
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
    return dict(
        conv=(rng.standard_normal((27, D, D)) / np.sqrt(27 * D)).astype(np.float32),
        gate_w=(rng.standard_normal((D, 3)) / np.sqrt(D)).astype(np.float32),
        gate_b=rng.standard_normal(3).astype(np.float32),
        q_gamma=(rng.random(D) + 0.5).astype(np.float32),
        k_gamma=(rng.random(D) + 0.5).astype(np.float32))


def run_and_compare(name, c, cu, grids, t, topk, r, dtype, use, rows=None, seed=0):
    """use: subset of {"conv", "gate", "prologue"}."""
    D = t["Q"].shape[2]
    w = _weights(D, seed)
    cuda = {k: torch.from_numpy(v).cuda() for k, v in w.items()}
    plan = make_plan(c, cu, grids, r)
    g = to_gpu(t)
    kw = {}
    if "conv" in use:
        kw["conv_w"] = cuda["conv"]
    if "gate" in use:
        kw.update(gate_w=cuda["gate_w"], gate_b=cuda["gate_b"])
    if "prologue" in use:
        kw.update(q_gamma=cuda["q_gamma"], k_gamma=cuda["k_gamma"], rope_theta=1000.0, eps=1e-6)
    out, sel = plan.forward_ex(g["Q"], g["K"], g["V"], None if "gate" in use else g["gates"],
                               None if "conv" in use else g["Wc"], topk, return_sel=True, **kw)
    torch.cuda.synchronize()
    assert plan.status() == 0
    ora = {}
    if "conv" in use:
        ora["conv"] = w["conv"]
    if "gate" in use:
        ora["gate"] = dict(w=w["gate_w"], b=w["gate_b"])
    if "prologue" in use:
        ora["prologue"] = dict(q_gamma=w["q_gamma"], k_gamma=w["k_gamma"], eps=1e-6, theta=1000.0)
    bs = plan.export()["blk_seq"].cpu().numpy()
    ref, _ = oracle_on_gpu_selection(c, cu, t, topk, r, sel.cpu().numpy(), bs, dtype, rows=rows, **ora)
    R = ref["rows"]
    got = out[torch.from_numpy(R).cuda()].double().cpu().numpy()
    check_close(got, ref["out"], dtype, f"{name} {sorted(use)} out")
    return plan, g, out


def _inputs(name, dtype):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = dict(tensors_of(name))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    for key in ("Q", "K", "V"):
        t[key] = t[key].float().to(tdt)
    return cfg, c, cu, g, t


@pytest.mark.parametrize("use", [("conv",), ("gate",), ("conv", "gate"), ("conv", "gate", "prologue")])
@pytest.mark.parametrize("name,dtype", [("tiny", "f32"), ("small", "bf16"), ("small", "f16")])
def test_variants_full_output(name, dtype, use):
    cfg, c, cu, g, t = _inputs(name, dtype)
    run_and_compare(name, c, cu, g, t, cfg.topk, cfg.radius, dtype, set(use), seed=cfg.index)


def test_centre_tap_equals_the_plain_forward_on_the_gpu():
    """A convolution whose only tap is the centre one, Wc, gives the plain forward (to rounding:
    the product with Wc is taken in another kernel)."""
    cfg, c, cu, g, t = _inputs("small", "f16")
    plan = make_plan(c, cu, g, cfg.radius)
    d = to_gpu(t)
    W = torch.from_numpy(oracle.center_only_conv(t["Wc"])).cuda()
    a = plan.forward(d["Q"], d["K"], d["V"], d["gates"], d["Wc"], cfg.topk)
    b = plan.forward_ex(d["Q"], d["K"], d["V"], d["gates"], None, cfg.topk, conv_w=W)
    torch.cuda.synchronize()
    check_close(b.double().cpu().numpy(), a.double().cpu().numpy(), "f16", "centre tap")


def test_variant_head_dims_and_ragged_varlen():
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:1333]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    for D, dtype in ((32, "f16"), (64, "bf16"), (128, "f16"), (64, "f32")):
        cfg = workloads.WorkloadConfig("var", 13, (), H=3, D=D, dtype=dtype, topk=5, radius=2)
        t = workloads.make_tensors(cfg, len(c))
        run_and_compare(f"D={D} {dtype}", c, cu, grids, t, 5, 2, dtype, {"conv", "gate"}, seed=D)


def test_variant_argument_errors():
    import spatial_sparse_attention_b200 as ssa
    cfg, c, cu, g, t = _inputs("tiny", "f16")
    plan = make_plan(c, cu, g, cfg.radius)
    d = to_gpu(t)
    D = t["Q"].shape[2]
    wg = torch.zeros(D, 3, device="cuda")
    with pytest.raises(ssa.SSAError) as e:   # gate weights without the bias
        plan.forward_ex(d["Q"], d["K"], d["V"], None, d["Wc"], cfg.topk, gate_w=wg)
    assert e.value.name == "SSA_ERR_INVALID_ARG"
    with pytest.raises(ssa.SSAError) as e:   # neither gates nor a predictor
        plan.forward_ex(d["Q"], d["K"], d["V"], None, d["Wc"], cfg.topk)
    assert e.value.name == "SSA_ERR_INVALID_ARG"


@pytest.mark.slow
def test_variants_full_size_every_query_tile():
    """The headline workload (110k tokens, 22 heads, fp16) with the convolution compression, the
    predicted gates and the prologue: every head of rows from every 128-token query tile."""
    cfg, c, cu, g, t = _inputs("pass3", "f16")
    perm = oracle.plan(c, cu, 8, cfg.radius)["perm"]
    rows = tile_rows(perm, cu, seed=cfg.index * 1000 + 96)
    run_and_compare("pass3", c, cu, g, t, cfg.topk, cfg.radius, "f16", {"conv", "gate", "prologue"},
                    rows=rows, seed=5)

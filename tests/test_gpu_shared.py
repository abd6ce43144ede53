"""Parity of the selection shared by the queries of a 4x4x4 sub-block (ssa_forward_ex with
select_share = 1) against the fp64 oracle, through the C ABI.

The Direct3D-S2 summary page ("Technical principles", SSA item) chooses the important blocks from
the compression module's attention scores and leaves open whose; this variant sums the compressed
attention weights of every query of a 4x4x4 sub-block of cells and gives all of them the own
block plus the top k-1 others by that sum. Every test checks that the tokens of each sub-block
hold one selection, that the selection is the oracle's up to near ties of the summed weights, and
compares every element of the outputs with the oracle evaluated on the GPU's selection.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import (check_close, check_selection_shared, coords_of, make_plan, tensors_of,
                         tile_rows, to_gpu, validate_shared_selection)

pytestmark = pytest.mark.gpu


def _inputs(name, dtype):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = dict(tensors_of(name))
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    for key in ("Q", "K", "V"):
        t[key] = t[key].float().to(tdt)
    return cfg, c, cu, g, t


def run_and_compare(name, c, cu, grids, t, topk, r, dtype, rows=None, extra=None):
    """extra: optional dict with prologue / conv / gate weights (numpy) for the options."""
    plan = make_plan(c, cu, grids, r)
    d = to_gpu(t)
    kw, ora = {}, {}
    gates, wc = d["gates"], d["Wc"]
    if extra:
        cu_t = {k: torch.from_numpy(v).cuda() for k, v in extra.items()}
        if "conv" in extra:
            kw["conv_w"] = cu_t["conv"]
            ora["conv"] = extra["conv"]
            wc = None
        if "gate_w" in extra:
            kw.update(gate_w=cu_t["gate_w"], gate_b=cu_t["gate_b"])
            ora["gate"] = dict(w=extra["gate_w"], b=extra["gate_b"])
            gates = None
        if "q_gamma" in extra:
            kw.update(q_gamma=cu_t["q_gamma"], k_gamma=cu_t["k_gamma"], rope_theta=1000.0, eps=1e-6)
            ora["prologue"] = dict(q_gamma=extra["q_gamma"], k_gamma=extra["k_gamma"], eps=1e-6,
                                   theta=1000.0)
    out, sel = plan.forward_ex(d["Q"], d["K"], d["V"], gates, wc, topk, return_sel=True,
                               share_selection=True, **kw)
    torch.cuda.synchronize()
    assert plan.status() == 0
    sel = sel.cpu().numpy()
    n_groups = check_selection_shared(c, cu, sel)
    assert n_groups < len(c)   # sub-blocks with several tokens exist: the sharing is exercised
    rows = np.arange(len(c)) if rows is None else np.asarray(rows)
    bs = plan.export()["blk_seq"].cpu().numpy()
    gs, _ = validate_shared_selection(c, cu, t, topk, sel, bs, dtype, rows,
                                      prologue=ora.get("prologue"), conv=ora.get("conv"))
    ref = oracle.forward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], topk, r, rows=rows,
                         sel_in=gs, **ora)
    got = out[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    check_close(got, ref["out"], dtype, f"{name} shared selection out")
    return plan, sel


def _sample(c, cu, r, seed):
    perm = oracle.plan(c, cu, 8, r)["perm"]
    return tile_rows(perm, cu, seed=seed)


@pytest.mark.parametrize("name,dtype", [("tiny", "f16"), ("tiny", "bf16"), ("small", "f16"),
                                        ("small", "bf16")])
def test_shared_selection_output(name, dtype):
    cfg, c, cu, g, t = _inputs(name, dtype)
    rows = None if name == "tiny" else _sample(c, cu, cfg.radius, cfg.index * 1000 + 97)
    run_and_compare(name, c, cu, g, t, cfg.topk, cfg.radius, dtype, rows=rows)


def test_shared_selection_with_prologue_convolution_and_predicted_gates():
    cfg, c, cu, g, t = _inputs("small", "f16")
    D = t["Q"].shape[2]
    rng = np.random.default_rng(7)
    extra = dict(conv=(rng.standard_normal((27, D, D)) / np.sqrt(27 * D)).astype(np.float32),
                 gate_w=(rng.standard_normal((D, 3)) / np.sqrt(D)).astype(np.float32),
                 gate_b=rng.standard_normal(3).astype(np.float32),
                 q_gamma=(rng.random(D) + 0.5).astype(np.float32),
                 k_gamma=(rng.random(D) + 0.5).astype(np.float32))
    rows = _sample(c, cu, cfg.radius, 98)
    run_and_compare("small", c, cu, g, t, cfg.topk, cfg.radius, "f16", rows=rows, extra=extra)


def test_shared_selection_head_dims_ragged_varlen_and_k():
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:1333]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    for D, dtype, k in ((32, "f16", 5), (64, "bf16", 9), (128, "f16", 3), (96, "f16", 1), (64, "f16", 20)):
        cfg = workloads.WorkloadConfig("var", 13, (), H=3, D=D, dtype=dtype, topk=k, radius=2)
        t = workloads.make_tensors(cfg, len(c))
        run_and_compare(f"D={D} {dtype} k={k}", c, cu, grids, t, k, 2, dtype)


def test_shared_selection_is_unsupported_for_fp32():
    import spatial_sparse_attention_b200 as ssa
    cfg = workloads.CONFIGS["tiny"]
    c, cu, g = coords_of("tiny")
    t = tensors_of("tiny")
    plan = make_plan(c, cu, g, cfg.radius)
    d = to_gpu(t)
    with pytest.raises(ssa.SSAError) as e:
        plan.forward_ex(d["Q"].float(), d["K"].float(), d["V"].float(), d["gates"], d["Wc"], cfg.topk,
                        share_selection=True)
    assert e.value.name == "SSA_ERR_UNSUPPORTED"


@pytest.mark.slow
def test_shared_selection_full_size_every_query_tile():
    """The headline workload (110k tokens, 22 heads, fp16): sharing over all rows, and rows from
    every 128-token query tile against the oracle."""
    cfg, c, cu, g, t = _inputs("pass3", "f16")
    rows = _sample(c, cu, cfg.radius, cfg.index * 1000 + 99)
    run_and_compare("pass3", c, cu, g, t, cfg.topk, cfg.radius, "f16", rows=rows)

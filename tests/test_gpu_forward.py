"""Forward parity (pooling, the three branches, gated combine) of the CUDA path against the fp64
oracle, through the C ABI.

Every compared row is compared on every element, against the oracle evaluated on the GPU's
selection once that selection has been validated (near ties only). Small configurations: every
row and head, and the three branch outputs. Full-size configurations (80k, 110k and the 340k-token
varlen batch, H=22, D=96, fp16, in the launch configuration the benchmark times): the whole output
of the 110k-token headline workload, every row of a seeded subset of heads of the other two, and
every head of rows drawn from every 128-token query tile of all three.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ssa_testlib import (check_close, coords_of, make_plan, oracle_on_gpu_selection, tensors_of,
                         tile_rows, to_gpu)

pytestmark = pytest.mark.gpu

BRANCHES = ("o_cmp", "o_sel", "o_win")


def gpu_forward(plan, t, topk, branches=False):
    """(out, sel, (o_cmp, o_sel, o_win) or None) as CUDA tensors."""
    g = to_gpu(t)
    res = plan.forward(g["Q"], g["K"], g["V"], g["gates"], g["Wc"], topk, return_sel=True,
                       return_branches=branches)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return res[0], res[1], (res[2] if branches else None)


def _pick(x, rows, heads):
    """Rows and heads of a CUDA tensor [N, H, D] as fp64 numpy."""
    y = x[torch.from_numpy(np.asarray(rows)).to(x.device)]
    if heads is not None:
        y = y[:, list(heads)]
    return y.double().cpu().numpy()


def compare(name, coords, cu, grids, t, topk, r, dtype, rows=None, heads=None, branches=False):
    plan = make_plan(coords, cu, grids, r)
    out, sel, br = gpu_forward(plan, t, topk, branches)
    bs = plan.export()["blk_seq"].cpu().numpy()
    ref, rep = oracle_on_gpu_selection(coords, cu, t, topk, r, sel.cpu().numpy(), bs, dtype,
                                       rows=rows, heads=heads)
    R = ref["rows"]
    check_close(_pick(out, R, heads), ref["out"], dtype, f"{name} out")
    if branches:
        for x, nm in zip(br, BRANCHES):
            check_close(_pick(x, R, heads), ref[nm], dtype, f"{name} {nm}", stored=False)
    return plan, out, sel, ref, br


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_full_output(name):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    compare(name, c, cu, g, tensors_of(name), cfg.topk, cfg.radius, cfg.dtype, branches=True)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["pass1", "pass3", "varlen"])
def test_forward_full_size_every_query_tile(name):
    """Every head of rows from every query tile (one per 32-row quarter plus the tile's last row),
    so that no tile of the union build, the pool compaction or the window masks goes unchecked."""
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    perm = oracle.plan(c, cu, 8, cfg.radius)["perm"]
    rows = tile_rows(perm, cu, seed=cfg.index * 1000 + 99)
    compare(name, c, cu, g, tensors_of(name), cfg.topk, cfg.radius, cfg.dtype, rows=rows,
            branches=True)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["pass1", "pass3", "varlen"])
def test_forward_full_size_every_row(name):
    """Every row of the full-size output for a seeded subset of heads (heads are independent:
    the oracle runs on those heads alone)."""
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    n_heads = {"pass1": 4, "pass3": cfg.H, "varlen": 2}[name]   # pass3: the whole output
    heads = None if n_heads == cfg.H else sorted(
        np.random.default_rng(cfg.index * 1000 + 98).choice(cfg.H, n_heads, replace=False).tolist())
    compare(name, c, cu, g, tensors_of(name), cfg.topk, cfg.radius, cfg.dtype, heads=heads)


def _branch_inputs(name, dtype):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    t = dict(tensors_of(name))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    for key in ("Q", "K", "V"):
        t[key] = t[key].float().to(tdt)
    return cfg, c, cu, g, t


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("branch", [0, 1, 2])
def test_each_branch_alone(dtype, branch):
    """One-hot gates isolate the compressed, selected and window branches in the gated sum."""
    cfg, c, cu, g, t = _branch_inputs("small", dtype)
    gates = torch.zeros_like(t["gates"])
    gates[:, :, branch] = 1.0
    t["gates"] = gates
    compare(f"branch{branch}", c, cu, g, t, cfg.topk, cfg.radius, dtype)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_branch_outputs_with_mixed_gates(dtype):
    """The three branch outputs of ssa_forward_debug, with random gates, each against the oracle's
    o_cmp, o_sel, o_win; and the gated sum of the GPU's branch outputs against its out."""
    name = "tiny" if dtype == "f32" else "small"
    cfg, c, cu, g, t = _branch_inputs(name, dtype)
    plan, out, sel, ref, br = compare(f"branches {dtype}", c, cu, g, t, cfg.topk, cfg.radius,
                                      dtype, branches=True)
    gates = t["gates"].cuda()
    mix = sum(gates[:, :, i:i + 1] * br[i] for i in range(3))
    check_close(out.double().cpu().numpy(), mix.double().cpu().numpy(), dtype, "gated sum")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_planted_topk_is_exact(dtype):
    """Queries e = 1, keys of block b = alpha_b * 1, Wc = I: the ranking is known exactly."""
    c, cu, g = coords_of("tiny")
    N, H, D, topk = len(c), 2, 32, 6
    perm, tok_blk, blk_off, blk_coord = oracle.partition(c)
    mb = len(blk_coord)
    rng = np.random.default_rng(7)
    alpha = (np.stack([rng.permutation(mb) for _ in range(H)], 1) - mb / 2) / 8.0
    alpha[7, 0] = alpha[3, 0]   # tie: the lower block index wins
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    t = dict(Q=torch.ones(N, H, D).to(tdt),
             K=torch.from_numpy(np.repeat(alpha[tok_blk][:, :, None], D, 2)).float().to(tdt),
             V=torch.randn(N, H, D, generator=torch.Generator().manual_seed(3)).to(tdt),
             gates=torch.rand(N, H, 3, generator=torch.Generator().manual_seed(4)),
             Wc=torch.eye(D))
    plan = make_plan(c, cu, g, 2)
    out, sel, _ = gpu_forward(plan, t, topk)
    out, sel = out.double().cpu().numpy(), sel.cpu().numpy()
    exp = np.full((N, H, topk), -1)
    for i in range(N):
        for h in range(H):
            others = sorted((b for b in range(mb) if b != tok_blk[i]), key=lambda b: (-alpha[b, h], b))
            exp[i, h] = [tok_blk[i]] + others[:topk - 1]
    assert np.array_equal(sel, exp)
    ref = oracle.forward(c, cu, t["Q"], t["K"], t["V"], t["gates"], t["Wc"], topk, 2)
    check_close(out, ref["out"], dtype, "planted")


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_fewer_blocks_than_k_and_dense_limit(dtype):
    """k >= Mb selects every block: with selection-only gates the output is dense attention."""
    c_all, _, g = coords_of("tiny")
    c = c_all[:300]                      # the first 300 voxels in (x, y, z) order: a few blocks
    cu = np.array([0, len(c)])
    mb = len(oracle.partition(c)[3])
    assert mb + 2 <= 32
    cfg = workloads.WorkloadConfig("dense", 7, (), H=2, D=32, dtype=dtype, topk=mb + 2, radius=2)
    t = workloads.make_tensors(cfg, len(c))
    gates = torch.zeros_like(t["gates"])
    gates[:, :, 1] = 1.0
    t["gates"] = gates
    plan, out, sel, ref, _ = compare("dense", c, cu, g, t, mb + 2, 2, dtype)
    out, sel = out.double().cpu().numpy(), sel.cpu().numpy()
    assert np.all(sel[:, :, mb:] == -1)
    # textbook dense attention over all tokens (library routine, fp64)
    q, k, v = (x.double().permute(1, 0, 2) for x in (t["Q"], t["K"], t["V"]))
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v).permute(1, 0, 2).numpy()
    check_close(out, dense, dtype, "dense limit")


@pytest.mark.parametrize("r", [0, 1, 3, 8])
def test_window_radii(r):
    cfg, c, cu, g, t = _branch_inputs("small", "f16")
    compare(f"r={r}", c, cu, g, t, cfg.topk, r, "f16")


def test_ragged_tiles_single_token_and_varlen_edge_cases():
    a, _, _ = coords_of("tiny")
    b = np.array([[5, 6, 7]], np.int32)
    c = np.concatenate([a[:700], b, a[700:1333]])
    cu = np.array([0, 700, 700, 701, len(c)])
    grids = np.array([[32, 32, 32], [16, 16, 16], [9, 9, 9], [32, 32, 32]], np.int32)
    cfg = workloads.WorkloadConfig("edge", 9, (), H=3, D=64, dtype="f16", topk=5, radius=2)
    t = workloads.make_tensors(cfg, len(c))
    compare("edge", c, cu, grids, t, 5, 2, "f16")


def test_head_dims_and_k_values():
    c, cu, g = coords_of("tiny")
    for D, topk in ((32, 1), (64, 9), (128, 17), (96, 32)):
        cfg = workloads.WorkloadConfig("hd", 8, (), H=2, D=D, dtype="bf16", topk=topk, radius=2)
        t = workloads.make_tensors(cfg, len(c))
        compare(f"D={D},k={topk}", c, cu, g, t, topk, 2, "bf16")


def test_repeat_calls_are_bitwise_identical_and_host_entry_matches():
    cfg = workloads.CONFIGS["small"]
    c, cu, g = coords_of("small")
    t = tensors_of("small")
    plan = make_plan(c, cu, g, cfg.radius)
    dev = to_gpu(t)
    a = plan.forward(dev["Q"], dev["K"], dev["V"], dev["gates"], dev["Wc"], cfg.topk)
    b = plan.forward(dev["Q"], dev["K"], dev["V"], dev["gates"], dev["Wc"], cfg.topk)
    host = {k: v.pin_memory() for k, v in t.items()}
    out_h = torch.empty_like(host["Q"]).pin_memory()
    plan.forward_host(host["Q"], host["K"], host["V"], host["gates"], host["Wc"], cfg.topk, out_h)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(a.cpu(), out_h)


@pytest.mark.parametrize("H,D,dtype", [(6, 32, "f32"), (22, 96, "f16"), (4, 64, "bf16")])
def test_host_entry_in_head_chunks_matches_the_device_forward(H, D, dtype):
    """The host-buffer entry point copies and computes the heads in chunks (6 x 32 fp32 in 3
    chunks of 2, 22 x 96 fp16 in 11, 4 x 64 bf16 in 2): every element equals the device forward."""
    c, cu, g = coords_of("small")
    cfg = workloads.WorkloadConfig("chunks", 17, (), H=H, D=D, dtype=dtype, topk=8, radius=2)
    t = workloads.make_tensors(cfg, len(c))
    plan = make_plan(c, cu, g, 2)
    dev = to_gpu(t)
    a = plan.forward(dev["Q"], dev["K"], dev["V"], dev["gates"], dev["Wc"], 8)
    host = {k: v.pin_memory() for k, v in t.items()}
    out_h = torch.empty_like(host["Q"]).pin_memory()
    for _ in range(2):   # the second call reuses the chunk buffers
        out_h.zero_()
        plan.forward_host(host["Q"], host["K"], host["V"], host["gates"], host["Wc"], 8, out_h)
        torch.cuda.synchronize()
        assert torch.equal(a.cpu(), out_h)


def test_forward_argument_errors():
    import spatial_sparse_attention_b200 as ssa
    c, cu, g = coords_of("tiny")
    plan = make_plan(c, cu, g, 2)
    N = len(c)
    q = torch.zeros(N, 2, 48, dtype=torch.float16, device="cuda")
    gates = torch.zeros(N, 2, 3, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        plan.forward(q, q, q, gates, torch.eye(48, device="cuda"), 4)
    assert e.value.name == "SSA_ERR_UNSUPPORTED"
    q = torch.zeros(N, 2, 32, dtype=torch.float16, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        plan.forward(q, q, q, gates, torch.eye(32, device="cuda"), 33)
    assert e.value.name == "SSA_ERR_UNSUPPORTED"


def test_too_many_blocks_in_a_sequence_is_unsupported():
    """The 16-bit path builds the union of selected blocks in on-chip memory: a sequence with more
    than 65,536 * D / 32 occupied blocks is rejected before any kernel runs."""
    import spatial_sparse_attention_b200 as ssa
    n = 70_000   # one token per block: 70,000 blocks > 65,536 for D = 32
    i = np.arange(n)
    coords = np.stack([8 * (i // (128 * 64)), 8 * ((i // 64) % 128), 8 * (i % 64)], 1).astype(np.int32)
    plan = ssa.Plan(torch.from_numpy(coords).cuda(), grid=(1024, 1024, 512), r=0)
    assert plan.num_blocks == n
    q = torch.zeros(n, 1, 32, dtype=torch.bfloat16, device="cuda")
    gates = torch.zeros(n, 1, 3, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        plan.forward(q, q, q, gates, torch.eye(32, device="cuda"), 2)
    assert e.value.name == "SSA_ERR_UNSUPPORTED"


def test_bounded_wait_timeout_is_reported_and_the_next_call_is_clean():
    """A bounded mbarrier wait that runs out (nothing ever arrives) is reported as
    SSA_ERR_DEVICE_TIMEOUT by the next status read; the plan and the context stay usable."""
    cfg = workloads.CONFIGS["small"]
    c, cu, g = coords_of("small")
    plan = make_plan(c, cu, g, cfg.radius)
    plan.debug_wait_timeout(2_000_000)   # about a millisecond at the SM clock
    assert plan.status() == 7             # SSA_ERR_DEVICE_TIMEOUT, and cleared by the read
    assert plan.status() == 0
    t = tensors_of("small")
    out, sel, _ = gpu_forward(plan, t, cfg.topk)
    bs = plan.export()["blk_seq"].cpu().numpy()
    ref, _ = oracle_on_gpu_selection(c, cu, t, cfg.topk, cfg.radius, sel.cpu().numpy(), bs, cfg.dtype)
    check_close(_pick(out, ref["rows"], None), ref["out"], cfg.dtype, "after timeout")

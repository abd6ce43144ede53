"""Helpers shared by the GPU parity tests: seeded inputs, GPU runs through the C ABI, oracle
comparison with the stated tolerances.

Tolerances (the method's outputs for 16-bit inputs with fp32 accumulation): max |delta| <= 1e-2
and relative L2 <= 5e-3 per output tensor; fp32 inputs: both <= 1e-5. The max |delta| bound is
read as the bound on the computed value: the rounding of the output to its storage type (half an
ulp, up to 2^-8 |value| for bf16, which alone passes 1e-2 from |value| = 2.56) comes on top. The
reference is the fp64 oracle with the compressed tokens left unrounded.

Top-k: the selection is compared as a set per (query, head). Where the GPU's set differs from the
oracle's, every block the GPU chose instead must be within the near-tie gap of the oracle's k-th
choice: 1e-4 in probability (the stated bar) and 1e-5 in scaled logit for fp32 inputs; for 16-bit
inputs, whose compressed tokens are stored in the input type, either the stated probability gap or
a scaled-logit gap within the storage rounding (LOGIT_GAP). The outputs of every row are then
compared with the oracle evaluated on the GPU's (validated) selection, so no row is left out.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
import workloads

TOL = {"f32": (1e-5, 1e-5), "bf16": (1e-2, 5e-3), "f16": (1e-2, 5e-3)}
# Largest scaled-logit gap accepted for a swapped block, on top of the stated probability gap.
# The GPU ranks blocks on compressed tokens stored in the input type, the oracle on unrounded
# ones: rounding changes a logit s*q.Kc by up to s*|q|*|Kc|*u (u the unit roundoff: 2^-11 for
# f16, 2^-8 for bf16). With s = 1/sqrt(D), |q| ~ sqrt(D) and |Kc| up to ~sqrt(D) (one-token
# blocks) that is about sqrt(D)*u: 5e-3 for f16 and 4e-2 for bf16 at D = 96..128 (rounded up);
# fp32 keeps 1e-5.
LOGIT_GAP = {"f32": 1e-5, "bf16": 4e-2, "f16": 5e-3}
P_GAP = 1e-4


@functools.lru_cache(maxsize=None)
def coords_of(name: str):
    return workloads.make_coords(workloads.CONFIGS[name])


@functools.lru_cache(maxsize=2)
def tensors_of(name: str, with_grad_out: bool = False):
    cfg = workloads.CONFIGS[name]
    c, cu, g = coords_of(name)
    return workloads.make_tensors(cfg, len(c), with_grad_out=with_grad_out)


def to_gpu(t: dict):
    return {k: v.cuda().contiguous() for k, v in t.items()}


def make_plan(coords, cu, grids, r):
    import spatial_sparse_attention_b200 as ssa
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).cuda()
    if len(cu) == 2:
        return ssa.Plan(c, grid=tuple(int(x) for x in grids[0]), r=r)
    return ssa.Plan(c, r=r, cu_seqlens=[int(x) for x in cu], grids=[tuple(g) for g in grids])


def rel_l2(a, b):
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / max(den, 1e-30))


# Unit roundoff of the output's storage type. The stated max |delta| bounds the computed value;
# storing it in the input type adds up to half an ulp, at most U_STORE * |value| (RNE), which is
# itself above 1e-2 for bf16 outputs of magnitude 2.56 and more. That part is allowed on top.
U_STORE = {"f32": 2.0 ** -24, "bf16": 2.0 ** -8, "f16": 2.0 ** -11}


def check_close(gpu, ref, dtype, what="", stored=True):
    """stored: the GPU values were stored in the input type (False for fp32 branch outputs)."""
    atol, rtol = TOL[dtype]
    raw = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    u = U_STORE[dtype] if stored else 0.0
    err = float((np.abs(gpu - ref) - u * np.abs(ref)).max()) if gpu.size else 0.0
    r = rel_l2(gpu, ref)
    print(f"{what}: max|d|={raw:.3e} (beyond the output's storage rounding {err:.3e}) relL2={r:.3e} ({dtype})")
    assert err <= atol and r <= rtol, (f"{what}: max|d| beyond storage rounding={err:.3e} (<= {atol}), "
                                       f"relL2={r:.3e} (<= {rtol})")
    return err, r


def check_grad_close(gpu, ref, dtype, what=""):
    """Gradients: no tolerance is stated for them, so the bound is taken relative to the tensor's
    scale: max|delta| <= 1e-2 * max|ref| (about 2.5 bf16 ulps at the largest element) and
    relative L2 <= 5e-3; fp32 inputs: 1e-5 for both."""
    atol, rtol = TOL[dtype]
    scale = float(np.abs(ref).max()) if ref.size else 1.0
    err = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    r = rel_l2(gpu, ref)
    assert err <= atol * scale and r <= rtol, (
        f"{what}: max|d|={err:.3e} (<= {atol}*{scale:.3e}), relL2={r:.3e} (<= {rtol})")
    return err, r


def selection_agreement(gpu_sel, ora_sel, z_rows, blk_base_of_row, dtype):
    """Check the GPU selection of rows whose set differs from the oracle's.

    gpu_sel / ora_sel: [R, H, k] global block indices; z_rows: list of [H, Mb_seq] scaled
    logits per row (oracle); blk_base_of_row: [R] first global block of each row's sequence.
    Raises if a GPU choice is not a valid near-tie alternative. Returns (mismatch mask [R, H],
    largest logit gap of an accepted swap).
    """
    R, H, k = gpu_sel.shape
    mism = np.zeros((R, H), bool)
    worst = 0.0
    for r in range(R):
        z = z_rows[r]
        base = blk_base_of_row[r]
        for h in range(H):
            g = set(int(b) for b in gpu_sel[r, h] if b >= 0)
            o = set(int(b) for b in ora_sel[r, h] if b >= 0)
            assert gpu_sel[r, h, 0] == ora_sel[r, h, 0], "slot 0 must be the own block"
            if g == o:
                continue
            mism[r, h] = True
            assert len(g) == len(o), "GPU selected a different number of blocks"
            others = [b for b in ora_sel[r, h, 1:] if b >= 0]
            kth = z[h, others[-1] - base]
            zz = z[h] - z[h].max()
            p = np.exp(zz) / np.exp(zz).sum()
            pk = p[others[-1] - base]
            for b in g - o:
                gap_z = kth - z[h, b - base]
                gap_p = pk - p[b - base]
                worst = max(worst, gap_z)
                # the stated near tie (probability gap), or for 16-bit inputs a logit gap within
                # what storing the compressed tokens in the input type can move a logit; fp32
                # inputs must meet both
                ok = (gap_p <= P_GAP and gap_z <= LOGIT_GAP[dtype]) if dtype == "f32" else (
                    gap_p <= P_GAP or gap_z <= LOGIT_GAP[dtype])
                assert ok, (f"row {r} head {h}: block {b} is {gap_z:.2e} below the k-th logit "
                            f"({gap_p:.2e} in probability)")
    return mism, worst


def blk_base_of_rows(cu, rows, plan_export_blk_seq):
    seq = np.searchsorted(np.asarray(cu), rows, side="right") - 1
    bs = np.asarray(plan_export_blk_seq)
    first = np.array([np.searchsorted(bs, s) for s in range(len(cu) - 1)])
    return first[seq]


def head_slice(t: dict, heads):
    """The inputs restricted to some heads (heads are independent in the method)."""
    if heads is None:
        return t
    hs = list(heads)
    return {k: (v[:, hs].contiguous() if k in ("Q", "K", "V", "gates", "dO") else v)
            for k, v in t.items()}


def validate_gpu_selection(coords, cu, t, topk, r, gpu_sel, blk_seq, dtype, rows=None,
                           heads=None, prologue=None, conv=None, gate=None):
    """Check the GPU's selection of `rows` (None = all) and `heads` (None = all) against the
    oracle's own: equal sets, or near ties within the stated gap. Returns (the GPU selection of
    those rows and heads, report)."""
    N = len(coords)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    th = head_slice(t, heads)
    gs = gpu_sel[rows] if heads is None else gpu_sel[rows][:, list(heads)]
    # the oracle's own selection (compressed branch only), then the rows whose set differs
    own = oracle.forward(coords, cu, th["Q"], th["K"], th["V"], th["gates"], th["Wc"], topk, r,
                         rows=rows, branches=False, prologue=prologue, conv=conv, gate=gate)["sel"]
    same = np.all(np.sort(gs, axis=2) == np.sort(own, axis=2), axis=2)
    assert np.array_equal(gs[:, :, 0], own[:, :, 0]), "slot 0 must be the own block"
    bad = np.nonzero(~same.all(axis=1))[0]
    worst = 0.0
    if len(bad):
        zr = oracle.forward(coords, cu, th["Q"], th["K"], th["V"], th["gates"], th["Wc"], topk, r,
                            rows=rows[bad], branches=False, want_z=True, prologue=prologue,
                            conv=conv, gate=gate)
        _, worst = selection_agreement(gs[bad], zr["sel"], zr["z"],
                                       blk_base_of_rows(cu, rows[bad], blk_seq), dtype)
    report = dict(pairs=int(same.size), mismatched=int((~same).sum()), worst_logit_gap=worst)
    print(f"selection: {report}")
    return gs, report


def oracle_on_gpu_selection(coords, cu, t, topk, r, gpu_sel, blk_seq, dtype, rows=None,
                            heads=None, prologue=None, conv=None, gate=None):
    """The fp64 oracle's forward for `rows` (None = all) and `heads` (None = all), evaluated with
    the GPU's selection once that selection has been validated against the oracle's own.

    Returns (reference dict with out / o_cmp / o_sel / o_win [R, H', D] and rows, report)."""
    rows = np.arange(len(coords)) if rows is None else np.asarray(rows)
    gs, report = validate_gpu_selection(coords, cu, t, topk, r, gpu_sel, blk_seq, dtype, rows,
                                        heads, prologue, conv, gate)
    th = head_slice(t, heads)
    ref = oracle.forward(coords, cu, th["Q"], th["K"], th["V"], th["gates"], th["Wc"], topk, r,
                         rows=rows, sel_in=gs, prologue=prologue, conv=conv, gate=gate)
    return ref, report


def tile_rows(perm, cu, per_quarter=1, seed=0):
    """Rows from every 128-token query tile of every sequence (tiles are 128 consecutive tokens in
    block order, the unit the fused kernel works on): one seeded row from each 32-row quarter of
    a tile, plus the tile's last row."""
    rng = np.random.default_rng(seed)
    perm = np.asarray(perm)
    out = []
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        for a in range(lo, hi, 128):
            b = min(a + 128, hi)
            for q in range(a, b, 32):
                e = min(q + 32, b)
                out.extend(perm[rng.integers(q, e, size=per_quarter)].tolist())
            out.append(int(perm[b - 1]))
    return np.unique(np.asarray(out, dtype=np.int64))


def subblock_groups(coords, cu):
    """Group id of every token: its sequence and 4x4x4 sub-block of cells."""
    c = np.asarray(coords)
    seq = np.searchsorted(np.asarray(cu), np.arange(len(c)), side="right") - 1
    key = np.concatenate([seq[:, None], c // 4], axis=1)
    _, grp = np.unique(key, axis=0, return_inverse=True)
    return grp.reshape(-1)


def check_selection_shared(coords, cu, gpu_sel):
    """Every token of a 4x4x4 sub-block has the same selection (all heads)."""
    grp = subblock_groups(coords, cu)
    order = np.argsort(grp, kind="stable")
    g, s = grp[order], gpu_sel[order]
    same_group = g[1:] == g[:-1]
    differ = np.any(s[1:] != s[:-1], axis=(1, 2))
    assert not np.any(same_group & differ), "a sub-block's tokens hold different selections"
    return int(len(np.unique(grp)))


def validate_shared_selection(coords, cu, t, topk, gpu_sel, blk_seq, dtype, rows,
                              prologue=None, conv=None):
    """Check the GPU's sub-block-shared selection of `rows` against the oracle's: equal sets, or
    near ties. The oracle ranks the summed compressed-attention weights of each sub-block. A
    logit error d (the compressed tokens are stored in the input type on the GPU; LOGIT_GAP)
    moves a weight by a factor within exp(+-2d), so a swapped block's summed weight must be
    within 2 LOGIT_GAP (relative) of the block it displaced. Returns (GPU selection of the rows,
    report)."""
    rows = np.asarray(rows)
    gs = gpu_sel[rows]
    Q, K, V = t["Q"], t["K"], t["V"]
    if prologue is not None:
        # the prologue's results (rounded to the input type) as fp64, and V in the same type
        kw = dict(eps=prologue.get("eps", 1e-6), theta=prologue.get("theta", 10000.0), round_to_input=True)
        Q = oracle.qk_prologue(Q, coords, prologue["q_gamma"], **kw)
        K = oracle.qk_prologue(K, coords, prologue["k_gamma"], **kw)
        V = oracle._exact_f64(V)
    ora = oracle.select_subblock(coords, cu, Q, K, V, t["Wc"], topk, rows=rows, conv=conv,
                                 want_score=True)
    osel, score = ora["sel"], ora["score"]
    assert np.array_equal(gs[:, :, 0], osel[:, :, 0]), "slot 0 must be the own block"
    base = blk_base_of_rows(cu, rows, blk_seq)
    tol = 2 * LOGIT_GAP[dtype]
    mism, worst = 0, 0.0
    for i in range(len(rows)):
        for h in range(gs.shape[1]):
            a = set(int(x) for x in gs[i, h, 1:] if x >= 0)
            b = set(int(x) for x in osel[i, h, 1:] if x >= 0)
            if a == b:
                continue
            mism += 1
            assert len(a) == len(b) and len(a) == len(gs[i, h, 1:][gs[i, h, 1:] >= 0]), (rows[i], h)
            s = score[i][h]
            lo_in = min(s[c - base[i]] for c in a - b)
            hi_out = max(s[c - base[i]] for c in b - a)
            gap = hi_out / max(lo_in, 1e-300) - 1.0
            worst = max(worst, gap)
            assert gap <= tol, (f"row {rows[i]} head {h}: block(s) {sorted(a - b)} displaced "
                                f"{sorted(b - a)} with a summed-weight gap {gap:.3g} > {tol:.3g}")
    report = dict(pairs=int(gs.shape[0] * gs.shape[1]), mismatched=mism, worst_rel_gap=worst)
    print(f"shared selection: {report}")
    return gs, report

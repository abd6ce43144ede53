"""Helpers shared by the GPU parity tests: seeded inputs, GPU runs through the C ABI, oracle
comparison with the stated tolerances.

Tolerances (the method's outputs for 16-bit inputs with fp32 accumulation): max |delta| <= 1e-2
and relative L2 <= 5e-3 per output tensor; fp32 inputs: both <= 1e-5.

Top-k: the selection is compared as a set per (query, head). A row whose GPU set differs from the
oracle's must be a valid alternative: every swapped-in block must be within the oracle's
near-tie gap of the k-th choice (1e-4 in probability, the stated bar, and additionally 2e-3 in
scaled logit for 16-bit / 1e-5 for fp32 inputs); such rows are excluded from the element-wise
output comparison and counted.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
import workloads

TOL = {"f32": (1e-5, 1e-5), "bf16": (1e-2, 5e-3), "f16": (1e-2, 5e-3)}
LOGIT_GAP = {"f32": 1e-5, "bf16": 2e-3, "f16": 2e-3}
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


def check_close(gpu, ref, dtype, what=""):
    atol, rtol = TOL[dtype]
    err = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    r = rel_l2(gpu, ref)
    assert err <= atol and r <= rtol, f"{what}: max|d|={err:.3e} (<= {atol}), relL2={r:.3e} (<= {rtol})"
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
    """Compare selections per (row, head). Returns (mismatch mask [R,H], report).

    gpu_sel / ora_sel: [R, H, k] global block indices; z_rows: list of [H, Mb_seq] scaled
    logits per row (oracle); blk_base_of_row: [R] first global block of each row's sequence.
    Raises if a GPU choice is not a valid near-tie alternative.
    """
    R, H, k = gpu_sel.shape
    mism = np.zeros((R, H), bool)
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
                assert gap_z <= LOGIT_GAP[dtype] and gap_p <= P_GAP, (
                    f"row {r} head {h}: block {b} is {gap_z:.2e} below the k-th logit")
    return mism, dict(rows=R * H, mismatched=int(mism.sum()))


def blk_base_of_rows(cu, rows, plan_export_blk_seq):
    seq = np.searchsorted(np.asarray(cu), rows, side="right") - 1
    bs = np.asarray(plan_export_blk_seq)
    first = np.array([np.searchsorted(bs, s) for s in range(len(cu) - 1)])
    return first[seq]

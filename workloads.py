"""Seeded synthetic inputs for Spatial Sparse Attention: voxel shells and tensors.

This module is shared by the tests, the benchmark and the oracle's callers. It
holds none of the attention method's arithmetic: it only draws integer voxel
coordinates on the surface shells of simple solids, and random Q/K/V, gates and
the compression map Wc. Every draw is seeded (seed = config index * 1000 + tensor
id), so any machine regenerates the same inputs.

Workload shapes follow the refinement-pass table and transformer shape of the
Hi3D v1.0 pipeline page ("How the pipeline works" table: 64^3/80,000,
128^3/90,000, 192^3/110,000 voxels; "Stage 3": 22 heads, width 2,112, fp16) and
the Direct3D-S2 description of sparse volumetric tokens with integer voxel
coordinates.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

# Tensor ids used in seeds: seed = cfg_index * 1000 + id.
TID_COORDS, TID_Q, TID_K, TID_V, TID_GATES, TID_WC, TID_DO = 0, 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class ShapeSpec:
    """One sequence of the workload: its grid and how its voxels are drawn."""
    grid: Tuple[int, int, int]
    kind: str               # "sphere", "torus", "union_grow", "union_scale"
    n_target: Optional[int] = None
    n_shapes: int = 0
    thickness: float = 1.0
    boxes: bool = False


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    index: int
    shapes: Tuple[ShapeSpec, ...]
    H: int
    D: int
    dtype: str              # "f32", "bf16", "f16"
    topk: int
    radius: int
    block: int = 8
    description: str = ""


CONFIGS = {
    "tiny": WorkloadConfig(
        "tiny", 1, (ShapeSpec((32, 32, 32), "sphere"),), H=2, D=32, dtype="f32",
        topk=4, radius=2,
        description="surface shell (thickness 1) of a radius-12 sphere centred in a 32^3 grid"),
    "small": WorkloadConfig(
        "small", 2, (ShapeSpec((128, 128, 128), "torus", n_target=20000),), H=8, D=64,
        dtype="bf16", topk=8, radius=2,
        description="20,000 cells sampled from the thickness-2 shell of a torus R=40, r=15 in 128^3"),
    "pass1": WorkloadConfig(
        "pass1", 3, (ShapeSpec((64, 64, 64), "union_grow", n_target=80000, n_shapes=3),),
        H=22, D=96, dtype="f16", topk=16, radius=2,
        description="80,000 cells from a thick shell of 3 random ellipsoids in 64^3 (~30% occupancy)"),
    "pass3": WorkloadConfig(
        "pass3", 4, (ShapeSpec((192, 192, 192), "union_scale", n_target=110000, n_shapes=5,
                               thickness=3.0, boxes=True),),
        H=22, D=96, dtype="f16", topk=16, radius=3,
        description="110,000 cells from the thickness-3 shell of 5 random ellipsoids/boxes in 192^3"),
    "varlen": WorkloadConfig(
        "varlen", 5, (
            ShapeSpec((64, 64, 64), "union_grow", n_target=80000, n_shapes=3),
            ShapeSpec((128, 128, 128), "union_scale", n_target=90000, n_shapes=4, thickness=3.0),
            ShapeSpec((192, 192, 192), "union_scale", n_target=110000, n_shapes=5, thickness=3.0,
                      boxes=True),
            ShapeSpec((128, 128, 128), "union_scale", n_target=60000, n_shapes=4, thickness=3.0),
        ), H=22, D=96, dtype="f16", topk=16, radius=2,
        description="4 packed shells of 80k/90k/110k/60k cells in 64^3/128^3/192^3/128^3 grids"),
}


# --------------------------------------------------------------------------------------------
# voxel shells
# --------------------------------------------------------------------------------------------

def _grid_points(grid):
    gx, gy, gz = grid
    x, y, z = np.meshgrid(np.arange(gx), np.arange(gy), np.arange(gz), indexing="ij")
    return np.stack([x.ravel(), y.ravel(), z.ravel()], axis=1).astype(np.int32)


def _random_rotation(rng):
    # QR of a Gaussian matrix, sign-fixed: a uniformly random rotation.
    a = rng.standard_normal((3, 3))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def _shape_params(rng, grid, n_shapes, boxes):
    g = np.asarray(grid, dtype=np.float64)
    shapes = []
    for s in range(n_shapes):
        kind = "box" if (boxes and s % 2 == 1) else "ellipsoid"
        centre = g * rng.uniform(0.35, 0.65, size=3)
        axes = g * rng.uniform(0.12, 0.26, size=3)
        shapes.append((kind, centre, axes, _random_rotation(rng)))
    return shapes


class _UnionField:
    """Approximate signed distance (voxels, negative inside) to a union of scaled solids.

    Per-shape local coordinates are computed once; each scale is then cheap.
    """

    def __init__(self, points, shapes):
        p = points.astype(np.float32) + np.float32(0.5)
        self.parts = []
        for kind, centre, axes, rot in shapes:
            local = (p - centre.astype(np.float32)) @ rot.astype(np.float32)
            if kind == "ellipsoid":
                k1 = np.linalg.norm(local / axes.astype(np.float32), axis=1)
                rad = np.linalg.norm(local, axis=1)
                self.parts.append((kind, axes, k1, rad))
            else:
                self.parts.append((kind, axes, np.abs(local), None))

    def distance(self, scale):
        best = None
        for kind, axes, a0, a1 in self.parts:
            if kind == "ellipsoid":
                # radial distance to the scaled surface along the ray from the centre
                d = np.where(a0 > 1e-6, (1.0 - scale / np.maximum(a0, 1e-6)) * a1,
                             -float(axes.min() * scale)).astype(np.float32)
            else:
                q = a0 - (axes * scale).astype(np.float32)
                d = np.linalg.norm(np.maximum(q, 0.0), axis=1) + np.minimum(q.max(axis=1), 0.0)
            best = d if best is None else np.minimum(best, d)
        return best


def _sample(rng, cells, n_target):
    if n_target is None or len(cells) <= n_target:
        return cells
    keep = np.sort(rng.choice(len(cells), size=n_target, replace=False))
    return cells[keep]


def shell_coords(spec: ShapeSpec, seed: int) -> np.ndarray:
    """int32 [n,3] voxel coordinates of one shell, in lexicographic (x, y, z) order."""
    rng = np.random.default_rng(seed)
    pts = _grid_points(spec.grid)
    if spec.kind == "sphere":
        c = np.asarray(spec.grid, dtype=np.float64) / 2.0
        rad = np.linalg.norm(pts - c, axis=1)
        cells = pts[(rad >= 11.5) & (rad < 12.5)]
    elif spec.kind == "torus":
        c = np.asarray(spec.grid, dtype=np.float64) / 2.0
        q = pts - c
        ring = np.linalg.norm(q[:, :2], axis=1) - 40.0
        d = np.sqrt(ring * ring + q[:, 2] ** 2) - 15.0
        cells = pts[np.abs(d) < 1.0]
    elif spec.kind == "union_grow":
        # shapes fixed; shell thickness grows one voxel at a time until it holds n_target cells
        field = _UnionField(pts, _shape_params(rng, spec.grid, spec.n_shapes, spec.boxes))
        scale = 1.0
        while True:
            d = field.distance(scale)
            if (d <= 0).sum() >= spec.n_target:
                break
            scale *= 1.08
        t = 1.0
        while True:
            cells = pts[(d <= 0) & (d > -t)]
            if len(cells) >= spec.n_target:
                break
            t += 1.0
    elif spec.kind == "union_scale":
        # thickness fixed; shapes scaled up by 5% steps until the shell holds n_target cells
        field = _UnionField(pts, _shape_params(rng, spec.grid, spec.n_shapes, spec.boxes))
        scale = 0.6
        while True:
            d = field.distance(scale)
            cells = pts[(d <= 0) & (d > -spec.thickness)]
            if len(cells) >= spec.n_target or scale > 4.0:
                break
            scale *= 1.05
    else:
        raise ValueError(spec.kind)
    return np.ascontiguousarray(_sample(rng, cells, spec.n_target), dtype=np.int32)


def make_coords(cfg: WorkloadConfig):
    """Packed coordinates of all sequences.

    Returns (coords int32 [N,3], cu_seqlens int64 [B+1], grids int32 [B,3]).
    """
    parts = [shell_coords(s, cfg.index * 1000 + TID_COORDS + 100 * i)
             for i, s in enumerate(cfg.shapes)]
    cu = np.zeros(len(parts) + 1, dtype=np.int64)
    cu[1:] = np.cumsum([len(p) for p in parts])
    grids = np.asarray([s.grid for s in cfg.shapes], dtype=np.int32)
    return np.ascontiguousarray(np.concatenate(parts, axis=0)), cu, grids


# --------------------------------------------------------------------------------------------
# tensors
# --------------------------------------------------------------------------------------------

def _torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]


def normal_tensor(shape: Sequence[int], dtype: str, seed: int, std: float = 1.0):
    """N(0, std^2) draws in fp32, rounded once to `dtype` (a CPU torch tensor)."""
    import torch
    x = np.random.default_rng(seed).standard_normal(tuple(shape), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return torch.from_numpy(x).to(_torch_dtype(dtype))


def uniform_tensor(shape: Sequence[int], seed: int):
    import torch
    return torch.from_numpy(np.random.default_rng(seed).random(tuple(shape), dtype=np.float32))


def make_tensors(cfg: WorkloadConfig, N: int, with_grad_out: bool = False):
    """Q, K, V [N,H,D] in cfg.dtype; gates [N,H,3] ~ U(0,1) fp32; Wc [D,D] ~ N(0,1/D) fp32."""
    base = cfg.index * 1000
    H, D = cfg.H, cfg.D
    out = dict(
        Q=normal_tensor((N, H, D), cfg.dtype, base + TID_Q),
        K=normal_tensor((N, H, D), cfg.dtype, base + TID_K),
        V=normal_tensor((N, H, D), cfg.dtype, base + TID_V),
        gates=uniform_tensor((N, H, 3), base + TID_GATES),
        Wc=normal_tensor((D, D), "f32", base + TID_WC, std=1.0 / np.sqrt(D)),
    )
    if with_grad_out:
        out["dO"] = normal_tensor((N, H, D), cfg.dtype, base + TID_DO)
    return out


def stratified_rows(cu_seqlens: np.ndarray, per_seq: int, seed: int) -> List[np.ndarray]:
    """A fixed, seeded sample of `per_seq` query rows from each sequence (global indices)."""
    rng = np.random.default_rng(seed)
    rows = []
    for s in range(len(cu_seqlens) - 1):
        lo, hi = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        n = hi - lo
        take = min(per_seq, n)
        rows.append(np.sort(rng.choice(n, size=take, replace=False)).astype(np.int64) + lo)
    return rows

"""The synthetic workloads follow the shapes the Hi3D v1.0 pipeline page prints."""
import os

import numpy as np

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pipeline_shapes.txt")


def _golden():
    passes, kv = [], {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        f = line.split()
        if f[0] == "pass":
            passes.append((int(f[1]), int(f[2])))
        else:
            kv[f[0]] = int(f[1])
    return passes, kv


def test_pass_shaped_workloads_match_the_pages_table():
    passes, kv = _golden()
    C = workloads.CONFIGS
    assert (C["pass1"].shapes[0].grid[0], C["pass1"].shapes[0].n_target) == passes[0]
    assert (C["pass3"].shapes[0].grid[0], C["pass3"].shapes[0].n_target) == passes[2]
    vl = C["varlen"].shapes
    assert [(s.grid[0], s.n_target) for s in vl[:3]] == passes
    for name in ("pass1", "pass3", "varlen"):
        assert C[name].H == kv["heads"] and C[name].H * C[name].D == kv["width"]


def test_generators_are_seeded_and_unique():
    cfg = workloads.CONFIGS["small"]
    a, cu, g = workloads.make_coords(cfg)
    b, _, _ = workloads.make_coords(cfg)
    assert np.array_equal(a, b)
    assert len(np.unique(a, axis=0)) == len(a) == 20000
    assert (a >= 0).all() and (a < 128).all()
    t1 = workloads.make_tensors(cfg, 100)
    t2 = workloads.make_tensors(cfg, 100)
    assert all((t1[k] == t2[k]).all() for k in t1)

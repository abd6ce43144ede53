"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against one of: a library routine for a special case
(dense softmax attention via torch's scaled_dot_product_attention, numpy/torch
float conversions), a closed form, an invariant of the method, a planted input
with a known answer, a brute-force restatement on tiny inputs, or finite
differences. A dropped term, a wrong sign or index, or a transposed operand in
the oracle fails at least one of them.

The method: Direct3D-S2 summary page, "Technical principles", SSA item
(partition by 3D coordinates; block compression; top-k blocks by compression
scores; local window; gated aggregation).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

F32, BF16, F16, F64 = oracle.F32, oracle.BF16, oracle.F16, oracle.F64


def _tiny_coords():
    c, cu, g = workloads.make_coords(workloads.CONFIGS["tiny"])
    return c, cu


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


def _gates(N, H, g, seed=0):
    if g is None:
        return np.random.default_rng(seed).random((N, H, 3)).astype(np.float32)
    return np.broadcast_to(np.asarray(g, np.float32), (N, H, 3)).copy()


def dense_attention(q, k, v):
    """softmax(q k^T / sqrt(D)) v per head via torch's library routine, fp64. [N,H,D] in/out."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)).permute(1, 0, 2) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    return o.permute(1, 0, 2).numpy()


def run(coords, q, k, v, gates, Wc, topk, r, **kw):
    cu = np.array([0, len(coords)])
    return oracle.forward(coords, cu, q, k, v, gates, Wc, topk, r, **kw)


# ---------------------------------------------------------------------------------------------
# storage-type decoding and rounding (checked against numpy / torch conversions)
# ---------------------------------------------------------------------------------------------

def test_decode_f16_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, F16)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_decode_bf16_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, BF16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_round_to_f16_matches_numpy():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-8, 5, 3000),
        (np.arange(-2000, 2000) + 0.5) * 2.0 ** -10,       # exact ties at the unit scale
        (np.arange(-300, 300) + 0.5) * 2.0 ** -24,         # ties in the subnormal range
        [65504.0, 65519.9, 65520.0, -70000.0, 0.0, -0.0],
    ])
    ours = oracle.round_to(x, F16)
    ref = x.astype(np.float16).astype(np.float64)
    assert np.array_equal(ours, ref)


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000)).astype(np.float32)
    ours = oracle.round_to(x.astype(np.float64), BF16)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------------------------------------
# partition and window lists
# ---------------------------------------------------------------------------------------------

def test_partition_matches_plain_grouping():
    c, _ = _tiny_coords()
    c = c[np.random.default_rng(3).permutation(len(c))]
    perm, tok_blk, blk_off, blk_coord = oracle.partition(c, 8)
    groups = {}
    for i, xyz in enumerate(c):
        groups.setdefault(tuple(int(t) // 8 for t in xyz), []).append(i)
    keys = sorted(groups)
    assert [tuple(b) for b in blk_coord] == keys
    assert list(perm) == [i for kk in keys for i in groups[kk]]
    assert list(np.diff(blk_off)) == [len(groups[kk]) for kk in keys]
    assert blk_off[-1] == len(c)
    for b, kk in enumerate(keys):
        assert all(tok_blk[i] == b for i in groups[kk])


@pytest.mark.parametrize("r", [0, 1, 2, 3])
def test_window_matches_pairwise_brute_force(r):
    c, _ = _tiny_coords()
    rng = np.random.default_rng(4 + r)
    sub = c[rng.choice(len(c), 500, replace=False)]
    off, idx = oracle.window(sub, r)
    d = np.abs(sub[:, None, :] - sub[None, :, :]).max(axis=2)
    for i in range(len(sub)):
        ref = np.nonzero(d[i] <= r)[0]
        assert np.array_equal(idx[off[i]:off[i + 1]], ref)
    off_b, idx_b = oracle.window(sub, r, brute=True)
    assert np.array_equal(off, off_b) and np.array_equal(idx, idx_b)


def test_window_invariants():
    c, _ = _tiny_coords()
    r = 2
    off, idx = oracle.window(c, r)
    pairs = set()
    for i in range(len(c)):
        row = idx[off[i]:off[i + 1]]
        assert i in row
        assert len(row) <= (2 * r + 1) ** 3
        assert np.all(np.diff(row) > 0)
        pairs.update((i, int(j)) for j in row)
    assert all((j, i) in pairs for (i, j) in pairs)


def test_window_rejects_duplicates():
    c = np.array([[1, 2, 3], [4, 5, 6], [1, 2, 3]], np.int32)
    with pytest.raises(ValueError):
        oracle.window(c, 1)


# ---------------------------------------------------------------------------------------------
# branches reduce to dense attention in their limiting cases
# ---------------------------------------------------------------------------------------------

def _tiny_inputs(seed=10, H=2, D=32):
    c, _ = _tiny_coords()
    N = len(c)
    q, k, v = (_rand((N, H, D), seed + t) for t in range(3))
    Wc = _rand((D, D), seed + 3) / np.sqrt(D)
    return c, q, k, v, Wc.astype(np.float32)


def test_selection_branch_is_dense_attention_when_k_covers_all_blocks():
    c, q, k, v, Wc = _tiny_inputs()
    mb = len(oracle.partition(c)[3])
    res = run(c, q, k, v, _gates(len(c), 2, (0, 1, 0)), Wc, topk=mb + 3, r=1)
    ref = dense_attention(q, k, v)
    np.testing.assert_allclose(res["o_sel"], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)
    assert np.all(res["sel"][:, :, mb:] == -1)
    assert np.all(np.sort(res["sel"][:, :, :mb], axis=2) == np.arange(mb))


def test_window_branch_is_dense_attention_when_radius_covers_grid():
    c, q, k, v, Wc = _tiny_inputs(seed=20)
    res = run(c, q, k, v, _gates(len(c), 2, (0, 0, 1)), Wc, topk=4, r=40)
    np.testing.assert_allclose(res["out"], dense_attention(q, k, v), rtol=0, atol=1e-12)


def test_compressed_branch_is_dense_attention_on_a_lattice():
    # one token per block (coordinates on multiples of 8) and Wc = I: compressed tokens are the
    # tokens themselves, so the compressed branch is dense attention over all tokens.
    g = np.arange(0, 64, 8)
    c = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3).astype(np.int32)
    N, H, D = len(c), 2, 16
    q, k, v = (_rand((N, H, D), 30 + t) for t in range(3))
    res = run(c, q, k, v, _gates(N, H, (1, 0, 0)), np.eye(D, dtype=np.float32), topk=3, r=1,
              round_compressed=False)
    np.testing.assert_allclose(res["out"], dense_attention(q, k, v), rtol=0, atol=1e-12)


def test_constant_values_give_closed_forms():
    c, q, k, v, Wc = _tiny_inputs(seed=40)
    ones = np.ones_like(v)
    res = run(c, q, k, ones, _gates(len(c), 2, None), Wc, topk=4, r=2, round_compressed=False)
    np.testing.assert_allclose(res["o_sel"], 1.0, atol=1e-13)
    np.testing.assert_allclose(res["o_win"], 1.0, atol=1e-13)
    colsum = Wc.astype(np.float64).sum(axis=0)      # 1^T . Wc: the compressed value of V = 1
    np.testing.assert_allclose(res["o_cmp"], np.broadcast_to(colsum, res["o_cmp"].shape),
                               atol=1e-12)


def test_pooling_of_block_constant_keys():
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    perm, tok_blk, blk_off, blk_coord = oracle.partition(c)
    mb = len(blk_coord)
    cb = _rand((mb, H, D), 50)
    k = cb[tok_blk]                      # every token carries its block's constant key
    Wc = _rand((D, D), 51).astype(np.float32)
    Kc, Vc = oracle.compress(c, k, k, Wc)
    ref = np.einsum("bhd,de->bhe", cb, Wc.astype(np.float64))
    np.testing.assert_allclose(Kc, ref, atol=1e-12)
    np.testing.assert_allclose(Vc, ref, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------------------------

def test_output_is_linear_in_the_gates():
    c, q, k, v, Wc = _tiny_inputs(seed=60)
    N = len(c)
    # multiples of 1/16, so ga + gb is exact in fp32
    ga = np.floor(_gates(N, 2, None, seed=1) * 16) / 16
    gb = np.floor(_gates(N, 2, None, seed=2) * 16) / 16
    ra = run(c, q, k, v, ga, Wc, 4, 2)["out"]
    rb = run(c, q, k, v, gb, Wc, 4, 2)["out"]
    rab = run(c, q, k, v, ga + gb, Wc, 4, 2)["out"]
    np.testing.assert_allclose(rab, ra + rb, atol=1e-12)


def test_permutation_equivariance():
    c, q, k, v, Wc = _tiny_inputs(seed=70)
    N = len(c)
    g = _gates(N, 2, None)
    base = run(c, q, k, v, g, Wc, 4, 2)
    p = np.random.default_rng(71).permutation(N)
    shuf = run(c[p], q[p], k[p], v[p], g[p], Wc, 4, 2)
    np.testing.assert_allclose(shuf["out"], base["out"][p], atol=1e-12)
    # blocks are indexed by coordinate, not by token order: the selection is unchanged
    assert np.array_equal(shuf["sel"], base["sel"][p])


def test_window_of_radius_zero_is_the_token_itself():
    # W(i) = {i} at r = 0: one key, weight exactly 1, so o_win is the token's own value
    c, q, k, v, Wc = _tiny_inputs(seed=75)
    off, idx = oracle.window(c, 0)
    assert np.array_equal(off, np.arange(len(c) + 1))
    assert np.array_equal(idx, np.arange(len(c)))
    res = run(c, q, k, v, _gates(len(c), 2, (0, 0, 1)), Wc, 4, 0)
    assert np.array_equal(res["o_win"], v)
    assert np.array_equal(res["out"], v)


def test_branches_are_linear_in_the_values():
    # V enters every branch only through the final weighted sum (the compressed one after the
    # linear mean and Wc), and the selection depends on Q and K alone
    c, q, k, v, Wc = _tiny_inputs(seed=76)
    v2 = _rand(v.shape, 77)
    g = _gates(len(c), 2, None)
    a = run(c, q, k, v, g, Wc, 4, 2)
    b = run(c, q, k, v2, g, Wc, 4, 2)
    ab = run(c, q, k, 2.0 * v - 3.0 * v2, g, Wc, 4, 2)
    for name in ("o_cmp", "o_sel", "o_win", "out"):
        np.testing.assert_allclose(ab[name], 2.0 * a[name] - 3.0 * b[name], rtol=0, atol=1e-12)
    assert np.array_equal(a["sel"], b["sel"]) and np.array_equal(a["sel"], ab["sel"])


def test_packed_sequences_are_independent():
    # a second, different shell packed behind the first: each sequence's rows equal a run on
    # that sequence alone; its block indices continue after the first sequence's blocks
    c1, q1, k1, v1, Wc = _tiny_inputs(seed=78)
    c2 = np.ascontiguousarray(c1[::2][:, [1, 0, 2]] + np.array([0, 3, 5], np.int32))
    n1, n2 = len(c1), len(c2)
    q2, k2, v2 = (_rand((n2, 2, 32), 79 + t) for t in range(3))
    g1, g2 = _gates(n1, 2, None, seed=3), _gates(n2, 2, None, seed=4)
    cat = lambda a, b: np.concatenate([a, b], axis=0)
    cu = np.array([0, n1, n1 + n2])
    both = oracle.forward(cat(c1, c2), cu, cat(q1, q2), cat(k1, k2), cat(v1, v2), cat(g1, g2),
                          Wc, 4, 2)
    one = run(c1, q1, k1, v1, g1, Wc, 4, 2)
    two = run(c2, q2, k2, v2, g2, Wc, 4, 2)
    mb1 = len(oracle.partition(c1)[3])
    for name in ("o_cmp", "o_sel", "o_win", "out"):
        np.testing.assert_allclose(both[name][:n1], one[name], rtol=0, atol=1e-13)
        np.testing.assert_allclose(both[name][n1:], two[name], rtol=0, atol=1e-13)
    assert np.array_equal(both["sel"][:n1], one["sel"])
    assert np.array_equal(both["sel"][n1:], np.where(two["sel"] >= 0, two["sel"] + mb1, -1))
    p = oracle.plan(cat(c1, c2), cu, r=2)
    p1, p2 = oracle.plan(c1, [0, n1], r=2), oracle.plan(c2, [0, n2], r=2)
    assert np.array_equal(p["perm"], cat(p1["perm"], p2["perm"] + n1))
    assert np.array_equal(p["blk_off"], cat(p1["blk_off"][:-1], p2["blk_off"] + n1))
    assert np.array_equal(p["nbr_idx"], cat(p1["nbr_idx"], p2["nbr_idx"] + n1))


def test_translation_by_whole_blocks():
    c, q, k, v, Wc = _tiny_inputs(seed=80)
    g = _gates(len(c), 2, None)
    base = run(c, q, k, v, g, Wc, 4, 2)
    moved = run(c + np.array([8, 16, 24], np.int32), q, k, v, g, Wc, 4, 2)
    np.testing.assert_allclose(moved["out"], base["out"], atol=1e-12)
    assert np.array_equal(moved["sel"], base["sel"])


# ---------------------------------------------------------------------------------------------
# planted top-k
# ---------------------------------------------------------------------------------------------

def planted_case(dtype=np.float64, H=2, D=16, seed=90):
    """Every query is e = 1; every key of block b is alpha_b * 1; Wc = I.

    Then Kc_b = alpha_b * 1 and the compressed logit is z_b = alpha_b * D / sqrt(D), so the
    expected ranking is by alpha (ties -> lower block index), independent of any arithmetic.
    Alphas are multiples of 1/8 (exact in every storage type); two blocks are tied on purpose.
    """
    c, _ = _tiny_coords()
    N = len(c)
    perm, tok_blk, blk_off, blk_coord = oracle.partition(c)
    mb = len(blk_coord)
    rng = np.random.default_rng(seed)
    alpha = np.stack([rng.permutation(mb) for _ in range(H)], axis=1).astype(np.float64)
    alpha = (alpha - mb / 2) / 8.0
    alpha[7, 0] = alpha[3, 0]                   # planted tie in head 0: block 3 must win it
    q = np.ones((N, H, D), dtype)
    k = np.repeat(alpha[tok_blk][:, :, None], D, axis=2).astype(dtype)
    v = _rand((N, H, D), seed + 1, dtype)
    return c, tok_blk, alpha, q, k, v


def expected_selection(tok_blk, alpha, topk):
    N, H = len(tok_blk), alpha.shape[1]
    mb = alpha.shape[0]
    sel = np.full((N, H, topk), -1, np.int64)
    for i in range(N):
        for h in range(H):
            own = tok_blk[i]
            others = sorted((b for b in range(mb) if b != own), key=lambda b: (-alpha[b, h], b))
            row = [own] + others[:topk - 1]
            sel[i, h, :len(row)] = row
    return sel


def test_planted_topk_is_exact():
    c, tok_blk, alpha, q, k, v = planted_case()
    N, H, D = q.shape
    topk = 6
    res = run(c, q, k, v, _gates(N, H, None), np.eye(D, dtype=np.float32), topk, 2)
    assert np.array_equal(res["sel"], expected_selection(tok_blk, alpha, topk))


def test_planted_topk_with_fewer_blocks_than_k():
    c, tok_blk, alpha, q, k, v = planted_case()
    N, H, D = q.shape
    mb = alpha.shape[0]
    res = run(c, q, k, v, _gates(N, H, None), np.eye(D, dtype=np.float32), mb + 2, 2)
    assert np.array_equal(res["sel"], expected_selection(tok_blk, alpha, mb + 2))


# ---------------------------------------------------------------------------------------------
# brute-force restatement on a tiny input (no plan, plain loops)
# ---------------------------------------------------------------------------------------------

def brute_forward(coords, q, k, v, gates, Wc, topk, r):
    N, H, D = q.shape
    s = 1.0 / np.sqrt(D)
    W = Wc.astype(np.float64)
    key = [tuple(int(t) // 8 for t in xyz) for xyz in coords]
    blocks = sorted(set(key))
    members = [[i for i in range(N) if key[i] == b] for b in blocks]
    out = np.zeros((N, H, D))

    def softmax_mix(qv, kk, vv):
        z = s * (kk @ qv)
        e = np.exp(z - z.max())
        return (e / e.sum()) @ vv

    for h in range(H):
        Kc = np.array([k[m, h].mean(axis=0) @ W for m in members])
        Vc = np.array([v[m, h].mean(axis=0) @ W for m in members])
        for i in range(N):
            z = s * (Kc @ q[i, h])
            o_cmp = softmax_mix(q[i, h], Kc, Vc)
            own = blocks.index(key[i])
            others = sorted((b for b in range(len(blocks)) if b != own), key=lambda b: (-z[b], b))
            J = [j for b in [own] + others[:topk - 1] for j in members[b]]
            o_sel = softmax_mix(q[i, h], k[J, h], v[J, h])
            Wn = [j for j in range(N) if np.abs(coords[j] - coords[i]).max() <= r]
            o_win = softmax_mix(q[i, h], k[Wn, h], v[Wn, h])
            g = gates[i, h].astype(np.float64)
            out[i, h] = g[0] * o_cmp + g[1] * o_sel + g[2] * o_win
    return out


def test_brute_force_agrees_on_tiny_input():
    c, _ = _tiny_coords()
    c = c[:260]
    N, H, D = len(c), 2, 8
    q, k, v = (_rand((N, H, D), 100 + t) for t in range(3))
    Wc = (_rand((D, D), 104) / np.sqrt(D)).astype(np.float32)
    g = _gates(N, H, None, seed=5)
    res = run(c, q, k, v, g, Wc, 3, 2, round_compressed=False)
    np.testing.assert_allclose(res["out"], brute_forward(c, q, k, v, g, Wc, 3, 2), atol=1e-12)


def test_fp16_inputs_are_decoded_exactly():
    c, q, k, v, Wc = _tiny_inputs(seed=110)
    qh, kh, vh = (x.astype(np.float16) for x in (q, k, v))
    g = _gates(len(c), 2, None)
    a = run(c, qh, kh, vh, g, Wc, 4, 2, round_compressed=False)
    b = run(c, qh.astype(np.float64), kh.astype(np.float64), vh.astype(np.float64), g, Wc, 4, 2,
            round_compressed=False)
    np.testing.assert_array_equal(a["out"], b["out"])


# ---------------------------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------------------------

def test_backward_selection_branch_is_dense_attention_backward():
    c, _ = _tiny_coords()
    c = c[:400]
    N, H, D = len(c), 2, 16
    q, k, v, dO = (_rand((N, H, D), 120 + t) for t in range(4))
    mb = len(oracle.partition(c)[3])
    g = _gates(N, H, (0, 1, 0))
    cu = np.array([0, N])
    dQ, dK, dV = oracle.backward(c, cu, q, k, v, g, np.eye(D, dtype=np.float32), dO, mb + 1, 1,
                                 round_compressed=False)
    qt, kt, vt = (torch.from_numpy(x).permute(1, 0, 2).requires_grad_() for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    (o * torch.from_numpy(dO).permute(1, 0, 2)).sum().backward()
    for ours, ref in ((dQ, qt.grad), (dK, kt.grad), (dV, vt.grad)):
        np.testing.assert_allclose(ours, ref.permute(1, 0, 2).numpy(), atol=1e-12)


def test_backward_matches_finite_differences():
    c, _ = _tiny_coords()
    c = c[:150]
    N, H, D = len(c), 1, 8
    rng = np.random.default_rng(130)
    q, k, v, dO = (rng.standard_normal((N, H, D)) for _ in range(4))
    Wc = (rng.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32)
    g = _gates(N, H, None, seed=7)
    topk, r = 2, 1
    cu = np.array([0, N])
    dQ, dK, dV = oracle.backward(c, cu, q, k, v, g, Wc, dO, topk, r, round_compressed=False)
    base_sel = run(c, q, k, v, g, Wc, topk, r, round_compressed=False)["sel"]

    def loss(qq, kk, vv):
        res = run(c, qq, kk, vv, g, Wc, topk, r, round_compressed=False)
        assert np.array_equal(res["sel"], base_sel)   # the selection must not move
        return float((res["out"] * dO).sum())

    eps = 1e-6
    for name, x, grad in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        for t in rng.choice(x.size, 12, replace=False):
            xp, xm = x.copy(), x.copy()
            xp.flat[t] += eps
            xm.flat[t] -= eps
            args_p = [xp if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad.flat[t]) <= 1e-6 * max(1.0, abs(fd)), (name, t, fd, grad.flat[t])


def test_backward_dq_rows_matches_full_backward():
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    q, k, v, dO = (_rand((N, H, D), 140 + t) for t in range(4))
    Wc = (_rand((D, D), 145) / np.sqrt(D)).astype(np.float32)
    g = _gates(N, H, None, seed=9)
    cu = np.array([0, N])
    dQ, _, _ = oracle.backward(c, cu, q, k, v, g, Wc, dO, 4, 2)
    rows = np.array([0, 5, 77, 1000, N - 1])
    dq = oracle.backward_dq_rows(c, cu, q, k, v, g, Wc, dO, 4, 2, rows)
    np.testing.assert_allclose(dq, dQ[rows], atol=1e-13)


def test_backward_gradient_sums():
    # sum_j dK_j = 0 for every head (each branch's dz rows sum to zero, and the compression
    # map spreads dKc_b evenly over the block); sum_j dV_j = sum_i (g0 dO_i Wc^T + g1 dO_i + g2 dO_i)
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    q, k, v, dO = (_rand((N, H, D), 150 + t) for t in range(4))
    Wc = (_rand((D, D), 155) / np.sqrt(D)).astype(np.float32)
    g = _gates(N, H, None, seed=11)
    cu = np.array([0, N])
    dQ, dK, dV = oracle.backward(c, cu, q, k, v, g, Wc, dO, 4, 2)
    np.testing.assert_allclose(dK.sum(axis=0), 0.0, atol=1e-10)
    gd = g.astype(np.float64)
    ref = (np.einsum("nh,nhd->hd", gd[:, :, 0], dO) @ Wc.astype(np.float64).T
           + np.einsum("nh,nhd->hd", gd[:, :, 1] + gd[:, :, 2], dO))
    np.testing.assert_allclose(dV.sum(axis=0), ref, atol=1e-10)


def _random_selection(tok_blk_global, blk_seq, topk, H, seed):
    """A valid selection that is not the oracle's: slot 0 the own block, then topk-1 distinct
    other blocks of the token's own sequence drawn at random (-1 where the sequence has fewer)."""
    rng = np.random.default_rng(seed)
    N = len(tok_blk_global)
    sel = np.full((N, H, topk), -1, np.int32)
    for i in range(N):
        own = tok_blk_global[i]
        pool = np.nonzero(blk_seq == blk_seq[own])[0]
        pool = pool[pool != own]
        for h in range(H):
            pick = rng.permutation(pool)[:topk - 1]
            sel[i, h, 0] = own
            sel[i, h, 1:1 + len(pick)] = pick
    return sel


def test_backward_with_a_given_selection_matches_finite_differences():
    # two packed sequences and a random valid selection (global block indices): the backward that
    # holds this selection is the derivative of the forward that uses it (central differences,
    # fp64), and dQ by rows with the same selection equals the full backward's rows
    c1, _ = _tiny_coords()
    c1 = c1[:120]
    c2 = np.ascontiguousarray(c1[::2][:, [2, 0, 1]])
    c = np.concatenate([c1, c2])
    cu = np.array([0, len(c1), len(c)])
    N, H, D, topk, r = len(c), 2, 8, 3, 1
    rng = np.random.default_rng(160)
    q, k, v, dO = (rng.standard_normal((N, H, D)) for _ in range(4))
    Wc = (rng.standard_normal((D, D)) / np.sqrt(D)).astype(np.float32)
    g = _gates(N, H, None, seed=13)
    p = oracle.plan(c, cu, r=r)
    sel = _random_selection(p["tok_blk"], p["blk_seq"], topk, H, seed=161)
    own = oracle.forward(c, cu, q, k, v, g, Wc, topk, r)["sel"]
    assert not np.array_equal(np.sort(own, 2), np.sort(sel, 2))   # a different choice
    dQ, dK, dV = oracle.backward(c, cu, q, k, v, g, Wc, dO, topk, r, sel=sel)

    def loss(qq, kk, vv):
        return float((oracle.forward(c, cu, qq, kk, vv, g, Wc, topk, r, sel_in=sel)["out"] * dO).sum())

    eps = 1e-6
    for name, x, grad in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        for t in rng.choice(x.size, 10, replace=False):
            xp, xm = x.copy(), x.copy()
            xp.flat[t] += eps
            xm.flat[t] -= eps
            args_p = [xp if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad.flat[t]) <= 1e-6 * max(1.0, abs(fd)), (name, t, fd, grad.flat[t])
    rows = np.array([0, 7, len(c1) - 1, len(c1), N - 1])
    dq, used = oracle.backward_dq_rows(c, cu, q, k, v, g, Wc, dO, topk, r, rows, sel_in=sel[rows],
                                       return_sel=True)
    assert np.array_equal(used, sel[rows])
    np.testing.assert_allclose(dq, dQ[rows], atol=1e-13)


def test_selection_only_mode_gives_the_same_selection_and_compressed_branch():
    c, q, k, v, Wc = _tiny_inputs(seed=170)
    g = _gates(len(c), 2, None, seed=14)
    full = run(c, q, k, v, g, Wc, 4, 2, want_z=True)
    part = run(c, q, k, v, g, Wc, 4, 2, want_z=True, branches=False)
    assert np.array_equal(full["sel"], part["sel"])
    np.testing.assert_array_equal(full["o_cmp"], part["o_cmp"])
    for a, b in zip(full["z"], part["z"]):
        np.testing.assert_array_equal(a, b)
    assert not part["out"].any() and not part["o_sel"].any() and not part["o_win"].any()


def test_backward_is_the_same_with_any_thread_count():
    # the key / value gradients are summed over per-thread copies; with one thread or several the
    # result agrees to rounding
    import subprocess
    import sys
    code = ("import numpy as np, sys; sys.path.insert(0, %r); import oracle, workloads;"
            "c, cu, g = workloads.make_coords(workloads.CONFIGS['tiny']); N = len(c);"
            "r = np.random.default_rng(180); q, k, v, d = (r.standard_normal((N, 2, 8)) for _ in range(4));"
            "W = (r.standard_normal((8, 8)) / 3).astype(np.float32); gt = r.random((N, 2, 3)).astype(np.float32);"
            "out = oracle.backward(c, cu, q, k, v, gt, W, d, 4, 2);"
            "np.save(sys.argv[1], np.stack(out))") % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),)
    import tempfile
    res = []
    with tempfile.TemporaryDirectory() as tmp:
        for threads in ("1", "5"):
            f = os.path.join(tmp, f"g{threads}.npy")
            env = dict(os.environ, OMP_NUM_THREADS=threads)
            subprocess.check_call([sys.executable, "-c", code, f], env=env)
            res.append(np.load(f))
    np.testing.assert_allclose(res[0], res[1], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# attention prologue: RMS normalisation of queries and keys, 3D rotary position embedding
# ---------------------------------------------------------------------------------------------

def test_prologue_rmsnorm_closed_forms():
    # at the origin every rotation angle is 0, so only the normalisation acts: with eps = 0 and a
    # unit weight the mean square over the head dimension is exactly 1; the result does not
    # depend on the input's scale; a weight vector multiplies channel by channel
    N, H, D = 40, 3, 32
    x = _rand((N, H, D), 190)
    zero = np.zeros((N, 3), np.int32)
    ones = np.ones(D, np.float32)
    u = oracle.qk_prologue(x, zero, ones, eps=0.0)
    np.testing.assert_allclose((u ** 2).mean(axis=2), 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.qk_prologue(3.7 * x, zero, ones, eps=0.0), u, rtol=1e-12)
    gamma = np.random.default_rng(191).random(D).astype(np.float32) + 0.5
    np.testing.assert_allclose(oracle.qk_prologue(x, zero, gamma, eps=0.0),
                               u * gamma.astype(np.float64), rtol=1e-13)
    # eps enters under the root: a constant row c gives c / sqrt(c^2 + eps)
    c = np.full((1, 1, D), 0.01)
    np.testing.assert_allclose(oracle.qk_prologue(c, zero[:1], ones, eps=1e-4),
                               0.01 / np.sqrt(1e-4 + 1e-4), rtol=1e-13)


@pytest.mark.parametrize("D", [32, 64, 96, 128])
def test_prologue_rotation_angles(D):
    # a unit vector on channel c (the first of a pair) normalises to sqrt(D) e_c; at position p
    # along the part's axis the pair becomes sqrt(D) (cos t, sin t), t = p theta^(-2j / width),
    # and the parts of the other two axes do not move
    widths = oracle.rope_split(D)
    assert sum(widths) == D and all(w % 2 == 0 for w in widths)
    theta = 10000.0
    starts = np.cumsum((0,) + widths[:2])
    ones = np.ones(D, np.float32)
    for a in range(3):
        for j in (0, 1, widths[a] // 2 - 1):
            c = starts[a] + 2 * j
            x = np.zeros((1, 1, D))
            x[0, 0, c] = 1.0
            for p in (1, 5, 37):
                pos = np.zeros((1, 3), np.int32)
                pos[0, a] = p
                u = oracle.qk_prologue(x, pos, ones, eps=0.0, theta=theta)[0, 0]
                t = p * theta ** (-2.0 * j / widths[a])
                exp = np.zeros(D)
                exp[c], exp[c + 1] = np.sqrt(D) * np.cos(t), np.sqrt(D) * np.sin(t)
                np.testing.assert_allclose(u, exp, atol=1e-12)


def test_prologue_scores_depend_on_relative_position():
    # rotations of both operands by their own positions: q.k depends only on the offset, so
    # moving both tokens by the same vector keeps every score
    D = 96
    rng = np.random.default_rng(192)
    q, k = rng.standard_normal((2, 1, 1, D))
    gq, gk = (rng.random(D).astype(np.float32) + 0.5 for _ in range(2))
    pq, pk = np.array([[3, 17, 40]], np.int32), np.array([[9, 2, 33]], np.int32)
    shift = np.array([[11, 250, 7]], np.int32)
    a = (oracle.qk_prologue(q, pq, gq) * oracle.qk_prologue(k, pk, gk)).sum()
    b = (oracle.qk_prologue(q, pq + shift, gq) * oracle.qk_prologue(k, pk + shift, gk)).sum()
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a))
    c = (oracle.qk_prologue(q, pq, gq) * oracle.qk_prologue(k, pq, gk)).sum()
    assert abs(a - c) > 1e-3   # the offset itself does matter


def test_forward_with_prologue_is_invariant_under_block_translation():
    # the whole method with the prologue: moving every token by whole blocks keeps the blocks,
    # the windows and (through the rotary embedding's relative form) every attention score. The
    # compressed keys are block means of rotated keys times Wc, so a Wc that commutes with the
    # rotations (a multiple of the identity) keeps the compressed scores relative as well.
    c, q, k, v, _ = _tiny_inputs(seed=193)
    g = _gates(len(c), 2, None, seed=15)
    D = q.shape[2]
    Wc = (0.7 * np.eye(D)).astype(np.float32)
    rng = np.random.default_rng(194)
    pro = dict(q_gamma=rng.random(D).astype(np.float32) + 0.5,
               k_gamma=rng.random(D).astype(np.float32) + 0.5, eps=1e-6, theta=100.0)
    a = run(c, q, k, v, g, Wc, 4, 2, prologue=pro)
    b = run(c + np.array([8, 16, 24], np.int32), q, k, v, g, Wc, 4, 2, prologue=pro)
    assert np.array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-11)
    # and the prologue changes the result (it is not silently skipped)
    plain = run(c, q, k, v, g, Wc, 4, 2)
    assert np.abs(plain["out"] - a["out"]).max() > 1e-2


def test_prologue_normalises_and_scales_before_rotating():
    # the rotation keeps the length of every channel pair, so each pair of the result has the
    # length of the pair after normalisation and weighting (weighting after the rotation would
    # not keep it, since the weights differ inside a pair)
    N, H, D = 30, 2, 96
    x = _rand((N, H, D), 195)
    pos = np.random.default_rng(196).integers(0, 200, (N, 3)).astype(np.int32)
    gamma = np.random.default_rng(197).random(D).astype(np.float32) * 2 + 0.1
    u = oracle.qk_prologue(x, pos, gamma, eps=0.0)
    rms = np.sqrt((x ** 2).mean(axis=2, keepdims=True))
    y = x / rms * gamma.astype(np.float64)
    pair = lambda a: np.sqrt(a[..., 0::2] ** 2 + a[..., 1::2] ** 2)
    np.testing.assert_allclose(pair(u), pair(y), rtol=1e-12)
    assert np.abs(u - y).max() > 1e-1   # and it does rotate


def test_prologue_results_rounded_to_the_input_type():
    # rounding the prologue's fp64 results to f16 equals numpy's f16 conversion of them
    N, H, D = 50, 2, 64
    x = _rand((N, H, D), 198).astype(np.float16)
    pos = np.random.default_rng(199).integers(0, 100, (N, 3)).astype(np.int32)
    g = np.random.default_rng(200).random(D).astype(np.float32) + 0.5
    exact = oracle.qk_prologue(x, pos, g)
    rounded = oracle.qk_prologue(x, pos, g, round_to_input=True)
    np.testing.assert_array_equal(rounded, exact.astype(np.float16).astype(np.float64))


# ---------------------------------------------------------------------------------------------
# compression by sparse 3D convolution over the block grid; gates predicted from the queries
# ---------------------------------------------------------------------------------------------

def _conv_weights(D, seed, scale=None):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((27, D, D)) / np.sqrt(27 * D) if scale is None
            else rng.standard_normal((27, D, D)) * scale).astype(np.float32)


def test_conv_compression_with_only_the_centre_tap_is_mean_times_wc():
    c, q, k, v, Wc = _tiny_inputs(seed=210)
    Kc, Vc = oracle.compress(c, k, v, Wc)
    Kc2, Vc2 = oracle.compress_conv(c, k, v, oracle.center_only_conv(Wc))
    np.testing.assert_allclose(Kc2, Kc, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Vc2, Vc, rtol=0, atol=1e-13)


def test_conv_compression_matches_brute_force_over_block_neighbours():
    # written out with dictionaries: the block means, then for every block the sum over the 27
    # offsets of the neighbour's mean times that offset's matrix (absent neighbours skipped)
    c, _ = _tiny_coords()
    c = c[:500]
    N, H, D = len(c), 2, 8
    k, v = _rand((N, H, D), 211), _rand((N, H, D), 212)
    W = _conv_weights(D, 213)
    members = {}
    for i, x in enumerate(c):
        members.setdefault(tuple(int(t) // 8 for t in x), []).append(i)
    blocks = sorted(members)
    mk = {b: k[members[b]].mean(axis=0) for b in blocks}
    mv = {b: v[members[b]].mean(axis=0) for b in blocks}
    Kc, Vc = oracle.compress_conv(c, k, v, W)
    for bi, b in enumerate(blocks):
        ek = np.zeros((H, D))
        ev = np.zeros((H, D))
        for dx in (-1, 0, 1):
            for dy in (-1, 0, 1):
                for dz in (-1, 0, 1):
                    nb = (b[0] + dx, b[1] + dy, b[2] + dz)
                    if nb not in mk:
                        continue
                    Wo = W[9 * (dx + 1) + 3 * (dy + 1) + (dz + 1)].astype(np.float64)
                    ek += mk[nb] @ Wo
                    ev += mv[nb] @ Wo
        np.testing.assert_allclose(Kc[bi], ek, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Vc[bi], ev, rtol=0, atol=1e-12)


def test_conv_compression_is_linear_in_the_kernel():
    c, q, k, v, _ = _tiny_inputs(seed=214, D=16)
    W1, W2 = _conv_weights(16, 215), _conv_weights(16, 216)
    W1[13:] = 0.0   # disjoint taps: the fp32 sum W1 + W2 is exact
    W2[:13] = 0.0
    a = oracle.compress_conv(c, k, v, W1)
    b = oracle.compress_conv(c, k, v, W2)
    ab = oracle.compress_conv(c, k, v, W1 + W2)
    for x, y, z in zip(a, b, ab):
        np.testing.assert_allclose(z, x + y, rtol=0, atol=1e-12)


def test_forward_with_centre_tap_and_explicit_gates_is_the_plain_forward():
    c, q, k, v, Wc = _tiny_inputs(seed=217)
    g = _gates(len(c), 2, None, seed=16)
    plain = run(c, q, k, v, g, Wc, 4, 2)
    conv = run(c, q, k, v, g, Wc, 4, 2, conv=oracle.center_only_conv(Wc))
    assert np.array_equal(plain["sel"], conv["sel"])
    for name in ("out", "o_cmp", "o_sel", "o_win"):
        np.testing.assert_allclose(conv[name], plain[name], rtol=0, atol=1e-12)


def test_predicted_gates():
    c, q, k, v, Wc = _tiny_inputs(seed=218)
    N, H, D = q.shape
    W = _conv_weights(D, 219)
    # a constant predictor (zero weights, bias logit(g)) is the constant gates g
    gc = np.array([0.2, 0.5, 0.9])
    const = run(c, q, k, v, None, Wc, 4, 2, conv=W,
                gate=dict(w=np.zeros((D, 3), np.float32), b=np.log(gc / (1 - gc)).astype(np.float32)))
    explicit = run(c, q, k, v, np.broadcast_to(gc.astype(np.float32), (N, H, 3)).copy(), Wc, 4, 2,
                   conv=W)
    np.testing.assert_allclose(const["out"], explicit["out"], rtol=0, atol=1e-6)
    # a query-dependent predictor equals explicit gates holding sigmoid(q . Wg + bg) per head
    rng = np.random.default_rng(220)
    Wg = (rng.standard_normal((D, 3)) / np.sqrt(D)).astype(np.float32)
    bg = rng.standard_normal(3).astype(np.float32)
    pred = run(c, q, k, v, None, Wc, 4, 2, conv=W, gate=dict(w=Wg, b=bg))
    logits = np.einsum("nhd,dc->nhc", q, Wg.astype(np.float64)) + bg.astype(np.float64)
    gates = (1.0 / (1.0 + np.exp(-logits))).astype(np.float32)
    ref = run(c, q, k, v, gates, Wc, 4, 2, conv=W)
    np.testing.assert_allclose(pred["out"], ref["out"], rtol=0, atol=2e-7)   # gates rounded to f32
    # the convolution changes the result (it is not silently the centre tap)
    plain = run(c, q, k, v, gates, Wc, 4, 2)
    assert np.abs(plain["out"] - ref["out"]).max() > 1e-2


def test_conv_forward_is_invariant_under_block_translation():
    c, q, k, v, Wc = _tiny_inputs(seed=221)
    g = _gates(len(c), 2, None, seed=17)
    W = _conv_weights(q.shape[2], 222)
    a = run(c, q, k, v, g, Wc, 4, 2, conv=W)
    b = run(c + np.array([16, 8, 24], np.int32), q, k, v, g, Wc, 4, 2, conv=W)
    assert np.array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# selection shared by the queries of a 4x4x4 sub-block (the pages leave open whose compression
# scores choose the blocks; this variant sums them over a sub-block's queries)
# ---------------------------------------------------------------------------------------------

def test_subblock_selection_with_one_query_per_subblock_is_the_per_query_selection():
    """Cells on a lattice of spacing 4: every 4x4x4 sub-block holds one query, and the sum of
    its weights ranks blocks as that query's logits do (softmax is increasing)."""
    rng = np.random.default_rng(21)
    lat = np.stack(np.meshgrid(*(np.arange(0, 48, 4),) * 3, indexing="ij"), -1).reshape(-1, 3)
    c = lat[np.sort(rng.choice(len(lat), 700, replace=False))].astype(np.int32)
    N, H, D = len(c), 2, 16
    q, k, v = (_rand((N, H, D), 22 + i) for i in range(3))
    g = _gates(N, H, None, 25)
    Wc = _rand((D, D), 26) / np.sqrt(D)
    a = run(c, q, k, v, g, Wc, 5, 2)
    b = run(c, q, k, v, g, Wc, 5, 2, share="subblock")
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-13)


def test_subblock_selection_matches_brute_force_on_tiny_input():
    """numpy restatement: blocks by np.unique of the 8-cell keys, Kc = block mean . Wc, each
    query's softmax, sums per (block, 4-cell sub-block) by np.add.at, ranking by lexsort."""
    c, _ = _tiny_coords()
    N, H, D, topk = len(c), 2, 8, 4
    q, k, v = (_rand((N, H, D), 31 + i) for i in range(3))
    Wc = (_rand((D, D), 34) / np.sqrt(D)).astype(np.float32)   # the oracle takes Wc in fp32
    ours = oracle.select_subblock(c, [0, N], q, k, v, Wc, topk, want_score=True)
    ukeys, tok_blk = np.unique(c // 8, axis=0, return_inverse=True)
    tok_blk = tok_blk.reshape(-1)
    mb = len(ukeys)
    cnt = np.bincount(tok_blk, minlength=mb)
    sub = ((c[:, 0] >> 2) & 1) * 4 + ((c[:, 1] >> 2) & 1) * 2 + ((c[:, 2] >> 2) & 1)
    grp = tok_blk * 8 + sub
    for h in range(H):
        kbar = np.zeros((mb, D))
        np.add.at(kbar, tok_blk, k[:, h])
        kc = (kbar / cnt[:, None]) @ Wc.astype(np.float64)
        z = q[:, h] @ kc.T / np.sqrt(D)
        p = np.exp(z - z.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        score = np.zeros((mb * 8, mb))
        np.add.at(score, grp, p)
        for i in range(N):
            s = score[grp[i]]
            np.testing.assert_allclose(ours["score"][i][h], s, rtol=1e-12, atol=1e-15)
            own = tok_blk[i]
            order = [b for b in np.lexsort((np.arange(mb), -s)) if b != own][:topk - 1]
            want = [own] + order + [-1] * (topk - 1 - len(order))
            assert list(ours["sel"][i, h]) == want, (i, h)


def test_subblock_selection_sums_weights_over_the_subblock():
    """Planted: three queries of one sub-block each rank another block first (A or C), but B is a
    close second for all three, so the summed weights pick B for every one of them; a query of a
    neighbouring sub-block of the same block keeps its own choice. Per-query selection differs."""
    D = 4
    c = np.array([[0, 0, 0], [1, 0, 0], [2, 0, 0], [5, 0, 0],    # own block (0,0,0)
                  [8, 0, 0], [16, 0, 0], [24, 0, 0]], np.int32)   # blocks A, B, C: one cell each
    alpha = 4.0
    k = np.zeros((7, 1, D))
    k[4, 0, 0] = k[5, 0, 1] = k[6, 0, 2] = alpha                 # Kc_A, Kc_B, Kc_C with Wc = I
    want_z = np.array([[5.0, 4.9, 0.0], [0.0, 4.0, 4.1], [0.0, 4.0, 4.1], [6.0, 0.0, 0.0]])
    q = np.zeros((7, 1, D))
    q[:4, 0, :3] = want_z * np.sqrt(D) / alpha                    # z_b = q . Kc_b / sqrt(D)
    v = _rand((7, 1, D), 40)
    g = _gates(7, 1, [0.0, 1.0, 0.0])
    Wc = np.eye(D)
    shared = run(c, q, k, v, g, Wc, 2, 1, share="subblock", rows=np.arange(4))
    alone = run(c, q, k, v, g, Wc, 2, 1, rows=np.arange(4))
    assert shared["sel"][:, 0].tolist() == [[0, 2], [0, 2], [0, 2], [0, 1]]
    assert alone["sel"][:, 0].tolist() == [[0, 1], [0, 3], [0, 3], [0, 1]]


def test_subblock_selection_is_shared_by_all_queries_of_a_subblock():
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    q, k, v = (_rand((N, H, D), 51 + i) for i in range(3))
    Wc = _rand((D, D), 54) / np.sqrt(D)
    sel = oracle.select_subblock(c, [0, N], q, k, v, Wc, 4)["sel"]
    key = np.concatenate([c // 4, np.zeros((N, 1), np.int32)], 1)
    _, grp = np.unique(key, axis=0, return_inverse=True)
    grp = grp.reshape(-1)
    for gi in np.unique(grp):
        m = np.nonzero(grp == gi)[0]
        assert (sel[m] == sel[m[0]]).all()
    assert len(np.unique(grp)) < N   # the tiny shell has sub-blocks with several cells


def test_subblock_selection_with_the_centre_tap_is_the_plain_one():
    """Convolution compression with only the centre tap (W_0 = Wc) gives the plain compressed
    tokens, hence the same shared selection and summed weights."""
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    q, k, v = (_rand((N, H, D), 61 + i) for i in range(3))
    Wc = (_rand((D, D), 64) / np.sqrt(D)).astype(np.float32)
    a = oracle.select_subblock(c, [0, N], q, k, v, Wc, 4, want_score=True)
    b = oracle.select_subblock(c, [0, N], q, k, v, Wc, 4, conv=oracle.center_only_conv(Wc), want_score=True)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    for x, y in zip(a["score"], b["score"]):
        np.testing.assert_allclose(y, x, rtol=1e-12, atol=1e-15)


def test_subblock_selection_is_invariant_under_block_translation():
    """Moving every cell by whole 8-cell blocks moves every 4-cell sub-block with its block: the
    same tokens share a selection, with the same blocks (block indices keep their order)."""
    c, _ = _tiny_coords()
    N, H, D = len(c), 2, 8
    q, k, v = (_rand((N, H, D), 71 + i) for i in range(3))
    Wc = (_rand((D, D), 74) / np.sqrt(D)).astype(np.float32)
    a = oracle.select_subblock(c, [0, N], q, k, v, Wc, 4)["sel"]
    b = oracle.select_subblock(c + np.array([8, 24, 16], np.int32), [0, N], q, k, v, Wc, 4)["sel"]
    np.testing.assert_array_equal(a, b)

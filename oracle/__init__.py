"""fp64 CPU oracle for Spatial Sparse Attention (SSA).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path. It shares no code with
the CUDA library. The arithmetic lives in ssa_oracle.c (plain C, fp64, OpenMP
over rows); this module only marshals arrays, walks packed sequences and maps
per-sequence block indices to global ones.

Every function follows the formulation written at the top of ssa_oracle.c
(Direct3D-S2 summary page, "Technical principles", SSA item; Direct3D-S2 model
page, "What is Direct3D-S2?").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssa_oracle.c")
_LIB = os.path.join(_HERE, "libssa_oracle.so")

F32, BF16, F16, F64 = 0, 1, 2, 3
_lib = None

c_i32p = ctypes.POINTER(ctypes.c_int32)
c_i64p = ctypes.POINTER(ctypes.c_int64)
c_f32p = ctypes.POINTER(ctypes.c_float)
c_f64p = ctypes.POINTER(ctypes.c_double)
c_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile ssa_oracle.c into libssa_oracle.so (gcc, -O2, OpenMP). Returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.oracle_decode_f16.restype = ctypes.c_double
        L.oracle_decode_f16.argtypes = [ctypes.c_uint16]
        L.oracle_decode_bf16.restype = ctypes.c_double
        L.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_round_to.restype = ctypes.c_double
        L.oracle_round_to.argtypes = [ctypes.c_double, ctypes.c_int]
        L.oracle_partition.restype = ctypes.c_int64
        L.oracle_partition.argtypes = [ctypes.c_int64, c_i32p, ctypes.c_int32, c_i32p, c_i32p,
                                       c_i32p, c_i32p]
        for f in (L.oracle_window, L.oracle_window_brute):
            f.restype = ctypes.c_int64
            f.argtypes = [ctypes.c_int64, c_i32p, ctypes.c_int32, c_i64p, c_i32p]
        L.oracle_compress.restype = ctypes.c_int
        L.oracle_compress.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, c_vp, c_vp, c_f32p, c_i32p, c_i32p,
                                      ctypes.c_int32, c_f64p, c_f64p]
        L.oracle_forward.restype = ctypes.c_int
        L.oracle_forward.argtypes = [
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_vp, c_vp, c_vp,
            c_f32p, c_f32p, ctypes.c_int32, ctypes.c_int32, c_i32p, c_i32p, c_i32p,
            ctypes.c_int64, c_i64p, c_i32p, ctypes.c_int64, c_i64p, c_i32p,
            c_f64p, c_f64p, c_f64p, c_f64p, c_i32p, c_f64p]
        L.oracle_backward.restype = ctypes.c_int
        L.oracle_backward.argtypes = [
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_vp, c_vp, c_vp,
            c_f32p, c_f32p, c_vp, ctypes.c_int32, ctypes.c_int32, c_i32p, c_i32p, c_i32p,
            ctypes.c_int64, c_i64p, c_i32p, c_i32p, c_f64p, c_f64p, c_f64p]
        L.oracle_backward_dq_rows.restype = ctypes.c_int
        L.oracle_backward_dq_rows.argtypes = [
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_vp, c_vp, c_vp,
            c_f32p, c_f32p, c_vp, ctypes.c_int32, ctypes.c_int32, c_i32p, c_i32p, c_i32p,
            ctypes.c_int64, c_i64p, c_i32p, ctypes.c_int64, c_i64p, c_i32p, c_f64p, c_i32p]
        L.oracle_forward_variant.restype = ctypes.c_int
        L.oracle_forward_variant.argtypes = [
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_vp, c_vp, c_vp,
            c_f32p, c_f32p, c_i32p, c_f32p, c_f32p, ctypes.c_int32, c_i32p, c_i32p, c_i32p,
            ctypes.c_int64, c_i64p, c_i32p, ctypes.c_int64, c_i64p, c_i32p,
            c_f64p, c_f64p, c_f64p, c_f64p, c_i32p, c_f64p]
        L.oracle_compress_conv.restype = ctypes.c_int
        L.oracle_compress_conv.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, c_vp, c_vp, c_f32p, c_i32p, c_i32p,
                                           c_i32p, c_f64p, c_f64p]
        L.oracle_select_subblock.restype = ctypes.c_int
        L.oracle_select_subblock.argtypes = [
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, c_vp, c_vp, c_vp,
            c_f32p, c_f32p, c_i32p, ctypes.c_int32, c_i32p, c_i32p, c_i32p, c_i32p,
            ctypes.c_int64, ctypes.c_int64, c_i64p, c_i32p, c_f64p]
        L.oracle_rope_split.restype = None
        L.oracle_rope_split.argtypes = [ctypes.c_int32, c_i32p, c_i32p, c_i32p]
        L.oracle_round_array.restype = None
        L.oracle_round_array.argtypes = [c_f64p, ctypes.c_int64, ctypes.c_int32]
        L.oracle_qk_prologue.restype = ctypes.c_int
        L.oracle_qk_prologue.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, c_vp, c_i32p, c_f32p, ctypes.c_double,
                                         ctypes.c_double, c_f64p]
    return _lib


# ----------------------------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------------------------

def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctype)


def _raw(t):
    """(contiguous numpy view of the storage bits, dtype code) of a CPU tensor or array."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.float64:
                return t.numpy(), F64
            if t.dtype == torch.float32:
                return t.numpy(), F32
            if t.dtype == torch.float16:
                return t.numpy(), F16
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy(), BF16
            raise TypeError(t.dtype)
    except ImportError:
        pass
    a = np.ascontiguousarray(t)
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.float16:
        return a, F16
    raise TypeError(a.dtype)


def _f32(t) -> np.ndarray:
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return np.ascontiguousarray(t.detach().cpu().float().numpy())
    except ImportError:
        pass
    return np.ascontiguousarray(t, dtype=np.float32)


def decode(bits: np.ndarray, dtype: int) -> np.ndarray:
    L = lib()
    f = L.oracle_decode_f16 if dtype == F16 else L.oracle_decode_bf16
    return np.array([f(int(b)) for b in np.asarray(bits, dtype=np.uint16).ravel()])


def round_to(x: np.ndarray, dtype: int) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_round_to(float(v), dtype) for v in np.asarray(x).ravel()])


# ----------------------------------------------------------------------------------------------
# plan: partition + window lists
# ----------------------------------------------------------------------------------------------

def partition(coords: np.ndarray, block: int = 8):
    """One sequence. Returns perm, tok_blk, blk_off, blk_coord (local indices)."""
    c = np.ascontiguousarray(coords, dtype=np.int32)
    n = len(c)
    perm = np.empty(n, np.int32)
    tok_blk = np.empty(n, np.int32)
    blk_off = np.empty(n + 1, np.int32)
    blk_coord = np.empty((max(n, 1), 3), np.int32)
    mb = lib().oracle_partition(n, _ptr(c, c_i32p), block, _ptr(perm, c_i32p),
                                _ptr(tok_blk, c_i32p), _ptr(blk_off, c_i32p),
                                _ptr(blk_coord, c_i32p))
    if mb < 0:
        raise ValueError("oracle_partition failed")
    return perm, tok_blk, blk_off[:mb + 1].copy(), blk_coord[:mb].copy()


def window(coords: np.ndarray, r: int, brute: bool = False):
    """One sequence. Returns (nbr_off int64 [n+1], nbr_idx int32 [nnz]), rows ascending."""
    c = np.ascontiguousarray(coords, dtype=np.int32)
    n = len(c)
    f = lib().oracle_window_brute if brute else lib().oracle_window
    off = np.zeros(n + 1, np.int64)
    nnz = f(n, _ptr(c, c_i32p), r, _ptr(off, c_i64p), None)
    if nnz == -2:
        raise ValueError("duplicate coordinate")
    if nnz < 0:
        raise ValueError("oracle_window failed")
    idx = np.empty(max(nnz, 1), np.int32)
    f(n, _ptr(c, c_i32p), r, _ptr(off, c_i64p), _ptr(idx, c_i32p))
    return off, idx[:nnz]


def plan(coords: np.ndarray, cu_seqlens, block: int = 8, r: int = 2) -> Dict[str, np.ndarray]:
    """Partition and window lists of a packed batch, with global token and block indices."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    perms, toks, offs, bcs, bseq, nos, nis = [], [], [], [], [], [], []
    blk_base = np.zeros(len(cu), np.int64)
    nnz_base = 0
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        perm, tok_blk, blk_off, blk_coord = partition(coords[lo:hi], block)
        mb = len(blk_coord)
        perms.append(perm.astype(np.int64) + lo)
        toks.append(tok_blk.astype(np.int64) + blk_base[s])
        offs.append(blk_off[:-1].astype(np.int64) + lo)
        bcs.append(blk_coord)
        bseq.append(np.full(mb, s, np.int32))
        blk_base[s + 1] = blk_base[s] + mb
        no, ni = window(coords[lo:hi], r)
        nos.append(no[:-1] + nnz_base)
        nis.append(ni.astype(np.int64) + lo)
        nnz_base += int(no[-1])
    mb_total = int(blk_base[-1])
    return dict(
        perm=np.concatenate(perms).astype(np.int32) if perms else np.zeros(0, np.int32),
        tok_blk=np.concatenate(toks).astype(np.int32),
        blk_off=np.concatenate(offs + [np.array([cu[-1]])]).astype(np.int32),
        blk_coord=np.concatenate(bcs).astype(np.int32).reshape(mb_total, 3),
        blk_seq=np.concatenate(bseq).astype(np.int32),
        blk_base=blk_base,
        nbr_off=np.concatenate(nos + [np.array([nnz_base])]).astype(np.int64),
        nbr_idx=np.concatenate(nis).astype(np.int32),
    )


# ----------------------------------------------------------------------------------------------
# forward / backward
# ----------------------------------------------------------------------------------------------

def _seq_plan(coords, lo, hi, block, r):
    perm, tok_blk, blk_off, blk_coord = partition(coords[lo:hi], block)
    no, ni = window(coords[lo:hi], r)
    return perm, tok_blk, blk_off, len(blk_coord), no, ni


def rope_split(D: int):
    """Widths of the x, y and z parts of the head dimension in the 3D rotary embedding."""
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    lib().oracle_rope_split(D, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return a.value, b.value, c.value


def qk_prologue(X, coords, gamma, eps: float = 1e-6, theta: float = 10000.0,
                round_to_input: bool = False) -> np.ndarray:
    """RMS normalisation over the head dimension (weight gamma [D]) followed by the 3D rotary
    embedding at the tokens' voxel coordinates; X [N, H, D] -> float64 [N, H, D]. With
    round_to_input, the results are rounded to X's storage type (what the method then sees)."""
    x, dt = _raw(X)
    N, H, D = x.shape
    c = np.ascontiguousarray(coords, dtype=np.int32)
    g = _f32(gamma)
    out = np.zeros((N, H, D))
    if lib().oracle_qk_prologue(N, H, D, dt, x.ctypes.data, _ptr(c, c_i32p), _ptr(g, c_f32p),
                                float(eps), float(theta), _ptr(out, c_f64p)) != 0:
        raise ValueError("oracle_qk_prologue failed")
    if round_to_input and dt != F64:
        lib().oracle_round_array(_ptr(out, c_f64p), out.size, dt)
    return out


def _exact_f64(t) -> np.ndarray:
    """Storage values of a CPU tensor or array as float64 (every f32/f16/bf16 value is exact)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().cpu().double().numpy()
    except ImportError:
        pass
    return np.asarray(t, dtype=np.float64)


def center_only_conv(Wc) -> np.ndarray:
    """The convolution kernel [27, D, D] whose only nonzero tap is the centre one, Wc: the
    convolution compression then equals the block mean times Wc."""
    w = _f32(Wc)
    D = w.shape[0]
    W = np.zeros((27, D, D), np.float32)
    W[13] = w
    return W


def forward(coords, cu_seqlens, Q, K, V, gates, Wc, topk: int, r: int, rows=None,
            block: int = 8, round_compressed: bool = False, sel_in=None,
            want_z: bool = False, branches: bool = True, prologue=None, conv=None,
            gate=None, share=None) -> Dict[str, object]:
    """Oracle forward for the query rows `rows` (global indices; None = all tokens).

    Returns out, o_cmp, o_sel, o_win ([R, H, D] float64), sel ([R, H, k] int32 global block
    indices, -1 = empty slot) and, if want_z, z: list of [H, Mb_seq] scaled compressed logits.
    sel_in ([R, H, k] global block indices) replaces the selection of the rows. With
    branches=False only the compressed attention and the selection run: the result has o_cmp
    and sel, and out / o_sel / o_win are left at zero. prologue = dict(q_gamma, k_gamma, eps,
    theta) first replaces Q and K by qk_prologue(Q), qk_prologue(K), rounded to their input type
    (the prologue's results are tensors of that type, as any layer's are). conv ([27, D, D]
    fp32) compresses blocks by the sparse 3D convolution over the block grid instead of the
    block mean times Wc; gate = dict(w=[D, 3], b=[3]) predicts the gates from each head's query
    (sigmoid(q . w + b)) instead of reading `gates`. share="subblock" selects the blocks once per
    4x4x4 sub-block of cells from the summed compressed-attention weights of its queries
    (select_subblock) instead of once per query.
    """
    if share not in (None, "subblock"):
        raise ValueError(f"unknown selection sharing {share!r}")
    if prologue is not None:
        pr = dict(prologue)
        kw = dict(eps=pr.get("eps", 1e-6), theta=pr.get("theta", 10000.0), round_to_input=True)
        Q = qk_prologue(Q, coords, pr["q_gamma"], **kw)
        K = qk_prologue(K, coords, pr["k_gamma"], **kw)
        V = _exact_f64(V)
        return forward(coords, cu_seqlens, Q, K, V, gates, Wc, topk, r, rows=rows, block=block,
                       round_compressed=round_compressed, sel_in=sel_in, want_z=want_z,
                       branches=branches, conv=conv, gate=gate, share=share)
    if share == "subblock" and sel_in is None:
        sh = select_subblock(coords, cu_seqlens, Q, K, V, Wc, topk, rows=rows, block=block, conv=conv)
        return forward(coords, cu_seqlens, Q, K, V, gates, Wc, topk, r, rows=rows, block=block,
                       round_compressed=round_compressed, sel_in=sh["sel"], want_z=want_z,
                       branches=branches, conv=conv, gate=gate)
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    q, dt = _raw(Q)
    k, _ = _raw(K)
    v, _ = _raw(V)
    g = _f32(gates)
    w = _f32(Wc)
    N, H, D = q.shape
    wconv = wg = bg = None
    if conv is not None or gate is not None:
        wconv = np.ascontiguousarray(_f32(conv) if conv is not None else center_only_conv(w),
                                     dtype=np.float32).reshape(27, D, D)
        if gate is not None:
            wg = np.ascontiguousarray(_f32(gate["w"]), dtype=np.float32).reshape(D, 3)
            bg = np.ascontiguousarray(_f32(gate["b"]), dtype=np.float32).reshape(3)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    R = len(rows)
    res = {name: np.zeros((R, H, D)) for name in ("out", "o_cmp", "o_sel", "o_win")}
    res["sel"] = np.full((R, H, topk), -1, np.int32)
    zs = [None] * R
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    blk_base = 0
    L = lib()
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        perm, tok_blk, blk_off, mb, no, ni = _seq_plan(coords, lo, hi, block, r)
        pick = np.nonzero(seq_of == s)[0]
        if len(pick):
            local = np.ascontiguousarray(rows[pick] - lo)
            n_r = len(local)
            outs = {name: np.zeros((n_r, H, D)) for name in ("out", "o_cmp", "o_sel", "o_win")}
            sel = np.zeros((n_r, H, topk), np.int32)
            zc = np.zeros((n_r, H, max(mb, 1))) if want_z else None
            sin = None
            if sel_in is not None:
                sin = np.ascontiguousarray(np.asarray(sel_in, dtype=np.int64)[pick], dtype=np.int64)
                sin = np.where(sin >= 0, sin - blk_base, -1).astype(np.int32)
            outs_args = (
                n_r, _ptr(local, c_i64p), _ptr(sin, c_i32p),
                _ptr(outs["out"] if branches else None, c_f64p), _ptr(outs["o_cmp"], c_f64p),
                _ptr(outs["o_sel"] if branches else None, c_f64p),
                _ptr(outs["o_win"] if branches else None, c_f64p),
                _ptr(sel, c_i32p), _ptr(zc, c_f64p))
            if conv is not None or gate is not None:
                bc = np.ascontiguousarray(partition(coords[lo:hi], block)[3], dtype=np.int32)
                rc = L.oracle_forward_variant(
                    hi - lo, H, D, dt,
                    q[lo:hi].ctypes.data, k[lo:hi].ctypes.data, v[lo:hi].ctypes.data,
                    _ptr(np.ascontiguousarray(g[lo:hi]), c_f32p), _ptr(wconv, c_f32p),
                    _ptr(bc, c_i32p), _ptr(wg, c_f32p), _ptr(bg, c_f32p), topk,
                    _ptr(perm, c_i32p), _ptr(tok_blk, c_i32p), _ptr(blk_off, c_i32p), mb,
                    _ptr(no, c_i64p), _ptr(ni, c_i32p), *outs_args)
                if rc != 0:
                    raise RuntimeError("oracle_forward_variant failed")
                for name in outs:
                    res[name][pick] = outs[name]
                res["sel"][pick] = np.where(sel >= 0, sel + blk_base, -1)
                if want_z:
                    for t_, p_ in enumerate(pick):
                        zs[p_] = zc[t_, :, :mb].copy()
                blk_base += mb
                continue
            rc = L.oracle_forward(
                hi - lo, H, D, dt,
                q[lo:hi].ctypes.data, k[lo:hi].ctypes.data, v[lo:hi].ctypes.data,
                _ptr(np.ascontiguousarray(g[lo:hi]), c_f32p), _ptr(w, c_f32p), topk,
                int(round_compressed), _ptr(perm, c_i32p), _ptr(tok_blk, c_i32p),
                _ptr(blk_off, c_i32p), mb, _ptr(no, c_i64p), _ptr(ni, c_i32p),
                n_r, _ptr(local, c_i64p), _ptr(sin, c_i32p),
                _ptr(outs["out"] if branches else None, c_f64p), _ptr(outs["o_cmp"], c_f64p),
                _ptr(outs["o_sel"] if branches else None, c_f64p),
                _ptr(outs["o_win"] if branches else None, c_f64p),
                _ptr(sel, c_i32p), _ptr(zc, c_f64p))
            if rc != 0:
                raise RuntimeError("oracle_forward failed")
            for name in outs:
                res[name][pick] = outs[name]
            res["sel"][pick] = np.where(sel >= 0, sel + blk_base, -1)
            if want_z:
                for t, p in enumerate(pick):
                    zs[p] = zc[t, :, :mb].copy()
        blk_base += mb
    if want_z:
        res["z"] = zs
    res["rows"] = rows
    return res


def select_subblock(coords, cu_seqlens, Q, K, V, Wc, topk: int, rows=None, block: int = 8,
                    conv=None, want_score: bool = False) -> Dict[str, object]:
    """Selection shared by the queries of each 4x4x4 sub-block of cells (oracle_select_subblock):
    the own block plus the top (k-1) other blocks by the sum over the sub-block's queries of
    their compressed-attention weights. Q and K are taken as given (apply qk_prologue first for
    the prologue). Returns sel ([R, H, k] global block indices, -1 = empty slot) for the rows
    (global indices; None = all tokens) and, if want_score, score: list of [H, Mb_seq] summed
    weights of each row's sub-block."""
    if block != 8:
        raise ValueError("sub-blocks of 4 cells are defined for blocks of 8 cells")
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    q, dt = _raw(Q)
    k, dk = _raw(K)
    v, dv = _raw(V)
    if dk != dt or dv != dt:
        raise ValueError("Q, K and V must have one storage type")
    w = _f32(Wc)
    N, H, D = q.shape
    wconv = None
    if conv is not None:
        wconv = np.ascontiguousarray(_f32(conv), dtype=np.float32).reshape(27, D, D)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    R = len(rows)
    out_sel = np.full((R, H, topk), -1, np.int32)
    scores = [None] * R
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    blk_base = 0
    L = lib()
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        perm, tok_blk, blk_off, blk_coord = partition(coords[lo:hi], block)
        mb = len(blk_off) - 1
        pick = np.nonzero(seq_of == s)[0]
        if len(pick) and mb > 0:
            local = np.ascontiguousarray(rows[pick] - lo)
            sel = np.zeros((len(pick), H, topk), np.int32)
            sc = np.zeros((len(pick), H, mb)) if want_score else None
            rc = L.oracle_select_subblock(
                hi - lo, H, D, dt, q[lo:hi].ctypes.data, k[lo:hi].ctypes.data, v[lo:hi].ctypes.data,
                _ptr(w, c_f32p), _ptr(wconv, c_f32p),
                _ptr(np.ascontiguousarray(blk_coord, dtype=np.int32), c_i32p), topk,
                _ptr(np.ascontiguousarray(coords[lo:hi]), c_i32p), _ptr(perm, c_i32p),
                _ptr(tok_blk, c_i32p), _ptr(blk_off, c_i32p), mb, len(local), _ptr(local, c_i64p),
                _ptr(sel, c_i32p), _ptr(sc, c_f64p))
            if rc != 0:
                raise RuntimeError("oracle_select_subblock failed")
            out_sel[pick] = np.where(sel >= 0, sel + blk_base, -1)
            if want_score:
                for t, p in enumerate(pick):
                    scores[p] = sc[t].copy()
        blk_base += mb
    res = {"sel": out_sel, "rows": rows}
    if want_score:
        res["score"] = scores
    return res


def backward(coords, cu_seqlens, Q, K, V, gates, Wc, dO, topk: int, r: int, block: int = 8,
             round_compressed: bool = False, sel=None):
    """Full fp64 backward: (dQ, dK, dV) [N, H, D] of sum(dO * out), selection held fixed.

    sel ([N, H, k] global block indices, -1 = empty slot) is the selection to hold; None = the
    oracle's own."""
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    q, dt = _raw(Q)
    k, _ = _raw(K)
    v, _ = _raw(V)
    go, _ = _raw(dO)
    g = _f32(gates)
    w = _f32(Wc)
    N, H, D = q.shape
    dQ, dK, dV = (np.zeros((N, H, D)) for _ in range(3))
    L = lib()
    blk_base = 0
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        n = hi - lo
        perm, tok_blk, blk_off, mb, no, ni = _seq_plan(coords, lo, hi, block, r)
        gs = np.ascontiguousarray(g[lo:hi])
        if sel is not None:
            ss = np.asarray(sel, dtype=np.int64)[lo:hi]
            ssel = np.ascontiguousarray(np.where(ss >= 0, ss - blk_base, -1), dtype=np.int32)
        else:
            ssel = np.zeros((n, H, topk), np.int32)
            rc = L.oracle_forward(n, H, D, dt, q[lo:hi].ctypes.data, k[lo:hi].ctypes.data,
                                  v[lo:hi].ctypes.data, _ptr(gs, c_f32p), _ptr(w, c_f32p), topk,
                                  int(round_compressed), _ptr(perm, c_i32p), _ptr(tok_blk, c_i32p),
                                  _ptr(blk_off, c_i32p), mb, _ptr(no, c_i64p), _ptr(ni, c_i32p),
                                  n, None, None, None, None, None, None, _ptr(ssel, c_i32p), None)
            if rc != 0:
                raise RuntimeError("oracle_forward failed")
        blk_base += mb
        a, b, c = (np.zeros((n, H, D)) for _ in range(3))
        rc = L.oracle_backward(n, H, D, dt, q[lo:hi].ctypes.data, k[lo:hi].ctypes.data,
                               v[lo:hi].ctypes.data, _ptr(gs, c_f32p), _ptr(w, c_f32p),
                               go[lo:hi].ctypes.data, topk, int(round_compressed),
                               _ptr(perm, c_i32p), _ptr(tok_blk, c_i32p), _ptr(blk_off, c_i32p),
                               mb, _ptr(no, c_i64p), _ptr(ni, c_i32p), _ptr(ssel, c_i32p),
                               _ptr(a, c_f64p), _ptr(b, c_f64p), _ptr(c, c_f64p))
        if rc != 0:
            raise RuntimeError("oracle_backward failed")
        dQ[lo:hi], dK[lo:hi], dV[lo:hi] = a, b, c
    return dQ, dK, dV


def backward_dq_rows(coords, cu_seqlens, Q, K, V, gates, Wc, dO, topk: int, r: int, rows,
                     block: int = 8, round_compressed: bool = False, return_sel: bool = False,
                     sel_in=None):
    """dQ [R, H, D] for the given global rows, evaluated row by row (any size).

    sel_in ([R, H, k] global block indices) replaces the rows' selection. With return_sel, also
    returns the selection used ([R, H, k] global block indices)."""
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    q, dt = _raw(Q)
    k, _ = _raw(K)
    v, _ = _raw(V)
    go, _ = _raw(dO)
    g = _f32(gates)
    w = _f32(Wc)
    N, H, D = q.shape
    rows = np.asarray(rows, dtype=np.int64)
    dQ = np.zeros((len(rows), H, D))
    sel_all = np.full((len(rows), H, topk), -1, np.int32)
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    L = lib()
    blk_base = 0
    for s in range(len(cu) - 1):
        pick = np.nonzero(seq_of == s)[0]
        lo, hi = int(cu[s]), int(cu[s + 1])
        perm, tok_blk, blk_off, mb, no, ni = _seq_plan(coords, lo, hi, block, r)
        if not len(pick):
            blk_base += mb
            continue
        local = np.ascontiguousarray(rows[pick] - lo)
        out = np.zeros((len(local), H, D))
        sel = np.zeros((len(local), H, topk), np.int32)
        sin = None
        if sel_in is not None:
            si = np.asarray(sel_in, dtype=np.int64)[pick]
            sin = np.ascontiguousarray(np.where(si >= 0, si - blk_base, -1), dtype=np.int32)
        rc = L.oracle_backward_dq_rows(
            hi - lo, H, D, dt, q[lo:hi].ctypes.data, k[lo:hi].ctypes.data, v[lo:hi].ctypes.data,
            _ptr(np.ascontiguousarray(g[lo:hi]), c_f32p), _ptr(w, c_f32p), go[lo:hi].ctypes.data,
            topk, int(round_compressed), _ptr(perm, c_i32p), _ptr(tok_blk, c_i32p),
            _ptr(blk_off, c_i32p), mb, _ptr(no, c_i64p), _ptr(ni, c_i32p), len(local),
            _ptr(local, c_i64p), _ptr(sin, c_i32p), _ptr(out, c_f64p), _ptr(sel, c_i32p))
        if rc != 0:
            raise RuntimeError("oracle_backward_dq_rows failed")
        dQ[pick] = out
        sel_all[pick] = np.where(sel >= 0, sel + blk_base, -1)
        blk_base += mb
    return (dQ, sel_all) if return_sel else dQ


def compress_conv(coords, K, V, W, block: int = 8):
    """Compressed tokens (Kc, Vc) [Mb, H, D] of a single sequence by the sparse 3D convolution
    over the block grid (W [27, D, D])."""
    k, dt = _raw(K)
    v, _ = _raw(V)
    N, H, D = k.shape
    Wf = np.ascontiguousarray(_f32(W), dtype=np.float32).reshape(27, D, D)
    perm, tok_blk, blk_off, blk_coord = partition(coords, block)
    mb = len(blk_coord)
    Kc = np.zeros((mb, H, D))
    Vc = np.zeros((mb, H, D))
    bc = np.ascontiguousarray(blk_coord, dtype=np.int32)
    lib().oracle_compress_conv(mb, H, D, dt, k.ctypes.data, v.ctypes.data, _ptr(Wf, c_f32p),
                               _ptr(perm, c_i32p), _ptr(blk_off, c_i32p), _ptr(bc, c_i32p),
                               _ptr(Kc, c_f64p), _ptr(Vc, c_f64p))
    return Kc, Vc


def compress(coords, K, V, Wc, block: int = 8, round_compressed: bool = False):
    """Compressed tokens (Kc, Vc) [Mb, H, D] of a single sequence."""
    k, dt = _raw(K)
    v, _ = _raw(V)
    w = _f32(Wc)
    N, H, D = k.shape
    perm, tok_blk, blk_off, blk_coord = partition(coords, block)
    mb = len(blk_coord)
    Kc = np.zeros((mb, H, D))
    Vc = np.zeros((mb, H, D))
    lib().oracle_compress(mb, H, D, dt, k.ctypes.data, v.ctypes.data, _ptr(w, c_f32p),
                          _ptr(perm, c_i32p), _ptr(blk_off, c_i32p), int(round_compressed),
                          _ptr(Kc, c_f64p), _ptr(Vc, c_f64p))
    return Kc, Vc

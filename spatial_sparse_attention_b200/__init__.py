"""Python binding of libssa.so: Spatial Sparse Attention forward on B200 (sm_100a).

Argument marshalling only. Every step of the method runs in the library's CUDA kernels; PyTorch
provides device memory and the current stream. There is no CPU fallback: importing this package
without the built library raises.

    plan = ssa.Plan(coords, grid=(192, 192, 192), r=3)          # block partition, window lists
    out = plan.forward(q, k, v, gates, wc, topk=16)             # three branches, gated sum
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "ssa.h")

STATUS = {
    0: "SSA_OK", 1: "SSA_ERR_INVALID_ARG", 2: "SSA_ERR_COORD_RANGE", 3: "SSA_ERR_DUPLICATE_COORD",
    4: "SSA_ERR_ALLOC", 5: "SSA_ERR_CUDA", 6: "SSA_ERR_UNSUPPORTED", 7: "SSA_ERR_DEVICE_TIMEOUT",
}
_DTYPE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


class SSAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{where}: {self.name}")


_vp = ctypes.c_void_p
_i32, _i64 = ctypes.c_int32, ctypes.c_int64
_SIGS = {
    "ssa_set_allocator": [_vp, _vp, _vp],
    "ssa_block_offsets_noalloc": [_vp, _i64, _vp, _vp, _i64, _vp, _vp],
    "ssa_plan": [_vp, _i64, _vp, _i32, _i32, _vp, _vp],
    "ssa_plan_varlen": [_vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp],
    "ssa_plan_rebuild": [_vp, _vp, _vp],
    "ssa_plan_info": [_vp, _vp, _vp, _vp, _vp],
    "ssa_plan_export": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "ssa_forward": [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp],
    "ssa_forward_debug": [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                          _vp, _vp],
    "ssa_forward_host": [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp],
    "ssa_forward_prologue": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float,
                             _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "ssa_forward_ex": [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "ssa_backward": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "ssa_last_device_status": [_vp, _vp],
    "ssa_debug_wait_timeout": [_vp, _i64, _vp],
    "ssa_plan_destroy": [_vp],
    "ssa_status_string": [_i32],
    "ssa_launch_count": [],
    "ssa_profile_enable": [_i32],
    "ssa_profile_reset": [],
    "ssa_profile_read": [_i32, _vp, _vp, _vp],
}


class Options(ctypes.Structure):
    """ssa_options_t (include/ssa.h): the optional parts of ssa_forward_ex."""
    _fields_ = [("q_gamma", _vp), ("k_gamma", _vp), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("conv_w", _vp), ("gate_w", _vp), ("gate_b", _vp),
                ("select_share", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built (run spatial_sparse_attention_b200/build.py); "
                          "there is no CPU fallback")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in _SIGS.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.ssa_status_string.restype = ctypes.c_char_p
    lib.ssa_launch_count.restype = ctypes.c_int64
    return lib


lib = _load()


def declared_symbols() -> Sequence[str]:
    """Entry points declared in include/ssa.h."""
    return re.findall(r"SSA_API\s+[\w\s\*]+?\b(ssa_\w+)\s*\(", open(HEADER).read())


def block_offsets_noalloc(coords: torch.Tensor, grid, stream=None):
    """ssa_block_offsets_noalloc: CSR token offsets of the occupied 8^3 blocks of one sequence,
    computed in the library's fixed scratch (no device allocation by the library). Returns
    (blk_off [n_blocks + 1] int32 on the device, n_blocks); n_blocks is -1 if a coordinate lies
    outside the grid."""
    c = _dev(coords, torch.int32)
    n = c.shape[0]
    g = (ctypes.c_int32 * 3)(*[int(x) for x in grid])
    nb = 1
    for x in grid:
        nb *= (int(x) + 7) // 8
    cap = min(n, nb) + 1
    # the library finds its scratch array on the current device: make it the coordinates' device
    with torch.cuda.device(c.device):
        blk_off = torch.empty(cap, dtype=torch.int32, device=c.device)
        nblk = torch.empty(1, dtype=torch.int32, device=c.device)
        st = torch.cuda.current_stream() if stream is None else stream
        _check(lib.ssa_block_offsets_noalloc(c.data_ptr(), n, g, blk_off.data_ptr(), cap,
                                             nblk.data_ptr(), st.cuda_stream),
               "ssa_block_offsets_noalloc")
        st.synchronize()   # the count is read on the host: wait for the stream the work went to
        k = int(nblk.item())
    return (blk_off[:k + 1] if k >= 0 else blk_off[:0]), k


def launch_count() -> int:
    return int(lib.ssa_launch_count())


def profile_enable(on: bool = True):
    lib.ssa_profile_enable(1 if on else 0)


def profile_reset():
    lib.ssa_profile_reset()


def profile_read():
    """{kernel name: (total ms, launches)} of the CUDA-event timings recorded so far."""
    n = 32
    names = ctypes.create_string_buffer(64 * n)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    k = lib.ssa_profile_read(n, names, ms, cnt)
    return {names.raw[64 * i:64 * (i + 1)].split(b"\0")[0].decode(): (ms[i], cnt[i])
            for i in range(k)}


def _check(code: int, where: str):
    if code != 0:
        raise SSAError(code, where)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype=None) -> torch.Tensor:
    if not t.is_cuda or not t.is_contiguous() or (dtype is not None and t.dtype != dtype):
        raise ValueError("expected a contiguous CUDA tensor" + (f" of {dtype}" if dtype else ""))
    return t


class Plan:
    """Block partition and window lists of a packed batch of voxel token sequences.

    coords: int32 CUDA tensor [N, 3]. Either `grid` (one sequence) or `cu_seqlens` + `grids`.
    """

    def __init__(self, coords: torch.Tensor, grid=None, r: int = 2, block: int = 8,
                 cu_seqlens: Optional[Sequence[int]] = None, grids=None, stream=None):
        _dev(coords, torch.int32)
        self._h = _vp()
        self.stream = stream
        st = _stream(stream)
        if cu_seqlens is None:
            g = (ctypes.c_int32 * 3)(*[int(x) for x in grid])
            _check(lib.ssa_plan(coords.data_ptr(), coords.shape[0], ctypes.addressof(g), block, r,
                                st, ctypes.byref(self._h)), "ssa_plan")
        else:
            B = len(cu_seqlens) - 1
            cu = (ctypes.c_int64 * (B + 1))(*[int(x) for x in cu_seqlens])
            flat = [int(x) for row in grids for x in row]
            gr = (ctypes.c_int32 * len(flat))(*flat)
            _check(lib.ssa_plan_varlen(coords.data_ptr(), ctypes.addressof(cu), B,
                                       ctypes.addressof(gr), block, r, st, ctypes.byref(self._h)),
                   "ssa_plan_varlen")
        self._sizes()
        self.r = r

    def rebuild(self, coords: torch.Tensor):
        """Recompute the plan in place for new coordinates (same count, layout, grids, r)."""
        _dev(coords, torch.int32)
        _check(lib.ssa_plan_rebuild(self._h, coords.data_ptr(), _stream(self.stream)),
               "ssa_plan_rebuild")
        self._sizes()
        return self

    def _sizes(self):
        n, mb, b = _i64(), _i64(), _i32()
        _check(lib.ssa_plan_info(self._h, ctypes.byref(n), ctypes.byref(mb), None, ctypes.byref(b)),
               "ssa_plan_info")
        self.N, self.num_blocks, self.batch = n.value, mb.value, b.value

    @property
    def nnz(self) -> int:
        """Total length of the per-token window neighbour lists (counted on first request)."""
        v = _i64()
        _check(lib.ssa_plan_info(self._h, None, None, ctypes.byref(v), None), "ssa_plan_info")
        return v.value

    def close(self):
        if self._h:
            lib.ssa_plan_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def export(self):
        """The canonical plan arrays as CUDA tensors (see ssa_plan_export)."""
        dev = torch.device("cuda")
        i32 = dict(dtype=torch.int32, device=dev)
        out = dict(perm=torch.empty(self.N, **i32), tok_blk=torch.empty(self.N, **i32),
                   blk_off=torch.empty(self.num_blocks + 1, **i32),
                   blk_coord=torch.empty(self.num_blocks, 3, **i32),
                   blk_seq=torch.empty(self.num_blocks, **i32),
                   nbr_off=torch.empty(self.N + 1, dtype=torch.int64, device=dev),
                   nbr_idx=torch.empty(max(self.nnz, 1), **i32))
        _check(lib.ssa_plan_export(self._h, *[_ptr(out[k]) for k in
                                              ("perm", "tok_blk", "blk_off", "blk_coord", "blk_seq",
                                               "nbr_off", "nbr_idx")], _stream(self.stream)),
               "ssa_plan_export")
        out["nbr_idx"] = out["nbr_idx"][:self.nnz]
        return out

    def _args(self, q, k, v, gates, wc):
        dt = q.dtype
        for t in (q, k, v):
            _dev(t, dt)
            if t.dim() != 3 or t.shape[0] != self.N:
                raise ValueError("q, k, v must be [N, H, D]")
        _dev(gates, torch.float32)
        _dev(wc, torch.float32)
        return dt, q.shape[1], q.shape[2]

    def forward(self, q, k, v, gates, wc, topk: int, out: Optional[torch.Tensor] = None,
                return_sel: bool = False, return_branches: bool = False):
        """out [N, H, D]; with return_sel also the selection [N, H, k] (int32, global block
        indices); with return_branches also (o_cmp, o_sel, o_win), fp32 [N, H, D] each."""
        dt, H, D = self._args(q, k, v, gates, wc)
        out = torch.empty_like(q) if out is None else _dev(out, dt)
        st = _stream(self.stream)
        if return_sel or return_branches:
            sel = torch.empty(self.N, H, topk, dtype=torch.int32, device=q.device) if return_sel else None
            br = [torch.empty(self.N, H, D, dtype=torch.float32, device=q.device)
                  for _ in range(3)] if return_branches else [None] * 3
            _check(lib.ssa_forward_debug(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         gates.data_ptr(), wc.data_ptr(), H, D, _DTYPE[dt], topk,
                                         out.data_ptr(), _ptr(sel), *[_ptr(b) for b in br], st),
                   "ssa_forward_debug")
            res = (out,)
            if return_sel:
                res += (sel,)
            if return_branches:
                res += (tuple(br),)
            return res
        _check(lib.ssa_forward(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), gates.data_ptr(),
                               wc.data_ptr(), H, D, _DTYPE[dt], topk, out.data_ptr(), st),
               "ssa_forward")
        return out

    def forward_prologue(self, q, k, v, gates, wc, topk: int, q_gamma, k_gamma,
                         rope_theta: float = 10000.0, eps: float = 1e-6,
                         out: Optional[torch.Tensor] = None, return_sel: bool = False):
        """ssa_forward_prologue: RMS-normalised, rotary-embedded q and k, then the method.
        q_gamma, k_gamma: fp32 CUDA tensors [D]."""
        dt, H, D = self._args(q, k, v, gates, wc)
        for gm in (q_gamma, k_gamma):
            _dev(gm, torch.float32)
            if gm.numel() != D:
                raise ValueError("q_gamma and k_gamma must hold D values")
        out = torch.empty_like(q) if out is None else _dev(out, dt)
        sel = torch.empty(self.N, H, topk, dtype=torch.int32, device=q.device) if return_sel else None
        _check(lib.ssa_forward_prologue(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        gates.data_ptr(), wc.data_ptr(), q_gamma.data_ptr(),
                                        k_gamma.data_ptr(), float(rope_theta), float(eps), H, D,
                                        _DTYPE[dt], topk, out.data_ptr(), _ptr(sel),
                                        _stream(self.stream)), "ssa_forward_prologue")
        return (out, sel) if return_sel else out

    def forward_ex(self, q, k, v, gates, wc, topk: int, q_gamma=None, k_gamma=None,
                   rope_theta: float = 10000.0, eps: float = 1e-6, conv_w=None, gate_w=None,
                   gate_b=None, out: Optional[torch.Tensor] = None, return_sel: bool = False,
                   share_selection: bool = False):
        """ssa_forward_ex: the prologue (q_gamma, k_gamma [D]), the compression by sparse 3D
        convolution over the block grid (conv_w [27, D, D]) and gates predicted from the queries
        (gate_w [D, 3], gate_b [3]), each optional (fp32 CUDA tensors). gates / wc may be None when
        predicted / replaced by the convolution. share_selection: one selection per 4x4x4
        sub-block of cells, from the summed compressed-attention weights of its queries."""
        dt = q.dtype
        for t in (q, k, v):
            _dev(t, dt)
            if t.dim() != 3 or t.shape[0] != self.N:
                raise ValueError("q, k, v must be [N, H, D]")
        H, D = q.shape[1], q.shape[2]
        for t in (gates, wc, q_gamma, k_gamma, conv_w, gate_w, gate_b):
            if t is not None:
                _dev(t, torch.float32)
        opt = Options(_ptr(q_gamma), _ptr(k_gamma), float(rope_theta), float(eps), _ptr(conv_w),
                      _ptr(gate_w), _ptr(gate_b), int(bool(share_selection)))
        out = torch.empty_like(q) if out is None else _dev(out, dt)
        sel = torch.empty(self.N, H, topk, dtype=torch.int32, device=q.device) if return_sel else None
        _check(lib.ssa_forward_ex(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(gates),
                                  _ptr(wc), H, D, _DTYPE[dt], topk, ctypes.byref(opt),
                                  out.data_ptr(), _ptr(sel), _stream(self.stream)), "ssa_forward_ex")
        return (out, sel) if return_sel else out

    def forward_host(self, q, k, v, gates, wc, topk: int, out: torch.Tensor):
        """Forward on host (preferably pinned) CPU tensors; copies run inside the library."""
        for t in (q, k, v, gates, wc, out):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("forward_host takes contiguous CPU tensors")
        H, D = q.shape[1], q.shape[2]
        _check(lib.ssa_forward_host(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    gates.data_ptr(), wc.data_ptr(), H, D, _DTYPE[q.dtype], topk,
                                    out.data_ptr(), _stream(self.stream)), "ssa_forward_host")
        return out

    def backward(self, q, k, v, gates, wc, dout, topk: int):
        dt, H, D = self._args(q, k, v, gates, wc)
        _dev(dout, dt)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        _check(lib.ssa_backward(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                gates.data_ptr(), wc.data_ptr(), dout.data_ptr(), H, D,
                                _DTYPE[dt], topk, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                _stream(self.stream)), "ssa_backward")
        return dq, dk, dv

    def debug_wait_timeout(self, max_cycles: int):
        """ssa_debug_wait_timeout: a bounded wait that runs out on purpose (failure detection)."""
        _check(lib.ssa_debug_wait_timeout(self._h, int(max_cycles), _stream(self.stream)),
               "ssa_debug_wait_timeout")

    def status(self):
        """Waits for the stream, returns and clears the device status (0 = ok)."""
        return lib.ssa_last_device_status(self._h, _stream(self.stream))

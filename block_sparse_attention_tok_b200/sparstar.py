"""Python binding of the C-ABI library (libsparstar.so): argument marshalling only.

Every step of the path (pooling, scoring, Top-K, attention) runs in the library's CUDA
kernels. Torch is used to allocate device memory and to name the current stream. The
binding raises if the library is missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import _build

BLOCK = 128
BUDGET_LITERAL = 0
BUDGET_CANDIDATES = 1

OK = 0
ERR_ARG = 1
ERR_UNSUPPORTED = 2
ERR_WORKSPACE = 3
ERR_CUDA = 4
ERR_DEVICE_TIMEOUT = 5
ERR_DEVICE_BOUNDS = 6

# Every function the header declares, with (restype, argtypes).
_c = ctypes
_SIGNATURES = {}


class Segments(ctypes.Structure):
    _fields_ = [("n_text", ctypes.c_int64), ("n_ctx", ctypes.c_int64), ("n_cur", ctypes.c_int64)]


class Grid(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int64), ("height", ctypes.c_int64), ("width", ctypes.c_int64)]


class Plan(ctypes.Structure):
    _fields_ = [("nqb", ctypes.c_int64), ("nkb", ctypes.c_int64), ("n_forced", ctypes.c_int64),
                ("n_cand", ctypes.c_int64), ("k_total", ctypes.c_int32), ("k_topk", ctypes.c_int32)]

    def as_dict(self):
        return {f: int(getattr(self, f)) for f, _ in self._fields_}


_SIGNATURES.update({
    "sparstar_abi_version": (_c.c_int, []),
    "sparstar_strerror": (_c.c_char_p, [_c.c_int]),
    "sparstar_make_plan": (_c.c_int, [_c.c_int64, Segments, _c.c_int, _c.c_double, _c.c_int, _c.POINTER(Plan)]),
    "sparstar_workspace_size": (_c.c_int, [_c.c_int, _c.c_int64, Segments, _c.c_int, _c.POINTER(_c.c_size_t)]),
    "sparstar_select": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, Segments, _c.c_int, _c.c_int,
                                   _c.c_double, _c.c_int, _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p,
                                   _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "sparstar_attn": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                 _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_float, _c.c_void_p, _c.c_void_p,
                                 _c.c_void_p]),
    "sparstar_forward": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, Segments, _c.c_int,
                                    _c.c_int, _c.c_double, _c.c_int, _c.c_float, _c.c_void_p, _c.c_void_p,
                                    _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "sparstar_device_status": (_c.c_int, [_c.c_void_p, _c.c_int]),
    "sparstar_selftest_wait_timeout": (_c.c_int, [_c.c_void_p]),
    "sparstar_make_plan_ex": (_c.c_int, [_c.c_int64, Segments, _c.c_int, _c.c_double, _c.c_int, _c.c_int,
                                         _c.POINTER(Plan)]),
    "sparstar_workspace_size_ex": (_c.c_int, [_c.c_int, _c.c_int64, Segments, _c.c_int, _c.c_int,
                                              _c.POINTER(_c.c_size_t)]),
    "sparstar_select_ex": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, Segments, _c.c_int, _c.c_int,
                                      _c.c_double, _c.c_int, _c.c_int, _c.c_void_p, _c.c_void_p, _c.c_int32,
                                      _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "sparstar_attn_ex": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                    _c.c_int, _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_float, _c.c_void_p,
                                    _c.c_void_p, _c.c_void_p]),
    "sparstar_forward_ex": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, Segments,
                                       _c.c_int, _c.c_int, _c.c_double, _c.c_int, _c.c_int, _c.c_float, _c.c_void_p,
                                       _c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                       _c.c_void_p]),
    "sparstar_select_noalloc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, Segments, _c.c_int,
                                           _c.c_int, _c.c_double, _c.c_int, _c.c_void_p, _c.c_void_p, _c.c_int32,
                                           _c.c_void_p]),
})
_SIGNATURES.update({
    "sparstar_retained_mass": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                          _c.c_void_p]),
    "sparstar_token_bound_workspace_size": (_c.c_int, [_c.c_int, _c.c_int64, _c.POINTER(_c.c_size_t)]),
    "sparstar_token_bound": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                        _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_float, _c.c_void_p,
                                        _c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "sparstar_topk": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int, _c.c_int, _c.c_int, _c.c_void_p, _c.c_void_p,
                                 _c.c_int32, _c.c_void_p]),
    "sparstar_read_probe": (_c.c_int, [_c.c_void_p, _c.c_size_t, _c.c_void_p, _c.c_void_p]),
    "sparstar_map_scores": (_c.c_int, [_c.c_void_p, _c.c_int, Segments, Grid, Segments, Grid, _c.c_void_p,
                                       _c.c_void_p]),
})
NOALLOC_SCRATCH_BYTES = 128 << 20

_LIB: Optional[ctypes.CDLL] = None


class SparstarError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


def lib_path() -> str:
    return _build.LIB_PATH


def load() -> ctypes.CDLL:
    """Load libsparstar.so from the package directory (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with __graft_entry__.build() "
                               "(there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def strerror(code: int) -> str:
    return load().sparstar_strerror(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise SparstarError(code, where)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr()) or None


def make_plan(n_q: int, n_text: int, n_ctx: int, n_cur: int, clip: int, density: float,
              budget_mode: int = BUDGET_LITERAL, block: int = BLOCK) -> Plan:
    plan = Plan()
    _check(load().sparstar_make_plan_ex(int(n_q), Segments(n_text, n_ctx, n_cur), int(clip), float(density),
                                        int(budget_mode), int(block), ctypes.byref(plan)), "sparstar_make_plan_ex")
    return plan


def workspace_size(heads: int, n_q: int, n_text: int, n_ctx: int, n_cur: int, head_dim: int,
                   block: int = BLOCK) -> int:
    out = ctypes.c_size_t()
    _check(load().sparstar_workspace_size_ex(int(heads), int(n_q), Segments(n_text, n_ctx, n_cur), int(head_dim),
                                             int(block), ctypes.byref(out)), "sparstar_workspace_size_ex")
    return int(out.value)


def _check_qkv(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("q/k/v must be contiguous bf16 CUDA tensors of shape [H, N, d]")


class Workspace:
    """Reusable device workspace sized for one shape (allocated once by torch)."""

    def __init__(self, heads, n_q, n_text, n_ctx, n_cur, head_dim, device, block: int = 128):
        nbytes = workspace_size(heads, n_q, n_text, n_ctx, n_cur, head_dim, block)
        self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        self.nbytes = nbytes


def select(q: torch.Tensor, k: torch.Tensor, n_text: int, n_ctx: int, n_cur: int, clip: int, density: float,
           budget_mode: int = BUDGET_LITERAL, want_scores: bool = False, workspace: Optional[Workspace] = None,
           idx: Optional[torch.Tensor] = None, cnt: Optional[torch.Tensor] = None, stream=None,
           block: int = BLOCK):
    """Block selection with `block`-token blocks (128, or 64). Returns (idx [H,nqb,K_total]
    int32, cnt [H,nqb] int32, scores or None)."""
    _check_qkv(q, k)
    H, n_q, d = q.shape
    plan = make_plan(n_q, n_text, n_ctx, n_cur, clip, density, budget_mode, block)
    nqb, nkb, kmax = int(plan.nqb), int(plan.nkb), max(int(plan.k_total), 1)
    if idx is None:
        idx = torch.empty(H, nqb, kmax, dtype=torch.int32, device=q.device)
    if cnt is None:
        cnt = torch.empty(H, nqb, dtype=torch.int32, device=q.device)
    scores = torch.empty(H, nqb, nkb, dtype=torch.float32, device=q.device) if want_scores else None
    if workspace is None:
        workspace = Workspace(H, n_q, n_text, n_ctx, n_cur, d, q.device, block)
    _check(load().sparstar_select_ex(_ptr(q), _ptr(k), H, n_q, Segments(n_text, n_ctx, n_cur), d, int(clip),
                                     float(density), int(budget_mode), int(block), _ptr(idx), _ptr(cnt),
                                     idx.shape[-1], _ptr(scores), _ptr(workspace.buf), workspace.nbytes,
                                     _stream_ptr(stream)), "sparstar_select_ex")
    return idx, cnt, scores


def attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, cnt: torch.Tensor,
         sm_scale: float = 0.0, o: Optional[torch.Tensor] = None, want_lse: bool = True,
         lse: Optional[torch.Tensor] = None, stream=None, block: int = BLOCK) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Block-sparse attention over the kept tiles (`block`-token blocks). Returns (o bf16
    [H,Nq,d], lse fp32 [H,Nq] or None)."""
    _check_qkv(q, k, v)
    H, n_q, d = q.shape
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or not idx.is_contiguous() or not cnt.is_contiguous():
        raise ValueError("idx/cnt must be contiguous int32")
    if o is None:
        o = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty(H, n_q, dtype=torch.float32, device=q.device)
    _check(load().sparstar_attn_ex(_ptr(q), _ptr(k), _ptr(v), H, n_q, k.shape[1], d, int(block), _ptr(idx),
                                   _ptr(cnt), idx.shape[-1], float(sm_scale), _ptr(o), _ptr(lse), _stream_ptr(stream)),
           "sparstar_attn_ex")
    return o, lse


def topk(scores: torch.Tensor, n_forced: int, k_topk: int, idx: Optional[torch.Tensor] = None,
         cnt: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Clip-aware retention + joint Top-K on given scores [..., nkb] (fp32, contiguous CUDA):
    each row keeps blocks 0..n_forced-1 and its k_topk best other columns, ascending.
    Returns (idx int32 [..., n_forced + k_topk] unless a wider idx is given, cnt int32 [...])."""
    if scores.dtype != torch.float32 or not scores.is_cuda or not scores.is_contiguous() or scores.dim() < 1:
        raise ValueError("scores must be a contiguous fp32 CUDA tensor [..., nkb]")
    lead, nkb = tuple(scores.shape[:-1]), scores.shape[-1]
    rows = scores.numel() // nkb if nkb else 0
    if idx is None:
        idx = torch.empty(*lead, n_forced + k_topk, dtype=torch.int32, device=scores.device)
    if cnt is None:
        cnt = torch.empty(*lead, dtype=torch.int32, device=scores.device)
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or not idx.is_contiguous() or not cnt.is_contiguous():
        raise ValueError("idx/cnt must be contiguous int32")
    _check(load().sparstar_topk(_ptr(scores), rows, nkb, int(n_forced), int(k_topk), _ptr(idx), _ptr(cnt),
                                idx.shape[-1], _stream_ptr(stream)), "sparstar_topk")
    return idx, cnt


def _check_lse(*ts):
    for t in ts:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 2:
            raise ValueError("LSEs must be contiguous fp32 CUDA tensors of shape [H, Nq]")


def retained_mass(lse_kept: torch.Tensor, lse_dense: torch.Tensor, want_tokens: bool = True, stream=None):
    """Retained dense softmax mass of a mask from the two LSEs of sparstar_attn (mask / all
    blocks). Returns (R fp32 [H,Nq] or None, per-query-block mean fp32 [H,nqb])."""
    _check_lse(lse_kept, lse_dense)
    H, n_q = lse_kept.shape
    nqb = -(-n_q // 128)
    r = torch.empty(H, n_q, dtype=torch.float32, device=lse_kept.device) if want_tokens else None
    e = torch.empty(H, nqb, dtype=torch.float32, device=lse_kept.device)
    _check(load().sparstar_retained_mass(_ptr(lse_kept), _ptr(lse_dense), H, n_q, _ptr(r), _ptr(e),
                                         _stream_ptr(stream)), "sparstar_retained_mass")
    return r, e


def token_bound(q: torch.Tensor, k: torch.Tensor, idx: torch.Tensor, cnt: torch.Tensor, lse_dense: torch.Tensor,
                sm_scale: float = 0.0, want_tokens: bool = True, stream=None):
    """Token-wise upper bound on the retained mass with each row's kept-token budget.
    Returns (U fp32 [H,Nq] or None, per-query-block mean fp32 [H,nqb])."""
    _check_qkv(q, k)
    _check_lse(lse_dense)
    H, n_q, d = q.shape
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or not idx.is_contiguous() or not cnt.is_contiguous():
        raise ValueError("idx/cnt must be contiguous int32")
    nqb = -(-n_q // 128)
    nbytes = ctypes.c_size_t()
    _check(load().sparstar_token_bound_workspace_size(H, n_q, ctypes.byref(nbytes)), "sparstar_token_bound_workspace_size")
    ws = torch.empty(max(int(nbytes.value), 256), dtype=torch.uint8, device=q.device)
    u = torch.empty(H, n_q, dtype=torch.float32, device=q.device) if want_tokens else None
    ub = torch.empty(H, nqb, dtype=torch.float32, device=q.device)
    _check(load().sparstar_token_bound(_ptr(q), _ptr(k), H, n_q, k.shape[1], d, _ptr(idx), _ptr(cnt), idx.shape[-1],
                                       _ptr(lse_dense), float(sm_scale), _ptr(u), _ptr(ub), _ptr(ws), int(nbytes.value),
                                       _stream_ptr(stream)), "sparstar_token_bound")
    return u, ub


def forward(q, k, v, n_text, n_ctx, n_cur, clip, density, budget_mode=BUDGET_LITERAL, sm_scale=0.0,
            workspace: Optional[Workspace] = None, idx=None, cnt=None, o=None, lse=None, want_lse=True,
            stream=None, block: int = BLOCK):
    """The whole per-scale path (selection then attention). Returns (o, lse, idx, cnt)."""
    _check_qkv(q, k, v)
    H, n_q, d = q.shape
    plan = make_plan(n_q, n_text, n_ctx, n_cur, clip, density, budget_mode, block)
    kmax = max(int(plan.k_total), 1)
    if idx is None:
        idx = torch.empty(H, int(plan.nqb), kmax, dtype=torch.int32, device=q.device)
    if cnt is None:
        cnt = torch.empty(H, int(plan.nqb), dtype=torch.int32, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty(H, n_q, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = Workspace(H, n_q, n_text, n_ctx, n_cur, d, q.device, block)
    _check(load().sparstar_forward_ex(_ptr(q), _ptr(k), _ptr(v), H, n_q, Segments(n_text, n_ctx, n_cur), d,
                                      int(clip), float(density), int(budget_mode), int(block), float(sm_scale),
                                      _ptr(idx), _ptr(cnt), idx.shape[-1], _ptr(o), _ptr(lse), _ptr(workspace.buf),
                                      workspace.nbytes, _stream_ptr(stream)), "sparstar_forward_ex")
    return o, lse, idx, cnt


def select_noalloc(q: torch.Tensor, k: torch.Tensor, n_text: int, n_ctx: int, n_cur: int, clip: int,
                   density: float, budget_mode: int = BUDGET_LITERAL, idx: Optional[torch.Tensor] = None,
                   cnt: Optional[torch.Tensor] = None, stream=None):
    """Block selection without any device allocation inside the library: its scratch is the
    library's fixed array (NOALLOC_SCRATCH_BYTES per device). For callers that cannot call
    cudaMalloc; they pass idx and cnt buffers they already own. Calls that overlap on the
    GPU share that array and race. Returns (idx, cnt)."""
    _check_qkv(q, k)
    H, n_q, d = q.shape
    plan = make_plan(n_q, n_text, n_ctx, n_cur, clip, density, budget_mode)
    if idx is None:
        idx = torch.empty(H, int(plan.nqb), max(int(plan.k_total), 1), dtype=torch.int32, device=q.device)
    if cnt is None:
        cnt = torch.empty(H, int(plan.nqb), dtype=torch.int32, device=q.device)
    _check(load().sparstar_select_noalloc(_ptr(q), _ptr(k), H, n_q, Segments(n_text, n_ctx, n_cur), d, int(clip),
                                          float(density), int(budget_mode), _ptr(idx), _ptr(cnt), idx.shape[-1],
                                          _stream_ptr(stream)), "sparstar_select_noalloc")
    return idx, cnt


def map_scores(scores_prev: torch.Tensor, seg_prev, grid_prev, seg_now, grid_now, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Block scores of a previous scale of the clip carried to the current scale through the
    nearest-raster-position block map (seg_* = (n_text, n_ctx, n_cur), grid_* = (frames, height,
    width) of the current tokens). Returns fp32 [H, nqb_now, nkb_now]."""
    if scores_prev.dtype != torch.float32 or not scores_prev.is_cuda or not scores_prev.is_contiguous() \
            or scores_prev.dim() != 3:
        raise ValueError("scores_prev must be a contiguous fp32 CUDA tensor [H, nqb, nkb]")
    H = scores_prev.shape[0]
    n_prefix = (seg_now[0] + seg_now[1]) // BLOCK
    nqb_now = -(-seg_now[2] // BLOCK)
    if out is None:
        out = torch.empty(H, nqb_now, n_prefix + nqb_now, dtype=torch.float32, device=scores_prev.device)
    _check(load().sparstar_map_scores(_ptr(scores_prev), H, Segments(*seg_prev), Grid(*grid_prev), Segments(*seg_now),
                                      Grid(*grid_now), _ptr(out), _stream_ptr(stream)), "sparstar_map_scores")
    return out


def read_probe(buf: torch.Tensor, sink: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Measurement aid: one streaming read of `buf` (a contiguous CUDA tensor whose size is a
    multiple of 16 bytes), XOR-folded into a 4-byte sink, which is returned."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    _check(load().sparstar_read_probe(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), _stream_ptr(stream)),
           "sparstar_read_probe")
    return sink


def device_status(clear: bool = True, stream=None) -> int:
    """Synchronize and return the device status code (OK, ERR_DEVICE_TIMEOUT or ERR_DEVICE_BOUNDS)."""
    return int(load().sparstar_device_status(_stream_ptr(stream), 1 if clear else 0))


def selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test: the next device_status() reports ERR_DEVICE_TIMEOUT."""
    _check(load().sparstar_selftest_wait_timeout(_stream_ptr(stream)), "sparstar_selftest_wait_timeout")


def exported_symbols():
    return list(_SIGNATURES)

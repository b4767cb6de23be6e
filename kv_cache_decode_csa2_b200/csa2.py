"""Thin Python binding of libcsa2 (include/csa2.h).

Argument marshalling only.  Every step of the CSA2 decode path runs in the
library's CUDA kernels.  PyTorch provides device buffers (inputs, outputs,
workspaces, the status word) and the stream.  There is no fallback: if the
library cannot be loaded, every call raises.

The functions keep the C names: csa2_index_full, csa2_topk_pool,
csa2_reindex, csa2_sparse_attn_fp4, csa2_layer_plan and csa2_fp4_quantize.
Each takes torch tensors.  It allocates the workspace the library asks for
(unless one is passed) and raises Csa2Error on a non-zero return.  Errors
found on the device land in the int32 ``status`` tensor; check_status() reads
it, which synchronises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcsa2.so")

FULL, REINDEX, REUSE = 0, 1, 2
STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA", 5: "SCORE_RANGE",
          6: "INDEX_RANGE", 7: "TIMEOUT", 8: "ORDER"}


class Csa2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} ({code})")
        self.code = code


class csa2_rows(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("row_bytes", ctypes.c_int64), ("n_rows", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("page_rows", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("seq_rows", ctypes.c_int64)]


class csa2_layer(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("w", ctypes.c_void_p), ("keys", csa2_rows),
                ("q_attn", ctypes.c_void_p), ("codes", csa2_rows), ("scales", csa2_rows),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("pool_idx", ctypes.c_void_p),
                ("pool_cnt", ctypes.c_void_p), ("sel_idx", ctypes.c_void_p), ("sel_cnt", ctypes.c_void_p),
                ("local_kv", csa2_rows)]


class csa2_plan_shape(ctypes.Structure):
    _fields_ = [("nq", ctypes.c_int32), ("H", ctypes.c_int32), ("D_idx", ctypes.c_int32),
                ("Hq", ctypes.c_int32), ("D", ctypes.c_int32), ("P", ctypes.c_int32),
                ("K", ctypes.c_int32), ("window", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("seq_of_query", ctypes.c_void_p),
                ("query_pos", ctypes.c_void_p), ("group_queries", ctypes.c_int32)]


_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_RP = ctypes.POINTER(csa2_rows)
_SIGS = {
    "csa2_index_full": (_I32, [_P, _P, _RP, _P, _P, _I32, _I32, _I32, _I32, _P, _I64, _I32, _P, _P, _I32,
                               _P, _P, _P, _SZ, _P, _P]),
    "csa2_index_full_workspace": (_SZ, [_I32, _I32, _I32, _I32]),
    "csa2_topk_pool": (_I32, [_P, _I64, _P, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P, _P]),
    "csa2_topk_pool_workspace": (_SZ, [_I32, _I32, _I32]),
    "csa2_topk_pool_noalloc": (_I32, [_P, _I64, _P, _P, _I32, _I32, _I32, _P, _P, _P, _P]),
    "csa2_reindex": (_I32, [_P, _P, _RP, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _SZ,
                            _P, _P]),
    "csa2_reindex_workspace": (_SZ, [_I32, _I32, _I32]),
    "csa2_sparse_attn_fp4": (_I32, [_P, _RP, _RP, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _F, _P,
                                    _P, _P, _SZ, _P, _P]),
    "csa2_sparse_attn_workspace": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "csa2_sparse_attn_fp4_local": (_I32, [_P, _RP, _RP, _RP, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _F,
                                          _P, _P, _P, _SZ, _P, _P]),
    "csa2_layer_plan": (_I32, [_P, _I32, ctypes.POINTER(csa2_layer), ctypes.POINTER(csa2_plan_shape), _P,
                               _SZ, _P, _P]),
    "csa2_layer_plan_workspace": (_SZ, [_P, _I32, ctypes.POINTER(csa2_plan_shape)]),
    "csa2_attn_combine": (_I32, [_P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P]),
    "csa2_fp4_quantize": (_I32, [_P, _I64, _I32, _I64, _P, _P, _I64, _P, _I64, _I64, _P, _P]),
    "csa2_fp4_quantize_bf16": (_I32, [_P, _I64, _I32, _I64, _P, _P, _I64, _P, _I64, _I64, _P, _P]),
    "csa2_status_string": (ctypes.c_char_p, [_I32]),
    "csa2_version": (_I32, []),
    "csa2_selftest_wait": (_I32, [_I32, ctypes.c_uint64, _P, _P, _P]),
    "csa2_trace_table_bytes": (_SZ, []),
    "csa2_trace_attach": (_I32, [_P]),
}
EXPORTS = tuple(_SIGS)

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libcsa2 with every prototype set.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m kv_cache_decode_csa2_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ----------------------------------------------------------------- helpers
def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(code: int, where: str) -> None:
    if code != 0:
        raise Csa2Error(code, where)


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status: torch.Tensor) -> None:
    """Raises Csa2Error if a kernel recorded an error (synchronises)."""
    code = int(status.item())
    if code:
        raise Csa2Error(code, "device")


@dataclass
class Rows:
    """A per-position row view (index keys, FP4 codes or FP4 scales).

    ``data`` is a 2-D uint8/int8 tensor of physical rows.  ``page_table``, if
    given, is int32 [n_seq][max_pages] with ``page_rows`` rows per page;
    otherwise sequence s starts at row s*seq_rows."""
    data: torch.Tensor
    page_table: torch.Tensor | None = None
    page_rows: int = 64
    seq_rows: int = 0

    def c(self) -> csa2_rows:
        d = self.data
        if not d.is_cuda or d.dim() != 2 or d.stride(1) != 1:
            raise ValueError("row data must be a 2-D CUDA tensor with unit inner stride")
        r = csa2_rows()
        r.base = d.data_ptr()
        r.row_bytes = d.stride(0) * d.element_size()
        r.n_rows = d.shape[0]
        if self.page_table is not None:
            _dev(self.page_table, torch.int32, "page_table")
            r.page_table = self.page_table.data_ptr()
            r.page_rows = self.page_rows
            r.max_pages = self.page_table.shape[1]
        else:
            r.page_table = None
            r.page_rows = 0
            r.max_pages = 0
        r.seq_rows = self.seq_rows
        return r


# ----------------------------------------------------------------- entry points
def csa2_index_full(q, w, keys: Rows, query_pos, max_ctx: int, *, seq_of_query=None, scores=None,
                    P: int = 0, pool_idx=None, pool_cnt=None, K: int = 0, sel_idx=None, sel_cnt=None,
                    status=None, ws=None, stream=None):
    """Full-mode index scores (+ pool of P, + top-K).  q int8 [nq][H][D], w int8 [nq][H]."""
    L = lib()
    _dev(q, torch.int8, "q")
    _dev(w, torch.int8, "w")
    _dev(query_pos, torch.int32, "query_pos")
    nq, H, D = q.shape
    status = new_status(q.device) if status is None else status
    need = L.csa2_index_full_workspace(nq, max_ctx, P, K)
    ws = _workspace(need, q.device) if ws is None else ws
    kr = keys.c()
    code = L.csa2_index_full(_ptr(q), _ptr(w), ctypes.byref(kr), _ptr(seq_of_query), _ptr(query_pos), nq, H, D,
                             max_ctx, _ptr(scores), scores.stride(0) if scores is not None else 0, P,
                             _ptr(pool_idx), _ptr(pool_cnt), K, _ptr(sel_idx), _ptr(sel_cnt), _ptr(ws),
                             ws.numel(), _ptr(status), _stream(stream))
    _check(code, "csa2_index_full")
    return status


def csa2_topk_pool(scores, k: int, out_idx, *, n_valid=None, cand_pos=None, out_cnt=None, n_max=None,
                   status=None, ws=None, stream=None):
    """Exact top-k of int32 scores [nq][ld]; ties to the lower position; ascending output."""
    L = lib()
    _dev(scores, torch.int32, "scores")
    nq, ld = scores.shape
    n_max = ld if n_max is None else n_max
    status = new_status(scores.device) if status is None else status
    need = L.csa2_topk_pool_workspace(nq, n_max, k)
    ws = _workspace(need, scores.device) if ws is None else ws
    code = L.csa2_topk_pool(_ptr(scores), ld, _ptr(n_valid), _ptr(cand_pos), nq, n_max, k, _ptr(out_idx),
                            _ptr(out_cnt), _ptr(ws), ws.numel(), _ptr(status), _stream(stream))
    _check(code, "csa2_topk_pool")
    return status


def csa2_reindex(q, w, keys: Rows, pool_idx, pool_cnt, K: int, sel_idx, *, sel_cnt=None, scores=None,
                 seq_of_query=None, status=None, ws=None, stream=None):
    """Re-score the pool with this layer's q, w, keys and keep the best K."""
    L = lib()
    _dev(q, torch.int8, "q")
    _dev(pool_idx, torch.int32, "pool_idx")
    nq, H, D = q.shape
    P = pool_idx.shape[1]
    status = new_status(q.device) if status is None else status
    need = L.csa2_reindex_workspace(nq, P, K)
    ws = _workspace(need, q.device) if ws is None else ws
    kr = keys.c()
    code = L.csa2_reindex(_ptr(q), _ptr(w), ctypes.byref(kr), _ptr(seq_of_query), _ptr(pool_idx),
                          _ptr(pool_cnt), nq, H, D, P, K, _ptr(sel_idx), _ptr(sel_cnt), _ptr(scores),
                          _ptr(ws), ws.numel(), _ptr(status), _stream(stream))
    _check(code, "csa2_reindex")
    return status


def csa2_sparse_attn_fp4(q, codes: Rows, scales: Rows, query_pos, sel_idx, out, *, sel_cnt=None,
                         seq_of_query=None, window: int = 128, softmax_scale: float = 0.0, lse=None,
                         local_kv: Rows | None = None, status=None, ws=None, stream=None):
    """Attention over selection U window on the FP4 cache.  q bf16 [nq][Hq][D].
    With ``local_kv`` (bf16 rows [n_seq * R][D], ``seq_rows`` = R >= window)
    the window rows come from the layer's local cache
    (csa2_sparse_attn_fp4_local)."""
    L = lib()
    _dev(q, torch.bfloat16, "q")
    _dev(out, torch.bfloat16, "out")
    nq, Hq, D = q.shape
    K = sel_idx.shape[1] if sel_idx is not None else 0
    status = new_status(q.device) if status is None else status
    need = L.csa2_sparse_attn_workspace(nq, Hq, D, K, window)
    ws = _workspace(need, q.device) if ws is None else ws
    cr, sr = codes.c(), scales.c()
    tail = (_ptr(seq_of_query), _ptr(query_pos), _ptr(sel_idx), _ptr(sel_cnt), nq, Hq, D, K, window,
            softmax_scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(status), _stream(stream))
    if local_kv is None:
        code = L.csa2_sparse_attn_fp4(_ptr(q), ctypes.byref(cr), ctypes.byref(sr), *tail)
        _check(code, "csa2_sparse_attn_fp4")
    else:
        if local_kv.data.dtype != torch.bfloat16:
            raise ValueError("local_kv rows must be bfloat16")
        lr = local_kv.c()
        code = L.csa2_sparse_attn_fp4_local(_ptr(q), ctypes.byref(cr), ctypes.byref(sr), ctypes.byref(lr), *tail)
        _check(code, "csa2_sparse_attn_fp4_local")
    return status


def csa2_fp4_quantize(x, codes, scales, *, dst_rows=None, status=None, stream=None):
    """Store float32 or bfloat16 rows x [n][D] as FP4 codes [*][D/2] and E4M3 scales [*][D/32]."""
    L = lib()
    if not x.is_cuda or x.dtype not in (torch.float32, torch.bfloat16) or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D float32 or bfloat16 CUDA tensor with unit inner stride")
    n, D = x.shape
    status = new_status(x.device) if status is None else status
    fn, name = ((L.csa2_fp4_quantize_bf16, "csa2_fp4_quantize_bf16") if x.dtype == torch.bfloat16
                else (L.csa2_fp4_quantize, "csa2_fp4_quantize"))
    code = fn(_ptr(x), n, D, x.stride(0), _ptr(dst_rows), _ptr(codes), codes.stride(0), _ptr(scales),
              scales.stride(0), codes.shape[0], _ptr(status), _stream(stream))
    _check(code, name)
    return status


def csa2_attn_combine(o_parts, lse_parts, out, *, lse_out=None, status=None, stream=None):
    """Attention over the union of R disjoint row sets from the R partial
    results: o_parts bf16 [R][nq][Hq][D], lse_parts float32 [R][nq][Hq]."""
    L = lib()
    _dev(o_parts, torch.bfloat16, "o_parts")
    _dev(lse_parts, torch.float32, "lse_parts")
    _dev(out, torch.bfloat16, "out")
    R, nq, Hq, D = o_parts.shape
    if tuple(lse_parts.shape) != (R, nq, Hq) or tuple(out.shape) != (nq, Hq, D):
        raise ValueError("csa2_attn_combine: shapes do not match")
    status = new_status(o_parts.device) if status is None else status
    _check(L.csa2_attn_combine(_ptr(o_parts), _ptr(lse_parts), R, nq, Hq, D, _ptr(out), _ptr(lse_out),
                               _ptr(status), _stream(stream)), "csa2_attn_combine")
    return status


def csa2_selftest_wait(kind: int, limit_ns: int, *, counter=None, status=None, stream=None):
    """Runs one bounded wait that nothing satisfies (kind 0: the grid
    barrier, on the zeroed int32 ``counter``; kind 1: the mbarrier wait); it
    records CSA2_ERR_TIMEOUT in ``status`` after about ``limit_ns``."""
    L = lib()
    status = new_status() if status is None else status
    if kind == 0 and counter is None:
        counter = torch.zeros(1, dtype=torch.int32, device=status.device)
    _check(L.csa2_selftest_wait(kind, limit_ns, _ptr(counter), _ptr(status), _stream(stream)),
           "csa2_selftest_wait")
    return status


@dataclass
class Layer:
    """Inputs and outputs of one layer of a plan (tensors on the device)."""
    q_attn: torch.Tensor
    codes: Rows
    scales: Rows
    out: torch.Tensor
    q: torch.Tensor | None = None
    w: torch.Tensor | None = None
    keys: Rows | None = None
    lse: torch.Tensor | None = None
    pool_idx: torch.Tensor | None = None
    pool_cnt: torch.Tensor | None = None
    sel_idx: torch.Tensor | None = None
    sel_cnt: torch.Tensor | None = None
    local_kv: Rows | None = None     # the layer's local window cache (bf16 ring of seq_rows rows)


class LayerPlan:
    """A marshalled csa2_layer_plan call: the C structs are built once, so
    run() is one C call (and can be captured in a CUDA graph)."""

    def __init__(self, modes, layers: list[Layer], *, query_pos, max_ctx: int, P: int, K: int,
                 window: int = 128, seq_of_query=None, softmax_scale: float = 0.0, group_queries: bool = False,
                 ws=None):
        self.lib = lib()
        self.keep = (layers, query_pos, seq_of_query)
        L = len(modes)
        self.modes = (ctypes.c_int32 * L)(*modes)
        self.layers = (csa2_layer * L)()
        first = layers[0]
        nq, Hq, D = first.q_attn.shape
        H, D_idx = (first.q.shape[1], first.q.shape[2]) if first.q is not None else (0, 0)
        for i, ly in enumerate(layers):
            c = self.layers[i]
            c.q, c.w = _ptr(ly.q), _ptr(ly.w)
            if ly.keys is not None:
                c.keys = ly.keys.c()
            c.q_attn, c.codes, c.scales = _ptr(ly.q_attn), ly.codes.c(), ly.scales.c()
            c.out, c.lse = _ptr(ly.out), _ptr(ly.lse)
            c.pool_idx, c.pool_cnt = _ptr(ly.pool_idx), _ptr(ly.pool_cnt)
            c.sel_idx, c.sel_cnt = _ptr(ly.sel_idx), _ptr(ly.sel_cnt)
            if ly.local_kv is not None:
                if ly.local_kv.data.dtype != torch.bfloat16:
                    raise ValueError(f"layer {i}: local_kv rows must be bfloat16")
                c.local_kv = ly.local_kv.c()
        s = csa2_plan_shape()
        s.nq, s.H, s.D_idx, s.Hq, s.D, s.P, s.K = nq, H, D_idx, Hq, D, P, K
        s.window, s.max_ctx, s.softmax_scale = window, max_ctx, softmax_scale
        s.seq_of_query, s.query_pos = _ptr(seq_of_query), _ptr(query_pos)
        s.group_queries = 1 if group_queries else 0
        self.shape = s
        need = self.lib.csa2_layer_plan_workspace(self.modes, L, ctypes.byref(s))
        if need == 0:
            raise Csa2Error(1, "csa2_layer_plan_workspace")
        self.ws = _workspace(need, first.q_attn.device) if ws is None else ws
        self.status = new_status(first.q_attn.device)
        self.n = L

    def run(self, stream=None) -> None:
        code = self.lib.csa2_layer_plan(self.modes, self.n, self.layers, ctypes.byref(self.shape),
                                        _ptr(self.ws), self.ws.numel(), _ptr(self.status), _stream(stream))
        _check(code, "csa2_layer_plan")


def csa2_layer_plan(modes, layers: list[Layer], **kw) -> LayerPlan:
    """Runs one decode step through the plan and returns the marshalled plan
    (call .run() again for further steps)."""
    plan = LayerPlan(modes, layers, **kw)
    plan.run()
    return plan

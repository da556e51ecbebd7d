"""Python binding of libjssa.so: torch CUDA tensors in, C-ABI calls out.

Argument marshalling only.  Every step of the decode path runs in the CUDA
kernels behind ``include/jssa.h``; there is no Python or CPU fallback, and a
missing library or a call on tensors that are not on a CUDA device raises.

Layouts (see the header for the full contract):
  q [B, Hq, d]   K [B, T_cap, Hkv, d]   V [B, T_cap, Hkv, dv] (None = latent cache, V is K)
  P [Hkv, d, r] fp32   Kt [B, Hkv, T_cap, r]   seq_lens int32 [B]
  idx int32 [B, Hkv, k] (ascending, -1 padded)   count int32 [B, Hkv]
  out [B, Hq, dv]   lse fp32 [B, Hq]
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjssa.so")

BF16, FP32 = 0, 1
AGG_SUM, AGG_MAX = 0, 1
OP_APPEND, OP_SCORE, OP_TOPK, OP_SELECT, OP_INDEXED_DECODE, OP_DENSE_DECODE, OP_GATHER_THEN_DENSE, OP_DECODE_STEP = \
    range(8)
OP_SELECT_HEADS, OP_INDEXED_DECODE_HEADS, OP_CALIBRATE = 8, 9, 10
DEV_SEQLEN, DEV_INDEX, DEV_POS, DEV_TIMEOUT = 1, 2, 4, 8


class JssaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("libjssa status %d: %s" % (code, msg))
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "d", "dv", "r", "T_cap", "kv_dtype", "kt_dtype")]

    def key(self):
        return tuple(getattr(self, n) for n, _ in self._fields_)


_lib = None

EXPORTS = ("jssa_version", "jssa_status_string", "jssa_last_error", "jssa_workspace_size", "jssa_workspace_init",
           "jssa_append_lowrank", "jssa_score", "jssa_topk", "jssa_select", "jssa_indexed_decode",
           "jssa_dense_decode", "jssa_gather_then_dense", "jssa_decode_step")


def lib():
    """Load libjssa.so (raises if it is missing; there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libjssa.so not found at %s: build it with `python -m token_level_sparse_kv_b200.build`"
                           % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    D = ctypes.POINTER(Dims)
    L.jssa_version.restype = i32
    L.jssa_status_string.restype = ctypes.c_char_p
    L.jssa_status_string.argtypes = [i32]
    L.jssa_last_error.restype = ctypes.c_char_p
    L.jssa_workspace_size.restype = i32
    L.jssa_workspace_size.argtypes = [D, i32, i32, ctypes.POINTER(sz)]
    L.jssa_topk_ex.restype = i32
    L.jssa_topk_ex.argtypes = [D, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    L.jssa_select_ex.restype = i32
    L.jssa_select_ex.argtypes = [D, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]
    L.jssa_decode_step_ex.restype = i32
    L.jssa_decode_step_ex.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.jssa_plan_info.restype = i32
    L.jssa_plan_info.argtypes = [D, i32, i32, i32, ctypes.POINTER(i32), ctypes.c_char_p, sz]
    L.jssa_block_norms.restype = i32
    L.jssa_block_norms.argtypes = [D, vp, vp, vp]
    L.jssa_calibrate_basis.restype = i32
    L.jssa_calibrate_basis.argtypes = [D, vp, i32, vp, vp, i32, i32, vp, vp, vp, sz, vp]
    L.jssa_host_step_bytes.restype = i32
    L.jssa_host_step_bytes.argtypes = [D, ctypes.POINTER(sz)]
    L.jssa_decode_step_host.restype = i32
    L.jssa_decode_step_host.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp, vp, vp, vp, vp, vp,
                                        sz, vp]
    L.jssa_select_heads.restype = i32
    L.jssa_select_heads.argtypes = [D, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    L.jssa_indexed_decode_heads.restype = i32
    L.jssa_indexed_decode_heads.argtypes = [D, vp, vp, vp, vp, vp, i32, vp, f32, vp, vp, vp, sz, vp]
    L.jssa_plan_info_ex.restype = i32
    L.jssa_plan_info_ex.argtypes = [D, i32, i32, i32, vp, ctypes.POINTER(i32), ctypes.c_char_p, sz]
    L.jssa_workspace_init.restype = i32
    L.jssa_workspace_init.argtypes = [vp, sz, vp]
    L.jssa_append_lowrank.restype = i32
    L.jssa_append_lowrank.argtypes = [D, vp, vp, vp, vp, i32, vp, sz, vp]
    L.jssa_score.restype = i32
    L.jssa_score.argtypes = [D, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    L.jssa_topk.restype = i32
    L.jssa_topk.argtypes = [D, vp, vp, i32, vp, vp, vp, sz, vp]
    L.jssa_select.restype = i32
    L.jssa_select.argtypes = [D, vp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
    L.jssa_indexed_decode.restype = i32
    L.jssa_indexed_decode.argtypes = [D, vp, vp, vp, vp, vp, i32, vp, f32, vp, vp, vp, sz, vp]
    L.jssa_dense_decode.restype = i32
    L.jssa_dense_decode.argtypes = [D, vp, vp, vp, vp, i32, f32, vp, vp, vp, sz, vp]
    L.jssa_gather_then_dense.restype = i32
    L.jssa_gather_then_dense.argtypes = [D, vp, vp, vp, vp, vp, i32, vp, f32, vp, sz, vp, vp, vp, sz, vp]
    L.jssa_decode_step.restype = i32
    L.jssa_decode_step.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp, vp, vp, vp, sz, vp]
    _lib = L
    return L


def _check(st):
    if st != 0:
        raise JssaError(st, lib().jssa_last_error().decode(errors="replace"))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dt(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError("bf16 or fp32 expected, got %s" % t.dtype)


def _cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("libjssa works on CUDA tensors only (got a %s tensor)" % t.device)
            if not t.is_contiguous():
                raise ValueError("libjssa needs contiguous tensors")


def make_dims(q, K, V, P=None, Kt=None, r=None):
    """Dims from tensor shapes; V None means a latent cache (V is K)."""
    B, Hq, d = q.shape
    _, T_cap, Hkv, dk = K.shape
    assert dk == d, "q and K widths differ"
    if V is None:
        dv = 512 if d == 576 else d
    else:
        dv = V.shape[3]
    if r is None:
        r = P.shape[2] if P is not None else (Kt.shape[3] if Kt is not None else 8)
    kt = _dt(Kt) if Kt is not None else BF16
    return Dims(B, Hq, Hkv, d, dv, r, T_cap, _dt(K), kt)


FORMS = {"auto": 0, "cluster": 1, "stream": 2, "scan": 3}


class SelectOpts(ctypes.Structure):
    """jssa_select_opts: tokens [0, n_sink) and [T_b - n_recent, T_b) are always
    selected; form forces a selection form; unfused keeps the decode step in
    separate launches."""
    _fields_ = [("n_sink", ctypes.c_int32), ("n_recent", ctypes.c_int32), ("form", ctypes.c_int32),
                ("unfused", ctypes.c_int32), ("block_norms", ctypes.c_void_p)]


NORM_BLOCK = 128


def _opts(n_sink=0, n_recent=0, form="auto", unfused=False, block_norms=None):
    f = FORMS[form] if isinstance(form, str) else int(form)
    if not n_sink and not n_recent and not f and not unfused and block_norms is None:
        return None
    if block_norms is not None:
        _cuda(block_norms)
    nb = None if block_norms is None else block_norms.data_ptr()
    return ctypes.byref(SelectOpts(int(n_sink), int(n_recent), f, 1 if unfused else 0, nb))


def block_norms(Kt, norms=None):
    """Screening bounds [B, Hkv, ceil(T_cap / 128)] fp32: the largest ||Kt[b,h,t,:]|| per block of 128 tokens."""
    _cuda(Kt, norms)
    B, Hkv, T_cap, r = Kt.shape
    if norms is None:
        norms = torch.empty((B, Hkv, (T_cap + NORM_BLOCK - 1) // NORM_BLOCK), dtype=torch.float32, device=Kt.device)
    dims = Dims(B, Hkv, Hkv, r, r, r, T_cap, BF16, _dt(Kt))
    _check(lib().jssa_block_norms(ctypes.byref(dims), _p(Kt), _p(norms), _stream(Kt.device)))
    return norms


def skip_count(ws: torch.Tensor) -> int:
    """Tiles the screening skipped (workspace word 1, cumulative); synchronises."""
    return int(ws[4:8].view(torch.int32).item()) & 0xFFFFFFFF


def plan_info(dims: Dims, k: int, op: int, agg: int = 0, form="auto", unfused=False):
    """(kernel launches per call, description of the forms chosen) for op."""
    n = ctypes.c_int32(0)
    buf = ctypes.create_string_buffer(160)
    _check(lib().jssa_plan_info_ex(ctypes.byref(dims), int(k), int(op), int(agg), _opts(0, 0, form, unfused),
                                   ctypes.byref(n), buf, 160))
    return int(n.value), buf.value.decode()


def workspace_size(dims: Dims, k: int, op: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().jssa_workspace_size(ctypes.byref(dims), int(k), int(op), ctypes.byref(n)))
    return int(n.value)


def new_workspace(dims: Dims, k: int, op: int, device) -> torch.Tensor:
    """Allocate (through torch) and zero a workspace for `op`."""
    n = max(workspace_size(dims, k, op), 256)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(lib().jssa_workspace_init(_p(ws), n, _stream(ws.device)))
    return ws


def workspace_init(ws: torch.Tensor):
    _check(lib().jssa_workspace_init(_p(ws), ws.numel(), _stream(ws.device)))


def device_status(ws: torch.Tensor) -> int:
    """Sticky device status word (JSSA_DEV_* bits); synchronises on the copy."""
    return int(ws[:4].view(torch.int32).item()) & 0xFFFFFFFF


def _ws(ws, dims, k, op, device):
    return new_workspace(dims, k, op, device) if ws is None else ws


# ------------------------------------------------------------------- ops ---
def append_lowrank(K, P, Kt, pos_begin, n_new, ws=None):
    """Kt[b,h,t,:] = round(K[b,t,h,:] @ P[h]) for t in [pos_begin[b], pos_begin[b] + n_new)."""
    _cuda(K, P, Kt, pos_begin)
    B, T_cap, Hkv, d = K.shape
    dims = Dims(B, 1 * Hkv, Hkv, d, 512 if d == 576 else d, P.shape[2], T_cap, _dt(K), _dt(Kt))
    ws = _ws(ws, dims, 1, OP_APPEND, K.device)
    _check(lib().jssa_append_lowrank(ctypes.byref(dims), _p(K), _p(P), _p(Kt), _p(pos_begin), int(n_new), _p(ws),
                                     ws.numel(), _stream(K.device)))
    return Kt


def build_lowrank_cache(K, P, kt_dtype=torch.bfloat16, ws=None):
    """Kt for all T_cap rows of K (prefix build)."""
    B, T_cap, Hkv, d = K.shape
    Kt = torch.empty((B, Hkv, T_cap, P.shape[2]), dtype=kt_dtype, device=K.device)
    pos = torch.zeros(B, dtype=torch.int32, device=K.device)
    return append_lowrank(K, P, Kt, pos, T_cap, ws=ws)


def score(q, P, Kt, seq_lens, agg=AGG_SUM, scores=None, ws=None):
    """Subspace scores [B, Hkv, T_cap] fp32 (t >= T_b not written)."""
    _cuda(q, P, Kt, seq_lens, scores)
    B, Hq, d = q.shape
    _, Hkv, T_cap, r = Kt.shape
    dims = Dims(B, Hq, Hkv, d, 512 if d == 576 else d, r, T_cap, _dt(q), _dt(Kt))
    if scores is None:
        scores = torch.full((B, Hkv, T_cap), float("nan"), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, 1, OP_SCORE, q.device)
    _check(lib().jssa_score(ctypes.byref(dims), _p(q), _p(P), _p(Kt), _p(seq_lens), int(agg), _p(scores), _p(ws),
                            ws.numel(), _stream(q.device)))
    return scores


def topk(scores, seq_lens, k, Hq=None, d=128, ws=None, n_sink=0, n_recent=0, form="auto"):
    """Per-(b,h) top-k of a score array: (idx [B,Hkv,k], count [B,Hkv]).
    n_sink / n_recent: always-selected first / last tokens; form: the selection
    form ("auto", "cluster", "stream", "scan"; jssa_select_opts)."""
    _cuda(scores, seq_lens)
    B, Hkv, T_cap = scores.shape
    dims = Dims(B, Hq or Hkv, Hkv, d, 512 if d == 576 else d, 8, T_cap, BF16, BF16)
    idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=scores.device)
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device=scores.device)
    ws = _ws(ws, dims, k, OP_TOPK, scores.device)
    _check(lib().jssa_topk_ex(ctypes.byref(dims), _p(scores), _p(seq_lens), int(k), _opts(n_sink, n_recent, form),
                              _p(idx), _p(cnt), _p(ws), ws.numel(), _stream(scores.device)))
    return idx, cnt


def select(q, P, Kt, seq_lens, k, agg=AGG_SUM, ws=None, idx=None, count=None, n_sink=0, n_recent=0, form="auto",
           block_norms=None):
    """Fused score + top-k: (idx [B,Hkv,k], count [B,Hkv]).
    n_sink / n_recent: always-selected first / last tokens; form: the selection
    form (jssa_select_opts)."""
    _cuda(q, P, Kt, seq_lens)
    B, Hq, d = q.shape
    _, Hkv, T_cap, r = Kt.shape
    dims = Dims(B, Hq, Hkv, d, 512 if d == 576 else d, r, T_cap, _dt(q), _dt(Kt))
    if idx is None:
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    ws = _ws(ws, dims, k, OP_SELECT, q.device)
    _check(lib().jssa_select_ex(ctypes.byref(dims), _p(q), _p(P), _p(Kt), _p(seq_lens), int(agg), int(k),
                                _opts(n_sink, n_recent, form, block_norms=block_norms), _p(idx), _p(count), _p(ws),
                                ws.numel(), _stream(q.device)))
    return idx, count


def select_heads(q, P, Kt, seq_lens, k, ws=None, idx=None, count=None, form="auto"):
    """Per-query-head selection (a variant for measurement): every query head g
    gets its own top-k over (P_h^T q_g) . Kt.  Returns (idx [B,Hq,k], count [B,Hq])."""
    _cuda(q, P, Kt, seq_lens)
    B, Hq, d = q.shape
    _, Hkv, T_cap, r = Kt.shape
    dims = Dims(B, Hq, Hkv, d, d, r, T_cap, _dt(q), _dt(Kt))
    if idx is None:
        idx = torch.empty((B, Hq, k), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
    ws = _ws(ws, dims, k, OP_SELECT_HEADS, q.device)
    _check(lib().jssa_select_heads(ctypes.byref(dims), _p(q), _p(P), _p(Kt), _p(seq_lens), int(k),
                                   _opts(0, 0, form), _p(idx), _p(count), _p(ws), ws.numel(), _stream(q.device)))
    return idx, count


def indexed_decode_heads(q, K, V, idx, count, seq_lens, scale, ws=None, out=None, lse=None):
    """Attention of each query head over its own list idx [B,Hq,k]: (out, lse)."""
    _cuda(q, K, V, idx, count, seq_lens, out, lse)
    k = idx.shape[2]
    dims = make_dims(q, K, V, r=8)
    if out is None:
        out = torch.empty((dims.B, dims.Hq, dims.dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, k, OP_INDEXED_DECODE_HEADS, q.device)
    _check(lib().jssa_indexed_decode_heads(ctypes.byref(dims), _p(q), _p(K), _p(V), _p(idx), _p(count), int(k),
                                           _p(seq_lens), float(scale), _p(out), _p(lse), _p(ws), ws.numel(),
                                           _stream(q.device)))
    return out, lse


def indexed_decode(q, K, V, idx, count, seq_lens, scale, ws=None, out=None, lse=None):
    """Gather-free attention over the selected rows: (out [B,Hq,dv], lse [B,Hq])."""
    _cuda(q, K, V, idx, count, seq_lens, out, lse)
    k = idx.shape[2]
    dims = make_dims(q, K, V, r=8)
    if out is None:
        out = torch.empty((dims.B, dims.Hq, dims.dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, k, OP_INDEXED_DECODE, q.device)
    _check(lib().jssa_indexed_decode(ctypes.byref(dims), _p(q), _p(K), _p(K if V is None else V), _p(idx),
                                     _p(count), int(k), _p(seq_lens), float(scale), _p(out), _p(lse), _p(ws),
                                     ws.numel(), _stream(q.device)))
    return out, lse


def dense_decode(q, K, V, seq_lens, scale, window=0, ws=None, out=None, lse=None):
    """Full-KV (window 0) or sliding-window decode attention: (out, lse)."""
    _cuda(q, K, V, seq_lens, out, lse)
    dims = make_dims(q, K, V, r=8)
    if out is None:
        out = torch.empty((dims.B, dims.Hq, dims.dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, 1, OP_DENSE_DECODE, q.device)
    _check(lib().jssa_dense_decode(ctypes.byref(dims), _p(q), _p(K), _p(K if V is None else V), _p(seq_lens),
                                   int(window), float(scale), _p(out), _p(lse), _p(ws), ws.numel(),
                                   _stream(q.device)))
    return out, lse


def gather_buffer_bytes(dims: Dims, k: int) -> int:
    """Bytes of the gather-then-dense buffer: K and V rows, or the latent rows
    once for a latent cache (V is K)."""
    copies = 1 if (dims.d == 576 and dims.dv == 512 and dims.Hkv == 1) else 2
    return copies * dims.B * dims.Hkv * k * dims.d * (2 if dims.kv_dtype == BF16 else 4)


def gather_then_dense(q, K, V, idx, count, seq_lens, scale, gather_buf=None, ws=None, out=None, lse=None):
    """Gather the selected rows into a contiguous buffer, then dense decode over them."""
    _cuda(q, K, V, idx, count, seq_lens, gather_buf, out, lse)
    k = idx.shape[2]
    dims = make_dims(q, K, V, r=8)
    if gather_buf is None:
        gather_buf = torch.empty(gather_buffer_bytes(dims, k), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((dims.B, dims.Hq, dims.dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, k, OP_GATHER_THEN_DENSE, q.device)
    _check(lib().jssa_gather_then_dense(ctypes.byref(dims), _p(q), _p(K), _p(K if V is None else V), _p(idx),
                                        _p(count), int(k), _p(seq_lens), float(scale), _p(gather_buf),
                                        gather_buf.numel() * gather_buf.element_size(), _p(out), _p(lse), _p(ws),
                                        ws.numel(), _stream(q.device)))
    return out, lse


def decode_step(q, K, V, P, Kt, seq_lens, pos_begin, k, scale, agg=AGG_SUM, ws=None, idx=None, count=None,
                out=None, lse=None, n_sink=0, n_recent=0, form="auto", unfused=False, block_norms=None):
    """Append the row at pos_begin, select, indexed decode: (out, lse, idx, count).
    n_sink / n_recent: always-selected first / last tokens; form: the selection
    form; unfused: keep the step in separate launches (jssa_select_opts)."""
    _cuda(q, K, V, P, Kt, seq_lens, pos_begin, idx, count, out, lse)
    dims = make_dims(q, K, V, P=P, Kt=Kt)
    B, Hkv = dims.B, dims.Hkv
    if idx is None:
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=q.device)
    if count is None:
        count = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty((B, dims.Hq, dims.dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, dims.Hq), dtype=torch.float32, device=q.device)
    ws = _ws(ws, dims, k, OP_DECODE_STEP, q.device)
    _check(lib().jssa_decode_step_ex(ctypes.byref(dims), _p(q), _p(K), _p(K if V is None else V), _p(P), _p(Kt),
                                     _p(seq_lens), _p(pos_begin), int(k), int(agg), float(scale),
                                     _opts(n_sink, n_recent, form, unfused, block_norms), _p(idx), _p(count), _p(out),
                                     _p(lse),
                                     _p(ws), ws.numel(), _stream(q.device)))
    return out, lse, idx, count


def calibrate_basis(q_cal, K, seq_lens, P_init, n_keys, iters=30, ws=None):
    """Calibrated basis [Hkv, d, r] fp32 (jssa_calibrate_basis): the dominant
    r-dim eigen-subspace of S_q/tr(S_q) + S_k/tr(S_k) per KV head, from the
    query rows q_cal [N, Hq, d] and n_keys sampled keys per batch row, by
    `iters` rounds of subspace iteration from P_init."""
    _cuda(q_cal, K, seq_lens, P_init)
    N, Hq, d = q_cal.shape
    B, T_cap, Hkv, _ = K.shape
    r = P_init.shape[2]
    dims = Dims(B, Hq, Hkv, d, d, r, T_cap, _dt(K), BF16)
    P_out = torch.empty_like(P_init)
    ws = _ws(ws, dims, 1, OP_CALIBRATE, K.device)
    _check(lib().jssa_calibrate_basis(ctypes.byref(dims), _p(q_cal), int(N), _p(K), _p(seq_lens), int(n_keys),
                                      int(iters), _p(P_init), _p(P_out), _p(ws), ws.numel(), _stream(K.device)))
    return P_out


def host_step_bytes(dims: Dims) -> int:
    """Bytes of the packed host input of decode_step_host: q [B,Hq,d], then the
    new K rows [B,Hkv,d], then the new V rows [B,Hkv,dv] (none for a latent cache)."""
    n = ctypes.c_size_t(0)
    _check(lib().jssa_host_step_bytes(ctypes.byref(dims), ctypes.byref(n)))
    return int(n.value)


def decode_step_host(in_host, stage, K, V, P, Kt, seq_lens, pos_begin, k, scale, out_host, ws, idx, count, out, lse,
                     agg=AGG_SUM, dims=None):
    """One step driven from (pinned) host memory through jssa_decode_step_host:
    in_host (uint8, host_step_bytes) is copied to the device buffer stage, the
    new K/V rows are written at pos_begin, the step runs, and out is copied to
    out_host.  Asynchronous: synchronise the stream before reading out_host."""
    _cuda(stage, K, V, P, Kt, seq_lens, pos_begin, ws, idx, count, out, lse)
    if dims is None:
        B, T_cap, Hkv, d = K.shape
        Hq = out.shape[1]
        dv = out.shape[2]
        dims = Dims(B, Hq, Hkv, d, dv, P.shape[2], T_cap, _dt(K), _dt(Kt))
    _check(lib().jssa_decode_step_host(ctypes.byref(dims), ctypes.c_void_p(in_host.data_ptr()), _p(stage), _p(K),
                                       _p(K if V is None else V), _p(P), _p(Kt), _p(seq_lens), _p(pos_begin), int(k),
                                       int(agg), float(scale), None, _p(idx), _p(count), _p(out), _p(lse),
                                       ctypes.c_void_p(out_host.data_ptr()), _p(ws), ws.numel(), _stream(K.device)))
    return out_host


class StepGraph:
    """A call sequence on fixed device buffers (e.g. one jssa_decode_step)
    captured in a CUDA graph: replay() re-launches the same kernels without
    host planning or argument marshalling.  The buffers the calls use must
    stay alive and are updated in place between replays.  One call runs
    before the capture (on a side stream) so that every plan is made and
    cached outside it."""

    def __init__(self, fn, device):
        self.fn = fn
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            fn()

    def replay(self):
        self.graph.replay()


class DecodeSession:
    """Device-resident state of one attention layer's decode (the public API
    of the end-to-end path): KV cache, low-rank key cache, basis, workspace
    and output buffers.  ``step_from_host`` takes one step's inputs from
    pinned host memory and returns the attention output in pinned host
    memory."""

    def __init__(self, K, V, P, seq_lens, k, scale, Kt=None, kt_dtype=torch.bfloat16, agg=AGG_SUM):
        _cuda(K, V, P, seq_lens)
        self.K, self.V, self.P, self.seq_lens = K, V, P, seq_lens  # V None: latent cache
        self.k, self.scale, self.agg = int(k), float(scale), int(agg)
        dev = K.device
        self.Kt = build_lowrank_cache(K, P, kt_dtype) if Kt is None else Kt
        B, T_cap, Hkv, d = K.shape
        self.B, self.Hkv, self.d = B, Hkv, d
        self.pos = (seq_lens.to(torch.int32) - 1).clamp_min(0).contiguous()
        self._dims = None
        self.ws = None
        self.q_dev = None
        self.out = self.lse = self.idx = self.count = None

    def _ensure(self, q_shape, dtype):
        if self.q_dev is not None and tuple(self.q_dev.shape) == tuple(q_shape):
            return
        dev = self.K.device
        self.q_dev = torch.empty(q_shape, dtype=dtype, device=dev)
        dims = make_dims(self.q_dev, self.K, self.V, P=self.P, Kt=self.Kt)
        self.ws = new_workspace(dims, self.k, OP_DECODE_STEP, dev)
        self.idx = torch.empty((self.B, self.Hkv, self.k), dtype=torch.int32, device=dev)
        self.count = torch.empty((self.B, self.Hkv), dtype=torch.int32, device=dev)
        self.out = torch.empty((dims.B, dims.Hq, dims.dv), dtype=dtype, device=dev)
        self.lse = torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=dev)
        self.out_host = torch.empty(self.out.shape, dtype=dtype, pin_memory=True)

    def step(self, q):
        """One step on a device-resident query (the new token's K/V row must
        already be at position seq_lens-1 of the cache)."""
        out, lse, idx, count = decode_step(q, self.K, self.V, self.P, self.Kt, self.seq_lens, self.pos, self.k,
                                           self.scale, agg=self.agg, ws=self.ws, idx=self.idx, count=self.count,
                                           out=self.out, lse=self.lse)
        return out

    def step_from_host(self, q_host, k_new_host, v_new_host, graph=False):
        """Copy q [B,Hq,d] and the new token's K/V rows [B,Hkv,d] from pinned host
        memory, write the rows at position seq_lens-1, run the step, and copy the
        output back to pinned host memory (returned; valid after a stream sync).
        graph=True replays the step from a CUDA graph captured on first use."""
        self._ensure(q_host.shape, q_host.dtype)
        self.q_dev.copy_(q_host, non_blocking=True)
        pos = int(self._host_pos())
        self.K[:, pos].copy_(k_new_host, non_blocking=True)
        if self.V is not None:
            self.V[:, pos].copy_(v_new_host, non_blocking=True)
        if graph:
            if getattr(self, "_graph", None) is None:
                self._graph = StepGraph(lambda: self.step(self.q_dev), self.K.device)
            self._graph.replay()
        else:
            self.step(self.q_dev)
        self.out_host.copy_(self.out, non_blocking=True)
        return self.out_host

    def _host_pos(self):
        if not hasattr(self, "_pos_cache"):
            p = self.pos.cpu()
            if not bool((p == p[0]).all()):
                raise ValueError("step_from_host needs one shared position across the batch")
            self._pos_cache = int(p[0])
        return self._pos_cache


class DecodeLoop:
    """Multi-layer, multi-step decode of an attention stack (the loop around
    the hot path): each step runs jssa_decode_step on every layer in turn,
    layer l + 1 taking layer l's output as its query (d == dv), then advances
    the shared sequence position on the device (seq_lens += 1, pos += 1).
    The new token's K/V rows are expected at position pos of each layer's
    cache before a step (a model writes them; this loop does not).

    layers: list of (K, V, P, Kt) per layer, all of one shape; seq_lens,
    pos: [B] int32 device tensors shared by the layers (advanced in place).
    step() runs eagerly; capture() records one whole step (every layer and
    the position advance) as a CUDA graph, replayed by step(graph=True)."""

    def __init__(self, layers, seq_lens, pos, k, scale, agg=AGG_SUM):
        if not layers:
            raise ValueError("DecodeLoop needs at least one layer")
        self.layers = layers
        self.seq_lens, self.pos = seq_lens, pos
        self.k, self.scale, self.agg = int(k), float(scale), int(agg)
        K0, V0, P0, Kt0 = layers[0]
        B, T_cap, Hkv, d = K0.shape
        self.T_cap = T_cap
        self._graph = None
        self.q = None

    def _ensure(self, q):
        if self.q is not None and tuple(self.q.shape) == tuple(q.shape):
            return
        K0, V0, P0, Kt0 = self.layers[0]
        dims = make_dims(q, K0, V0, P=P0, Kt=Kt0)
        if dims.dv != dims.d:
            raise ValueError("a chained stack needs dv == d")
        dev = q.device
        self.q = torch.empty_like(q)
        self.ws = new_workspace(dims, self.k, OP_DECODE_STEP, dev)
        self.idx = [torch.empty((dims.B, dims.Hkv, self.k), dtype=torch.int32, device=dev) for _ in self.layers]
        self.count = [torch.empty((dims.B, dims.Hkv), dtype=torch.int32, device=dev) for _ in self.layers]
        self.out = [torch.empty((dims.B, dims.Hq, dims.dv), dtype=q.dtype, device=dev) for _ in self.layers]
        self.lse = [torch.empty((dims.B, dims.Hq), dtype=torch.float32, device=dev) for _ in self.layers]

    def _run(self):
        x = self.q
        for l, (K, V, P, Kt) in enumerate(self.layers):
            decode_step(x, K, V, P, Kt, self.seq_lens, self.pos, self.k, self.scale, agg=self.agg, ws=self.ws,
                        idx=self.idx[l], count=self.count[l], out=self.out[l], lse=self.lse[l])
            x = self.out[l]
        self.seq_lens.add_(1)
        self.pos.add_(1)

    def set_query(self, q):
        """Copy the first layer's query for the next step (device tensor)."""
        self._ensure(q)
        self.q.copy_(q)

    def capture(self):
        """Record one whole step as a CUDA graph (runs one eager step first, on
        a side stream, which also advances the position once)."""
        if self.q is None:
            raise RuntimeError("set_query() before capture()")
        self._graph = StepGraph(self._run, self.q.device)
        return self._graph

    def step(self, graph=False):
        """One decode step of the whole stack; returns the last layer's output."""
        if graph:
            if self._graph is None:
                self.capture()
            self._graph.replay()
        else:
            self._run()
        return self.out[-1]

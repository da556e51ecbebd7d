"""JSSA decode-step oracle: fp64 CPU reference (TEST INFRASTRUCTURE ONLY).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls anything here, and this
package imports nothing from the product.

The arithmetic lives in ``jssa_oracle.c`` (plain C, fp64, OpenMP over the
(batch, KV head) pairs); this module only marshals numpy / torch-CPU buffers
through ctypes.  ``brute.py`` holds pure-Python brute force for tiny inputs.

Method pages (cited by title and section in the C source):
  "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Abstract;
  "JSSA makes token-level sparse decoding gather-free ..." (news item),
  Synopsis / Interpretation / Perspective.

Layouts (row-major):
  q   [B, Hq, d]            K, V [B, T_cap, Hkv, d]      P [Hkv, d, r] fp32
  Kt  [B, Hkv, T_cap, r]    scores [B, Hkv, T_cap]       idx [B, Hkv, k]
  out [B, Hq, dv]           lse [B, Hq]
bf16 buffers are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "jssa_oracle.c")
_SO = os.path.join(_HERE, "libjssa_oracle.so")

BF16, FP32 = 0, 1
AGG_SUM, AGG_MAX = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libjssa_oracle.so`` with gcc."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_round_bf16.restype = dbl
        L.oracle_round_bf16.argtypes = [dbl]
        L.oracle_append_lowrank.restype = i32
        L.oracle_append_lowrank.argtypes = [i32] * 5 + [vp, i32, vp, vp, i32, vp, i32, vp]
        L.oracle_score.restype = i32
        L.oracle_score.argtypes = [i32] * 6 + [vp, i32, vp, vp, i32, vp, i32, vp, i32, vp]
        L.oracle_topk.restype = i32
        L.oracle_topk.argtypes = [i32, i32, i32, vp, vp, i32, vp, i32, vp, vp]
        L.oracle_topk_forced.restype = i32
        L.oracle_topk_forced.argtypes = [i32, i32, i32, vp, vp, i32, i32, i32, vp, i32, vp, vp]
        L.oracle_attend.restype = i32
        L.oracle_attend.argtypes = [i32] * 6 + [vp, i32, vp, vp, i32, i32, vp, vp, i32, vp, dbl, vp, i32, vp, vp]
        L.oracle_score_heads.restype = i32
        L.oracle_score_heads.argtypes = [i32] * 6 + [vp, i32, vp, vp, i32, vp, vp, i32, vp]
        L.oracle_attend_heads.restype = i32
        L.oracle_attend_heads.argtypes = [i32] * 6 + [vp, i32, vp, vp, i32, i32, vp, vp, i32, vp, dbl, vp, i32, vp, vp]
        L.oracle_dense.restype = i32
        L.oracle_dense.argtypes = [i32] * 6 + [vp, i32, vp, vp, i32, i32, vp, i32, dbl, vp, i32, vp, vp]
        _lib = L
    return _lib


def set_threads(n: int | None) -> None:
    """OpenMP thread count used by the oracle (None = library default)."""
    if n is not None:
        os.environ["OMP_NUM_THREADS"] = str(int(n))
        try:
            ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
        except OSError:
            pass


# ----------------------------------------------------------------- marshalling
def raw(x):
    """Return (contiguous numpy array, dtype code) for a bf16/fp32 buffer.

    Accepts torch CPU tensors (bf16 -> uint16 bit view) or numpy arrays
    (uint16 = bf16 bits, float32)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous().cpu()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)), BF16
            if x.dtype == torch.float32:
                return np.ascontiguousarray(x.numpy()), FP32
            raise TypeError("oracle buffers are bf16 or fp32, got %s" % x.dtype)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, FP32
    raise TypeError("oracle buffers are bf16 bits (uint16) or float32, got %s" % x.dtype)


def _i32(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _f32(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _bh(bh_list):
    if bh_list is None:
        return None, 0
    a = _i32(bh_list).reshape(-1)
    return a, int(a.size)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(x) -> np.ndarray:
    a, code = raw(x)
    return bf16_bits_to_f64(a) if code == BF16 else a.astype(np.float64)


# ------------------------------------------------------------------ functions
def round_bf16(x: float) -> float:
    """Single round-to-nearest-even of a double onto the bf16 grid."""
    return float(lib().oracle_round_bf16(float(x)))


def append_lowrank(K, P, pos_begin, n_new, kt_dtype=BF16, Kt=None, want_exact=False):
    """Kt[b,h,t,:] = round(K[b,t,h,:] @ P[h]) for t in [pos_begin[b], pos_begin[b]+n_new).

    Kt (optional) is updated in place (numpy, uint16 bits or float32) and
    returned; a new zero array of shape [B,Hkv,T_cap,r] is made otherwise."""
    Kr, kcode = raw(K)
    B, T_cap, Hkv, d = Kr.shape
    Pf = _f32(P)
    r = Pf.shape[2]
    pos = _i32(pos_begin)
    if Kt is None:
        Kt = np.zeros((B, Hkv, T_cap, r), dtype=np.uint16 if kt_dtype == BF16 else np.float32)
    else:
        Kt, code = raw(Kt)
        assert code == kt_dtype
    exact = np.zeros(Kt.shape, dtype=np.float64) if want_exact else None
    rc = lib().oracle_append_lowrank(B, T_cap, Hkv, d, r, _p(Kr), kcode, _p(Pf), _p(pos), int(n_new),
                                     _p(Kt), kt_dtype, _p(exact))
    if rc != 0:
        raise ValueError("oracle_append_lowrank: bad arguments (rc=%d)" % rc)
    return (Kt, exact) if want_exact else Kt


def score(q, P, Kt, seq_lens, agg=AGG_SUM, bh_list=None):
    """Subspace scores s[b,h,t] (fp64); t >= T_b holds -inf."""
    qr, qcode = raw(q)
    B, Hq, d = qr.shape
    Pf = _f32(P)
    Hkv, _, r = Pf.shape
    Ktr, ktcode = raw(Kt)
    T_cap = Ktr.shape[2]
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    out = np.full((B, Hkv, T_cap), -np.inf, dtype=np.float64)
    rc = lib().oracle_score(B, Hq, Hkv, d, r, T_cap, _p(qr), qcode, _p(Pf), _p(Ktr), ktcode, _p(sl),
                            int(agg), _p(bh), nbh, _p(out))
    if rc != 0:
        raise ValueError("oracle_score: bad arguments (rc=%d)" % rc)
    return out


def topk(scores, seq_lens, k, bh_list=None, n_sink=0, n_recent=0):
    """Per-(b,h) top-k by (score desc, index asc); ascending indices, -1 padded.
    n_sink / n_recent: tokens [0, n_sink) and [T_b - n_recent, T_b) are always
    selected (smallest indices first when they alone exceed k_b)."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    B, Hkv, T_cap = s.shape
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    idx = np.full((B, Hkv, k), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    if n_sink or n_recent:
        rc = lib().oracle_topk_forced(B, Hkv, T_cap, _p(s), _p(sl), int(k), int(n_sink), int(n_recent), _p(bh), nbh,
                                      _p(idx), _p(cnt))
    else:
        rc = lib().oracle_topk(B, Hkv, T_cap, _p(s), _p(sl), int(k), _p(bh), nbh, _p(idx), _p(cnt))
    if rc != 0:
        raise ValueError("oracle_topk: bad arguments (rc=%d)" % rc)
    return idx, cnt


def attend(q, K, V, idx, count, seq_lens, scale, dv=None, bh_list=None, v_aliases_k=False):
    """Attention over per-(b,h) index lists.  Returns (out [B,Hq,dv], lse [B,Hq]) fp64.

    v_aliases_k: V is the latent cache itself (V row = first dv dims of the K row)."""
    qr, qcode = raw(q)
    B, Hq, d = qr.shape
    Kr, kvcode = raw(K)
    _, T_cap, Hkv, _ = Kr.shape
    if v_aliases_k:
        Vr, v_ld = Kr, d
        dv = d if dv is None else dv
    else:
        Vr, vcode = raw(V)
        assert vcode == kvcode
        v_ld = Vr.shape[3]
        dv = v_ld if dv is None else dv
    ix = _i32(idx)
    k = ix.shape[2]
    cn = _i32(count)
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    lse = np.full((B, Hq), np.nan, dtype=np.float64)
    rc = lib().oracle_attend(B, Hq, Hkv, d, dv, T_cap, _p(qr), qcode, _p(Kr), _p(Vr), kvcode, v_ld,
                             _p(ix), _p(cn), k, _p(sl), float(scale), _p(bh), nbh, _p(out), _p(lse))
    if rc == -2:
        raise ValueError("oracle_attend: an index lies outside [0, T_b) or a count outside [0, k]")
    if rc != 0:
        raise ValueError("oracle_attend: bad arguments (rc=%d)" % rc)
    return out, lse


def score_heads(q, P, Kt, seq_lens, bh_list=None):
    """Per-query-head subspace scores s[b,g,t] (fp64) [B, Hq, T_cap]; t >= T_b
    holds -inf.  bh_list lists flattened (b*Hq + g) rows."""
    qr, qcode = raw(q)
    B, Hq, d = qr.shape
    Pf = _f32(P)
    Hkv, _, r = Pf.shape
    Ktr, ktcode = raw(Kt)
    T_cap = Ktr.shape[2]
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    out = np.full((B, Hq, T_cap), -np.inf, dtype=np.float64)
    rc = lib().oracle_score_heads(B, Hq, Hkv, d, r, T_cap, _p(qr), qcode, _p(Pf), _p(Ktr), ktcode, _p(sl), _p(bh),
                                  nbh, _p(out))
    if rc != 0:
        raise ValueError("oracle_score_heads: bad arguments (rc=%d)" % rc)
    return out


def attend_heads(q, K, V, idx, count, seq_lens, scale, bh_list=None):
    """Attention of each query head over its own list: idx [B, Hq, k], count
    [B, Hq].  Returns (out [B,Hq,dv], lse [B,Hq]) fp64."""
    qr, qcode = raw(q)
    B, Hq, d = qr.shape
    Kr, kvcode = raw(K)
    _, T_cap, Hkv, _ = Kr.shape
    Vr, vcode = raw(V)
    assert vcode == kvcode
    dv = v_ld = Vr.shape[3]
    ix = _i32(idx)
    k = ix.shape[2]
    cn = _i32(count)
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    lse = np.full((B, Hq), np.nan, dtype=np.float64)
    rc = lib().oracle_attend_heads(B, Hq, Hkv, d, dv, T_cap, _p(qr), qcode, _p(Kr), _p(Vr), kvcode, v_ld, _p(ix),
                                   _p(cn), k, _p(sl), float(scale), _p(bh), nbh, _p(out), _p(lse))
    if rc == -2:
        raise ValueError("oracle_attend_heads: an index lies outside [0, T_b) or a count outside [0, k]")
    if rc != 0:
        raise ValueError("oracle_attend_heads: bad arguments (rc=%d)" % rc)
    return out, lse


def dense(q, K, V, seq_lens, scale, window=0, dv=None, bh_list=None, v_aliases_k=False):
    """Full-KV (window = 0) or sliding-window attention.  Returns (out, lse) fp64."""
    qr, qcode = raw(q)
    B, Hq, d = qr.shape
    Kr, kvcode = raw(K)
    _, T_cap, Hkv, _ = Kr.shape
    if v_aliases_k:
        Vr, v_ld = Kr, d
        dv = d if dv is None else dv
    else:
        Vr, vcode = raw(V)
        assert vcode == kvcode
        v_ld = Vr.shape[3]
        dv = v_ld if dv is None else dv
    sl = _i32(seq_lens)
    bh, nbh = _bh(bh_list)
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    lse = np.full((B, Hq), np.nan, dtype=np.float64)
    rc = lib().oracle_dense(B, Hq, Hkv, d, dv, T_cap, _p(qr), qcode, _p(Kr), _p(Vr), kvcode, v_ld,
                            _p(sl), int(window), float(scale), _p(bh), nbh, _p(out), _p(lse))
    if rc != 0:
        raise ValueError("oracle_dense: bad arguments (rc=%d)" % rc)
    return out, lse


def step(q, K, V, P, Kt, seq_lens, k, scale, pos_begin=None, n_new=1, agg=AGG_SUM, dv=None,
         bh_list=None, v_aliases_k=False, kt_dtype=None, n_sink=0, n_recent=0):
    """One decode step: append n_new rows at pos_begin, score, select, attend.

    Kt (numpy bits / fp32, or torch CPU tensor) holds the prefix low-rank cache and
    is updated in place on a copy, which is returned with the rest:
    (Kt, scores, idx, count, out, lse)."""
    Ktr, code = raw(Kt)
    Ktr = Ktr.copy()
    if kt_dtype is not None:
        assert code == kt_dtype
    if pos_begin is not None and n_new > 0:
        Ktr = append_lowrank(K, P, pos_begin, n_new, kt_dtype=code, Kt=Ktr)
    s = score(q, P, Ktr, seq_lens, agg=agg, bh_list=bh_list)
    idx, cnt = topk(s, seq_lens, k, bh_list=bh_list, n_sink=n_sink, n_recent=n_recent)
    out, lse = attend(q, K, V, idx, cnt, seq_lens, scale, dv=dv, bh_list=bh_list, v_aliases_k=v_aliases_k)
    return Ktr, s, idx, cnt, out, lse


def default_scale(d: int) -> float:
    """Softmax scale used by the synthetic workloads: 1/sqrt(d)."""
    return 1.0 / math.sqrt(d)

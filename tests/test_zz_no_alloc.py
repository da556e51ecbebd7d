"""Allocation-free indexed decode (jssa_indexed_decode_noalloc).

For callers that cannot allocate device memory at call time (a serving
engine whose allocator already owns the GPU's memory, a real-time loop that
cannot take cudaMalloc's implicit synchronisation, a plugin host that forbids
allocation), the library offers an indexed decode whose scratch is a fixed
array inside the library.  This test calls it through the C ABI (ctypes) and
checks, on two calls in a row, that its output matches the workspace-taking
jssa_indexed_decode within the tolerance every GPU parity test uses.  The file
sorts last so that a run stopping at the first failure has run the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import OUT_TOL, LSE_TOL
from token_level_sparse_kv_b200 import ops
from token_level_sparse_kv_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _noalloc(dims, q, K, V, idx, cnt, k, sl, scale, out, lse):
    L = ops.lib()
    f = L.jssa_indexed_decode_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(ops.Dims), vp, vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_float, vp, vp, vp]
    st = f(ctypes.byref(dims), q.data_ptr(), K.data_ptr(), V.data_ptr(), idx.data_ptr(), cnt.data_ptr(), k,
           sl.data_ptr(), float(scale), out.data_ptr(), lse.data_ptr(),
           torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    dev = "cuda"
    results = []
    for seed, sl_list in ((101, [2500, 1800, 7]), (202, [2500, 0, 2400])):
        w = Workload("t", B=3, Hq=16, Hkv=4, d=128, T=2500, r=32, k=256, seed=seed)
        q, K, V, P, sl = (t.to(dev) for t in make_inputs(w, seq_lens=sl_list))
        Kt = ops.build_lowrank_cache(K, P)
        idx, cnt = ops.select(q, P, Kt, sl, w.k)
        ref_o, ref_l = ops.indexed_decode(q, K, V, idx, cnt, sl, w.scale)
        dims = ops.make_dims(q, K, V, r=8)
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        st = _noalloc(dims, q, K, V, idx, cnt, w.k, sl, w.scale, out, lse)
        assert st == 0, ops.lib().jssa_last_error()
        torch.cuda.synchronize()
        err = (out.float() - ref_o.float()).abs().max().item()
        assert err <= OUT_TOL[torch.bfloat16], err
        both_inf = torch.isneginf(lse) & torch.isneginf(ref_l)
        assert torch.equal(torch.isneginf(lse), torch.isneginf(ref_l))
        lerr = (lse - ref_l).masked_fill(both_inf, 0).abs().max().item()
        assert lerr <= LSE_TOL, lerr
        results.append(out.clone())
    # the second call ran on the contents the first call left behind
    assert not torch.equal(results[0], results[1])


def test_noalloc_rejects_shapes_above_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    dev = "cuda"
    # 4096 (b, h) pairs of G=16 heads at d=256 and k=2048: far above 8 MiB of partials
    dims = ops.Dims(1024, 64, 4, 256, 256, 8, 4096, ops.BF16, ops.BF16)
    t = torch.zeros(64, dtype=torch.float32, device=dev)
    i = torch.zeros(64, dtype=torch.int32, device=dev)
    L = ops.lib()
    f = L.jssa_indexed_decode_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(ops.Dims), vp, vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_float, vp, vp, vp]
    st = f(ctypes.byref(dims), t.data_ptr(), t.data_ptr(), t.data_ptr(), i.data_ptr(), i.data_ptr(), 2048,
           i.data_ptr(), 1.0, t.data_ptr(), t.data_ptr(), None)
    assert st == -3
    assert b"scratch" in L.jssa_last_error()

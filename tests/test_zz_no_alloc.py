"""Allocation-free indexed decode (jssa_indexed_decode_noalloc).

Some callers cannot hand the library device scratch memory because they
cannot allocate at call time: a serving engine whose allocator already owns
the GPU's memory for its KV-cache pool, a real-time decode loop that cannot
take the implicit device synchronisation of cudaMalloc / cudaFree, or a
plugin host that forbids allocation inside its hooks.  For them the library
offers an indexed decode whose scratch is a fixed array inside the library.

These tests call it through the C ABI (ctypes) and check, on two calls in a
row, that its output matches the workspace-taking jssa_indexed_decode and the
fp64 oracle within the tolerance every GPU parity test uses; that a repeat
call on the same inputs gives bit-identical results (the state the first call
leaves in the shared array does not leak into the next); that NULL count and
NULL lse behave as in jssa_indexed_decode; and that a latent-cache shape is
served too.  The file sorts last so that a run stopping at the first failure
has run the rest.
"""
import ctypes

import pytest
import torch

import oracle
from parity import check_attention, host
from token_level_sparse_kv_b200 import ops
from token_level_sparse_kv_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _fn():
    f = ops.lib().jssa_indexed_decode_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(ops.Dims), vp, vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_float, vp, vp, vp]
    return f


def _ptr(t):
    return None if t is None else t.data_ptr()


def _noalloc(dims, q, K, V, idx, cnt, k, sl, scale, out, lse):
    return _fn()(ctypes.byref(dims), _ptr(q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cnt), k, _ptr(sl), float(scale),
                 _ptr(out), _ptr(lse), torch.cuda.current_stream().cuda_stream)


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")


def _case(w, sl_list, latent=False):
    """Inputs on the device, a selection by the library, and the reference
    results of jssa_indexed_decode (workspace entry point) on them."""
    q, K, V, P, sl = make_inputs(w, seq_lens=sl_list)
    qd, Kd, Pd, sld = (t.to("cuda") for t in (q, K, P, sl))
    Vd = None if V is None else V.to("cuda")
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    return (q, K, V, sl), (qd, Kd, Vd, sld), idx, cnt


def test_noalloc_matches_workspace_entry_point_and_oracle_twice():
    _need_gpu()
    w = Workload("t", B=3, Hq=16, Hkv=4, d=128, T=2500, r=32, k=256, seed=101)
    (q, K, V, sl), (qd, Kd, Vd, sld), idx, cnt = _case(w, [2500, 1800, 7])
    ref_o, ref_l = ops.indexed_decode(qd, Kd, Vd, idx, cnt, sld, w.scale)
    or_o, or_l = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    dims = ops.make_dims(qd, Kd, Vd, r=8)
    outs = []
    for _ in range(2):  # two calls in a row on one shared scratch array
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        st = _noalloc(dims, qd, Kd, Vd, idx, cnt, w.k, sld, w.scale, out, lse)
        assert st == 0, ops.lib().jssa_last_error()
        torch.cuda.synchronize()
        check_attention(out, lse, or_o, or_l, torch.bfloat16)
        check_attention(out, lse, ref_o.double().cpu().numpy(), ref_l.double().cpu().numpy(), torch.bfloat16)
        outs.append((out.clone(), lse.clone()))
    # the second call ran on what the first left in the array: same bits
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1].nan_to_num(), outs[1][1].nan_to_num())


def test_noalloc_null_count_and_lse():
    _need_gpu()
    w = Workload("t", B=2, Hq=8, Hkv=2, d=128, T=1200, r=32, k=128, seed=303)
    (q, K, V, sl), (qd, Kd, Vd, sld), idx, cnt = _case(w, [1200, 90])
    ref_o, _ = ops.indexed_decode(qd, Kd, Vd, idx, None, sld, w.scale)
    dims = ops.make_dims(qd, Kd, Vd, r=8)
    out = torch.full_like(ref_o, float("nan"))
    st = _noalloc(dims, qd, Kd, Vd, idx, None, w.k, sld, w.scale, out, None)
    assert st == 0, ops.lib().jssa_last_error()
    torch.cuda.synchronize()
    # count = NULL: the count is the number of leading non-negative slots
    or_o, _ = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    check_attention(out, None, or_o, None, torch.bfloat16)
    assert (out.float() - ref_o.float()).abs().max().item() <= 2e-2


def test_noalloc_latent_cache_shape():
    _need_gpu()
    w = Workload("mla", B=1, Hq=128, Hkv=1, d=576, dv=512, T=3000, r=64, k=256, latent=True, seed=404)
    (q, K, V, sl), (qd, Kd, Vd, sld), idx, cnt = _case(w, [3000])
    assert Vd is None
    ref_o, ref_l = ops.indexed_decode(qd, Kd, None, idx, cnt, sld, w.scale)
    or_o, or_l = oracle.attend(q, K, None, host(idx), host(cnt), sl, w.scale, dv=512, v_aliases_k=True)
    dims = ops.make_dims(qd, Kd, None, r=8)
    outs = []
    for _ in range(2):
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        st = _noalloc(dims, qd, Kd, Kd, idx, cnt, w.k, sld, w.scale, out, lse)
        assert st == 0, ops.lib().jssa_last_error()
        torch.cuda.synchronize()
        check_attention(out, lse, or_o, or_l, torch.bfloat16)
        assert (out.float() - ref_o.float()).abs().max().item() <= 2e-2
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])


def test_noalloc_rejects_shapes_above_its_scratch():
    _need_gpu()
    # 4096 (b, h) pairs of G=16 heads at d=256 and k=2048: far above 8 MiB of partials
    dims = ops.Dims(1024, 64, 4, 256, 256, 8, 4096, ops.BF16, ops.BF16)
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    i = torch.zeros(64, dtype=torch.int32, device="cuda")
    st = _fn()(ctypes.byref(dims), t.data_ptr(), t.data_ptr(), t.data_ptr(), i.data_ptr(), i.data_ptr(), 2048,
               i.data_ptr(), 1.0, t.data_ptr(), t.data_ptr(), None)
    assert st == -3
    assert b"scratch" in ops.lib().jssa_last_error()

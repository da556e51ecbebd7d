"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Every case draws seeded inputs (token_level_sparse_kv_b200.inputs), runs the
kernels through ops.* (ctypes -> libjssa.so) and compares with oracle.*
under the rules in tests/parity.py.  Stage-isolated checks feed the oracle the
GPU's own upstream result (its low-rank cache, its scores, its indices), so a
near-tie resolved differently upstream cannot leak downstream.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_append, check_attention, check_end_to_end, check_scores, check_selection, host
from token_level_sparse_kv_b200 import ops
from token_level_sparse_kv_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests selected but no CUDA device is visible")
    ops.lib()


def W(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=1500, r=32, k=64, kind="spiked", seed=11)
    base.update(kw)
    return Workload(**base)


def draw(w, dtype=torch.bfloat16, seq_lens=None):
    q, K, V, P, sl = make_inputs(w, device="cpu", dtype=dtype, seq_lens=seq_lens)
    dev = lambda t: None if t is None else t.to(DEV).contiguous()
    return (q, K, V, P, sl), (dev(q), dev(K), dev(V), dev(P), dev(sl))


def score_scale(q, P, Kt_host, G, agg):
    """sum_j (sum_i |q_i| |P_ij|) |Kt_j| per (b,h,t): the size of the terms of a score."""
    qa = np.abs(oracle.to_f64(q))
    B, Hq, d = qa.shape
    Hkv = Hq // G
    qa = qa.reshape(B, Hkv, G, d).sum(2)
    pa = np.abs(P.to(torch.float64).numpy())
    qp = np.einsum("bhi,hij->bhj", qa, pa)
    return np.einsum("bhj,bhtj->bht", qp, np.abs(oracle.to_f64(Kt_host)))


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("d,r,Hkv,kt", [(128, 32, 2, torch.bfloat16), (128, 32, 2, torch.float32),
                                        (256, 64, 2, torch.bfloat16), (64, 8, 3, torch.bfloat16),
                                        (576, 64, 1, torch.bfloat16)])
def test_append_prefix_and_step(d, r, Hkv, kt):
    w = W(d=d, r=r, Hkv=Hkv, Hq=Hkv * 2, T=333, dv=512 if d == 576 else None, latent=d == 576)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    Kt = ops.build_lowrank_cache(Kd, Pd, kt_dtype=kt)
    torch.cuda.synchronize()
    check_append(Kt, K, P, [0] * w.B, w.T)
    # per-step append at a different position per batch row; rows elsewhere untouched
    before = Kt.clone()
    K2 = K.clone()
    pos = [5, 300][: w.B]
    for b, p in enumerate(pos):
        K2[b, p] = torch.randn(K2[b, p].shape, generator=torch.Generator().manual_seed(b)).to(K2.dtype)
    Kd.copy_(K2.to(DEV))
    ops.append_lowrank(Kd, Pd, Kt, torch.tensor(pos, dtype=torch.int32, device=DEV), 1)
    torch.cuda.synchronize()
    check_append(Kt, K2, P, pos, 1)
    changed = (Kt != before).reshape(w.B, Hkv, w.T, -1).any(-1).cpu()
    for b in range(w.B):
        rows = torch.nonzero(changed[b].any(0)).flatten().tolist()
        assert set(rows) <= {pos[b]}


# ------------------------------------------------------------------- score
@pytest.mark.parametrize("agg", [ops.AGG_SUM, ops.AGG_MAX])
@pytest.mark.parametrize("kt", [torch.bfloat16, torch.float32])
def test_score_parity(agg, kt):
    w = W(T=2049, Hq=8, Hkv=2)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[2049, 700])
    Kt = ops.build_lowrank_cache(Kd, Pd, kt_dtype=kt)
    s = ops.score(qd, Pd, Kt, sld, agg=agg)
    torch.cuda.synchronize()
    Kt_h = host(Kt)
    ref = oracle.score(q, P, Kt_h, sl, agg=agg)
    sg = host(s).numpy()
    check_scores(sg, ref, score_scale(q, P, Kt_h, w.G, agg))
    assert np.all(np.isnan(sg[1, :, 700:])), "entries past T_b were written"


# Every selection form (one cluster per (b,h) holding its keys in shared
# memory; the warp-specialised streaming pass; the block-synchronous streaming
# pass) must return the same indices; jssa_select_opts.form forces one.
FORMS = ["auto", "cluster", "stream", "scan"]


@pytest.fixture(params=FORMS)
def form(request):
    return request.param


# -------------------------------------------------------------------- topk
def test_topk_is_exact_on_the_same_scores(form):
    w = W(B=3, Hkv=2, Hq=4, T=9000)
    g = torch.Generator().manual_seed(3)
    s = torch.randn(w.B, w.Hkv, w.T, generator=g)
    s[0, 0, 100:4000] = torch.round(s[0, 0, 100:4000] * 4) / 4  # heavy exact ties
    s[1, 1, :] = 0.0
    s[1, 1, ::3] = -0.0  # -0.0 and +0.0 are one value
    s[2, 0, 10:20] = 1e30
    sl = torch.tensor([9000, 8999, 300], dtype=torch.int32)
    for k in (1, 64, 300, 2048):
        idx, cnt = ops.topk(s.to(DEV), sl.to(DEV), k, form=form)
        torch.cuda.synchronize()
        ref_idx, ref_cnt = oracle.topk(s.double().numpy(), sl, k)
        np.testing.assert_array_equal(host(idx).numpy(), ref_idx)
        np.testing.assert_array_equal(host(cnt).numpy(), ref_cnt)


def test_topk_ragged_and_empty(form):
    g = torch.Generator().manual_seed(4)
    s = torch.randn(4, 1, 5000, generator=g)
    sl = torch.tensor([0, 1, 255, 5000], dtype=torch.int32)
    idx, cnt = ops.topk(s.to(DEV), sl.to(DEV), 256, form=form)
    torch.cuda.synchronize()
    ref_idx, ref_cnt = oracle.topk(s.double().numpy(), sl, 256)
    np.testing.assert_array_equal(host(idx).numpy(), ref_idx)
    np.testing.assert_array_equal(host(cnt).numpy(), ref_cnt)


# ------------------------------------------------------------------ select
@pytest.mark.parametrize("case", ["small", "multi_segment", "r64", "fp32", "max"])
def test_select_equals_score_then_topk_and_matches_oracle(case, form):
    kt = torch.bfloat16
    agg = ops.AGG_SUM
    if case == "small":
        w, sl = W(T=1500, k=64), [1500, 1111]
    elif case == "multi_segment":
        w, sl = W(B=4, Hkv=8, Hq=32, T=40000, k=256, seed=12), [40000, 39999, 12345, 257]
    elif case == "r64":
        w, sl = W(d=256, r=64, Hq=16, Hkv=2, T=5000, k=256, seed=13), [5000, 4097]
    elif case == "fp32":
        w, sl, kt = W(T=3000, k=100, seed=14), [3000, 2999], torch.float32
    else:
        w, sl, agg = W(T=3000, k=128, seed=15), [3000, 1500], ops.AGG_MAX
    dtype = torch.float32 if kt == torch.float32 else torch.bfloat16
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, dtype=dtype, seq_lens=sl)
    Kt = ops.build_lowrank_cache(Kd, Pd, kt_dtype=kt)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k, agg=agg, form=form)
    s = ops.score(qd, Pd, Kt, sld, agg=agg)
    idx2, cnt2 = ops.topk(s, sld, w.k, form=form)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(idx).numpy(), host(idx2).numpy())
    np.testing.assert_array_equal(host(cnt).numpy(), host(cnt2).numpy())
    ref = oracle.score(q, P, host(Kt), slh, agg=agg)
    check_selection(host(idx).numpy(), host(cnt).numpy(), ref, slh.numpy(), w.k)


def test_select_exact_ties_take_lowest_index(form):
    w = W(B=1, Hkv=2, Hq=4, T=3000, k=50, kind="plain", seed=16)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    # head 0: every row equal -> every score equal -> the first k tokens
    Kd[0, :, 0, :] = Kd[0, 7, 0, :]
    # head 1: a block of 100 identical rows at 1000..1099 along P P^T (sum of the
    # group's queries), far above every other token -> the first 50 of the block
    x = q[0, 2:4, :].float().sum(0)
    y = P[1] @ (P[1].T @ x)
    Kd[0, 1000:1100, 1, :] = (50.0 * y / y.norm()).to(Kd.dtype).to(DEV)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k, form=form)
    torch.cuda.synchronize()
    assert host(idx)[0, 0].tolist() == list(range(50))
    assert host(idx)[0, 1].tolist() == list(range(1000, 1050))
    # permuting the tokens permutes the selection (distinct scores)
    perm = torch.randperm(w.T, generator=torch.Generator().manual_seed(1))
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(W(B=1, Hkv=2, Hq=4, T=3000, k=50, seed=17))
    Kt = ops.build_lowrank_cache(Kd, Pd)
    i1, _ = ops.select(qd, Pd, Kt, sld, w.k, form=form)
    Kp = Kd[:, perm.to(DEV)].contiguous()
    Ktp = ops.build_lowrank_cache(Kp, Pd)
    i2, _ = ops.select(qd, Pd, Ktp, sld, w.k, form=form)
    torch.cuda.synchronize()
    for h in range(2):
        assert sorted(perm[host(i2)[0, h].long()].tolist()) == host(i1)[0, h].tolist()


# ------------------------------------------------------------------ attend
@pytest.mark.parametrize("d,G,dtype", [(128, 4, torch.bfloat16), (128, 4, torch.float32), (256, 8, torch.bfloat16),
                                       (64, 1, torch.bfloat16), (128, 16, torch.bfloat16), (256, 2, torch.float32)])
def test_indexed_decode_parity(d, G, dtype):
    w = W(d=d, Hq=2 * G, Hkv=2, T=1000, k=200, r=8, seed=20 + d + G)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, dtype=dtype, seq_lens=[1000, 450])
    g = torch.Generator().manual_seed(5)
    idx = torch.full((w.B, w.Hkv, w.k), -1, dtype=torch.int32)
    cnt = torch.tensor([[200, 131], [1, 0]], dtype=torch.int32)
    for b in range(w.B):
        for h in range(w.Hkv):
            c = int(cnt[b, h])
            idx[b, h, :c] = torch.sort(torch.randperm(int(sl[b]), generator=g)[:c])[0].to(torch.int32)
    out, lse = ops.indexed_decode(qd, Kd, Vd, idx.to(DEV), cnt.to(DEV), sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(q, K, V, idx, cnt, sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, dtype)
    # count = NULL: the count is the number of leading non-negative slots
    out2, lse2 = ops.indexed_decode(qd, Kd, Vd, idx.to(DEV), None, sld, w.scale)
    torch.cuda.synchronize()
    check_attention(out2, lse2, ref_o, ref_l, dtype)


@pytest.mark.parametrize("window", [0, 100, 5000])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dense_decode_parity(window, dtype):
    w = W(T=3000, Hq=8, Hkv=2, seed=30)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, dtype=dtype, seq_lens=[3000, 77])
    out, lse = ops.dense_decode(qd, Kd, Vd, sld, w.scale, window=window)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, V, sl, w.scale, window=window)
    check_attention(out, lse, ref_o, ref_l, dtype)


@pytest.mark.parametrize("d,G,window", [(64, 1, 0), (128, 16, 0), (256, 2, 300), (64, 8, 64), (128, 3, 0)])
def test_dense_decode_shapes_and_ragged_rows(d, G, window):
    """The tensor-core dense pass over every head width, group sizes 1..16,
    windows shorter and longer than a tile, and rows of 0, 1, 63, 65 and a
    few thousand tokens (tile edges and empty rows)."""
    w = W(B=5, d=d, Hq=2 * G, Hkv=2, T=2100, r=8, seed=34 + d + G)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[2100, 0, 1, 63, 65])
    out, lse = ops.dense_decode(qd, Kd, Vd, sld, w.scale, window=window)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, V, sl, w.scale, window=window)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_dense_decode_long_many_splits():
    w = W(B=1, T=70000, Hq=16, Hkv=2, d=256, r=8, seed=31)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    out, lse = ops.dense_decode(qd, Kd, Vd, sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, V, sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_sparse_with_k_equal_T_equals_dense():
    w = W(T=640, k=640, seed=32)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    o1, l1 = ops.indexed_decode(qd, Kd, Vd, idx, cnt, sld, w.scale)
    o2, l2 = ops.dense_decode(qd, Kd, Vd, sld, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx[:, :, :640].cpu(), torch.arange(640, dtype=torch.int32).expand(2, 2, 640))
    torch.testing.assert_close(o1.float(), o2.float(), rtol=0, atol=2e-2)
    torch.testing.assert_close(l1, l2, rtol=0, atol=1e-3)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gather_then_dense_matches_indexed_and_oracle(dtype):
    w = W(T=4000, k=256, seed=33)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, dtype=dtype, seq_lens=[4000, 100])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    o1, l1 = ops.indexed_decode(qd, Kd, Vd, idx, cnt, sld, w.scale)
    o2, l2 = ops.gather_then_dense(qd, Kd, Vd, idx, cnt, sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    check_attention(o1, l1, ref_o, ref_l, dtype)
    check_attention(o2, l2, ref_o, ref_l, dtype)


# ------------------------------------------------------------- whole step
@pytest.mark.parametrize("agg", [ops.AGG_SUM, ops.AGG_MAX])
def test_decode_step_end_to_end(agg):
    w = W(B=3, T=6000, k=256, seed=40)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[6000, 5999, 1])
    pos = (sl - 1).clamp_min(0)
    # prefix cache built without the newest row, which the step appends
    Kt0 = ops.build_lowrank_cache(Kd, Pd)
    for b in range(w.B):
        Kt0[b, :, int(pos[b])] = 0
    out, lse, idx, cnt = ops.decode_step(qd, Kd, Vd, Pd, Kt0, sld, pos.to(DEV), w.k, w.scale, agg=agg)
    torch.cuda.synchronize()
    # stage-isolated: oracle scores on the GPU's low-rank cache (after the append)
    check_append(Kt0, K, P, pos.tolist(), 1)
    ref_s = oracle.score(q, P, host(Kt0), sl, agg=agg)
    check_selection(host(idx).numpy(), host(cnt).numpy(), ref_s, sl.numpy(), w.k)
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)
    # end to end: the oracle's own step from its own low-rank cache.  The
    # index sets must be identical except for tokens whose oracle score lies
    # within the tie window of the k-th score; outputs are compared wherever
    # the sets are identical
    Kt_or = oracle.append_lowrank(K, P, [0] * w.B, w.T)
    _, s_or, idx_or, cnt_or, out_or, lse_or = oracle.step(q, K, V, P, Kt_or, sl, w.k, w.scale, agg=agg)
    check_end_to_end(out, lse, idx, cnt, s_or, idx_or, out_or, lse_or, sl, w.k, w.G)


@pytest.mark.parametrize("shape", ["d128_g4", "d256_g8_r64", "d128_g16", "d128_g1", "ragged"])
def test_fused_decode_step_matches_three_launch_and_oracle(shape):
    """The one-launch decode step (append and folded query in the streaming
    kernel's prologue, attention in its epilogue) against the three-launch
    step and the oracle: same appended rows and selections bit for bit, outputs
    within the bf16 tolerance."""
    if shape == "d128_g4":
        w, sl = W(B=3, T=20000, k=256, seed=80), [20000, 19999, 7000]
    elif shape == "d256_g8_r64":
        w, sl = W(B=2, Hq=16, Hkv=2, d=256, r=64, T=9000, k=256, seed=81), [9000, 4321]
    elif shape == "d128_g16":
        w, sl = W(B=2, Hq=32, Hkv=2, T=5000, k=300, seed=82), [5000, 100]
    elif shape == "d128_g1":
        w, sl = W(B=2, Hq=4, Hkv=4, T=3000, k=64, seed=83), [3000, 1]
    else:
        w, sl = W(B=4, T=12000, k=128, seed=84), [12000, 0, 1, 6001]
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    pos = (slh - 1).clamp_min(0)
    Kt0 = ops.build_lowrank_cache(Kd, Pd)
    for b in range(w.B):
        Kt0[b, :, int(pos[b])] = 0
    Kt1 = Kt0.clone()
    out1, lse1, idx1, cnt1 = ops.decode_step(qd, Kd, Vd, Pd, Kt0, sld, pos.to(DEV), w.k, w.scale, form="stream")
    out2, lse2, idx2, cnt2 = ops.decode_step(qd, Kd, Vd, Pd, Kt1, sld, pos.to(DEV), w.k, w.scale, form="stream",
                                             unfused=True)
    torch.cuda.synchronize()
    assert torch.equal(Kt0, Kt1)
    assert torch.equal(idx1, idx2) and torch.equal(cnt1, cnt2)
    assert (out1.float() - out2.float()).abs().max().item() <= 2e-2
    l1, l2 = host(lse1).double().numpy(), host(lse2).double().numpy()
    assert np.array_equal(np.isinf(l1), np.isinf(l2))
    fin = np.isfinite(l1)
    assert np.abs(l1[fin] - l2[fin]).max(initial=0.0) <= 1e-3
    check_append(Kt0, K, P, pos.tolist(), 1)
    ref_o, ref_l = oracle.attend(q, K, V, host(idx1), host(cnt1), slh, w.scale)
    check_attention(out1, lse1, ref_o, ref_l, torch.bfloat16)


# -------------------------------------------------------------- edge cases
def test_empty_and_short_sequences():
    w = W(B=3, T=300, k=64, seed=50)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[0, 5, 300])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    out, lse = ops.indexed_decode(qd, Kd, Vd, idx, cnt, sld, w.scale)
    do, dl = ops.dense_decode(qd, Kd, Vd, sld, w.scale)
    torch.cuda.synchronize()
    c = host(cnt)
    assert c[0].tolist() == [0, 0] and c[1].tolist() == [5, 5] and c[2].tolist() == [64, 64]
    assert torch.all(host(idx)[0] == -1)
    assert host(idx)[1, 0, :5].tolist() == [0, 1, 2, 3, 4]
    assert torch.all(host(out)[0] == 0) and torch.all(torch.isneginf(host(lse)[0]))
    assert torch.all(host(do)[0] == 0) and torch.all(torch.isneginf(host(dl)[0]))
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), c, sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_device_status_flags_bad_data_without_fault():
    w = W(B=2, T=500, k=16, seed=51)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    idx = torch.arange(16, dtype=torch.int32).expand(2, 2, 16).contiguous()
    bad = idx.clone()
    bad[1, 1, 3] = 100000  # outside [0, T_b): skipped and flagged
    cnt = torch.full((2, 2), 16, dtype=torch.int32)
    dims = ops.make_dims(qd, Kd, Vd, r=8)
    ws = ops.new_workspace(dims, 16, ops.OP_INDEXED_DECODE, qd.device)
    out, lse = ops.indexed_decode(qd, Kd, Vd, bad.to(DEV), cnt.to(DEV), sld, w.scale, ws=ws)
    assert ops.device_status(ws) & ops.DEV_INDEX
    keep = bad.clone()
    keep[1, 1, 3:15] = keep[1, 1, 4:16].clone()
    kc = cnt.clone()
    kc[1, 1] = 15
    ref_o, ref_l = oracle.attend(q, K, V, keep, kc, sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)
    # seq_lens above T_cap: clamped and flagged
    ops.workspace_init(ws)
    big = torch.tensor([10**6, 500], dtype=torch.int32, device=DEV)
    ops.indexed_decode(qd, Kd, Vd, idx.to(DEV), cnt.to(DEV), big, w.scale, ws=ws)
    assert ops.device_status(ws) & ops.DEV_SEQLEN
    # append position out of range: row skipped and flagged
    Kt = ops.build_lowrank_cache(Kd, Pd)
    before = Kt.clone()
    wsa = ops.new_workspace(dims, 1, ops.OP_APPEND, qd.device)
    ops.append_lowrank(Kd, Pd, Kt, torch.tensor([499, 500], dtype=torch.int32, device=DEV), 1, ws=wsa)
    assert ops.device_status(wsa) & ops.DEV_POS
    assert torch.equal(Kt[1], before[1])


def test_rows_past_the_range_do_not_leak():
    """Cache rows past T_b and gather-buffer rows past the count are not part
    of the attention and may hold anything (an unwritten KV slot): NaN planted
    there must not reach any output (dense, gathered, latent dense, latent
    gathered)."""
    w = W(B=2, T=700, k=128, seed=58)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[650, 100])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    for b, tb in enumerate((650, 100)):
        Kd[b, tb:] = float("nan")
        Vd[b, tb:] = float("nan")
    dims = ops.make_dims(qd, Kd, Vd, r=8)
    gbuf = torch.full((ops.gather_buffer_bytes(dims, w.k) // 2,), float("nan"), dtype=torch.bfloat16, device=DEV)
    do, dl = ops.dense_decode(qd, Kd, Vd, sld, w.scale)
    go, gl = ops.gather_then_dense(qd, Kd, Vd, idx, cnt, sld, w.scale, gather_buf=gbuf.view(torch.uint8))
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, V, sl, w.scale)
    check_attention(do, dl, ref_o, ref_l, torch.bfloat16)
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    check_attention(go, gl, ref_o, ref_l, torch.bfloat16)
    m = MW(T=900, k=512, seed=59)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(m, seq_lens=[900, 300])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, m.k)
    Kd[1, 300:] = float("nan")
    dims = ops.make_dims(qd, Kd, None, r=8)
    gbuf = torch.full((ops.gather_buffer_bytes(dims, m.k) // 2,), float("nan"), dtype=torch.bfloat16, device=DEV)
    do, dl = ops.dense_decode(qd, Kd, None, sld, m.scale)
    go, gl = ops.gather_then_dense(qd, Kd, None, idx, cnt, sld, m.scale, gather_buf=gbuf.view(torch.uint8))
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, None, sl, m.scale, dv=512, v_aliases_k=True)
    check_attention(do, dl, ref_o, ref_l, torch.bfloat16)
    ref_o, ref_l = oracle.attend(q, K, None, host(idx), host(cnt), sl, m.scale, dv=512, v_aliases_k=True)
    check_attention(go, gl, ref_o, ref_l, torch.bfloat16)


def test_invalid_arguments_raise():
    w = W(B=1, Hq=64, Hkv=2, T=100, k=8, seed=52)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    idx = torch.zeros((1, 2, 8), dtype=torch.int32, device=DEV)
    with pytest.raises(ops.JssaError) as e:
        ops.indexed_decode(qd, Kd, Vd, idx, None, sld, 1.0)  # G = 32 > 16
    assert e.value.code == -2
    w = W(B=1, T=100, k=8, seed=53)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    dims = ops.make_dims(qd, Kd, Vd, r=8)
    small = torch.zeros(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(ops.JssaError) as e:
        ops.indexed_decode(qd, Kd, Vd, idx, None, sld, 1.0, ws=small)
    assert e.value.code == -3
    with pytest.raises(ops.JssaError) as e:
        ops.select(qd, Pd, ops.build_lowrank_cache(Kd, Pd), sld, 4096)
    assert e.value.code == -1
    assert dims.B == 1


def test_bounded_waits_expire_with_a_status_and_the_context_stays_usable():
    """Failure detection without a fault: the library's bounded on-chip waits
    (an mbarrier phase, the abort-aware wait, a device word) run on a barrier
    and a word that nothing completes, with a short limit; every one gives up,
    the status word carries JSSA_DEV_TIMEOUT, the kernel returns, and the next
    call on the same context computes normally."""
    import time

    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    L = ops.lib()
    L.jssa_check_wait_expiry.restype = ctypes.c_int
    L.jssa_check_wait_expiry.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_void_p]
    t0 = time.perf_counter()
    st = L.jssa_check_wait_expiry(ws.data_ptr(), 256, 200000, torch.cuda.current_stream().cuda_stream)
    assert st == 0, L.jssa_last_error()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert ops.device_status(ws) & ops.DEV_TIMEOUT
    assert int(ws[128:132].view(torch.int32).item()) == 3
    assert elapsed < 5.0, "the waits did not give up near their 200 us limit (%.2f s)" % elapsed
    # argument checks: limits outside [1 us, 1 s] are rejected on the host
    assert L.jssa_check_wait_expiry(ws.data_ptr(), 256, 10, None) == -1
    assert L.jssa_check_wait_expiry(ws.data_ptr(), 64, 200000, None) == -3
    # the context is still usable: a normal decode step after the expiries
    w = W(B=1, T=600, k=32, seed=57)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    out, lse, idx, cnt = ops.decode_step(qd, Kd, Vd, Pd, Kt, sld, (sld - 1).clamp_min(0), w.k, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), host(cnt), sl, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_host_buffer_step_equals_device_step():
    """jssa_decode_step_host (pinned host input block -> staged copy -> new
    K/V rows written at pos -> decode step -> output copied to the host) gives
    bit for bit what writing the rows on the device and calling
    jssa_decode_step gives; the GQA and the latent form."""
    for w, sl in ((W(B=3, T=5000, k=256, seed=130), [5000, 4000, 77]), (MW(T=3000, k=512, seed=131), [3000, 2500])):
        (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
        pos = (sld - 1).clamp_min(0).contiguous()
        g = torch.Generator().manual_seed(9)
        kn = torch.randn((w.B, w.Hkv, w.d), generator=g).to(torch.bfloat16)
        vn = None if Vd is None else torch.randn((w.B, w.Hkv, w.Dv), generator=g).to(torch.bfloat16)
        # device path: write the rows, then the step
        K1, V1 = Kd.clone(), None if Vd is None else Vd.clone()
        Kt1 = ops.build_lowrank_cache(K1, Pd)
        for b in range(w.B):
            K1[b, int(pos[b])] = kn[b].to(DEV)
            if V1 is not None:
                V1[b, int(pos[b])] = vn[b].to(DEV)
        o1, l1, i1, c1 = ops.decode_step(qd, K1, V1, Pd, Kt1, sld, pos, w.k, w.scale)
        # host path
        K2, V2 = Kd.clone(), None if Vd is None else Vd.clone()
        Kt2 = ops.build_lowrank_cache(K2, Pd)
        dims = ops.make_dims(qd, K2, V2, P=Pd, Kt=Kt2)
        parts = [q.reshape(-1), kn.reshape(-1)] + ([] if vn is None else [vn.reshape(-1)])
        blob = torch.cat(parts).view(torch.uint8)
        in_host = torch.empty(ops.host_step_bytes(dims), dtype=torch.uint8).pin_memory()
        assert in_host.numel() == blob.numel()
        in_host.copy_(blob)
        stage = torch.empty_like(in_host, device=DEV)
        out_host = torch.empty(o1.shape, dtype=o1.dtype).pin_memory()
        ws = ops.new_workspace(dims, w.k, ops.OP_DECODE_STEP, qd.device)
        o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
        i2, c2 = torch.empty_like(i1), torch.empty_like(c1)
        ops.decode_step_host(in_host, stage, K2, V2, Pd, Kt2, sld, pos, w.k, w.scale, out_host, ws, i2, c2, o2, l2,
                             dims=dims)
        torch.cuda.synchronize()
        assert torch.equal(K1, K2) and (V1 is None or torch.equal(V1, V2)) and torch.equal(Kt1, Kt2)
        assert torch.equal(i1, i2) and torch.equal(c1, c2)
        assert torch.equal(o1.cpu(), out_host) and torch.equal(o1, o2)
        assert ops.device_status(ws) == 0


# ------------------------------------------------ exact block screening
def test_block_norms_match_numpy():
    w = W(B=2, Hq=8, Hkv=2, T=1000, r=32, seed=159)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    nrm = ops.block_norms(Kt)
    torch.cuda.synchronize()
    kt = host(Kt).double().numpy()
    rn = np.sqrt((kt * kt).sum(-1))  # [B, Hkv, T]
    nb = (w.T + 127) // 128
    ref = np.stack([rn[:, :, j * 128:(j + 1) * 128].max(-1) for j in range(nb)], -1)
    np.testing.assert_allclose(host(nrm).double().numpy(), ref, rtol=1e-5)


def test_block_screening_is_exact_and_skips():
    """Exact screening over the low-rank cache: with block norm bounds the
    streaming form skips tiles that cannot beat its segment's k-th key, and
    every result stays bit-identical (selection alone, fused and unfused
    decode step; the other selection forms ignore the bounds).  Inputs where
    it must trigger: every row's keys past token 1024 are zero, so once a
    segment holds k candidates its remaining tiles are bounded by 0."""
    w = W(B=16, Hq=32, Hkv=8, T=16384, k=64, kind="plain", seed=160)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w)
    Kd[:, 1024:] = 0
    Kt = ops.build_lowrank_cache(Kd, Pd)
    nrm = ops.block_norms(Kt)
    dims = ops.make_dims(qd, Kd, Vd, P=Pd, Kt=Kt)
    i1, c1 = ops.select(qd, Pd, Kt, sld, w.k, form="stream")
    ws = ops.new_workspace(dims, w.k, ops.OP_SELECT, qd.device)
    i2, c2 = ops.select(qd, Pd, Kt, sld, w.k, form="stream", ws=ws, block_norms=nrm)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
    skipped = ops.skip_count(ws)
    assert skipped > 0, "no tile was screened out"
    for f in ("cluster", "scan", "auto"):
        i3, c3 = ops.select(qd, Pd, Kt, sld, w.k, form=f, block_norms=nrm)
        torch.cuda.synchronize()
        assert torch.equal(i1, i3) and torch.equal(c1, c3), f
    # the selection against the oracle on a few rows (the GPU's own low-rank cache)
    ref_s = oracle.score(q[:2], P, host(Kt[:2]), sl[:2])
    check_selection(host(i2[:2]).numpy(), host(c2[:2]).numpy(), ref_s, sl[:2].numpy(), w.k)
    # the decode step, fused and unfused, with and without screening
    pos = (sld - 1).clamp_min(0)
    for unfused in (False, True):
        Kt1, Kt2, n2 = Kt.clone(), Kt.clone(), nrm.clone()
        wsd = ops.new_workspace(dims, w.k, ops.OP_DECODE_STEP, qd.device)
        o1, l1, j1, d1 = ops.decode_step(qd, Kd, Vd, Pd, Kt1, sld, pos, w.k, w.scale, form="stream", unfused=unfused)
        o2, l2, j2, d2 = ops.decode_step(qd, Kd, Vd, Pd, Kt2, sld, pos, w.k, w.scale, form="stream", unfused=unfused,
                                         ws=wsd, block_norms=n2)
        torch.cuda.synchronize()
        assert torch.equal(Kt1, Kt2) and torch.equal(j1, j2) and torch.equal(d1, d2)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        assert ops.skip_count(wsd) > 0
        # the bounds still cover every row of the cache after the append
        assert torch.all(n2 >= ops.block_norms(Kt2) * (1 - 1e-6))


# ------------------------------------------------------- calibration of P
@pytest.mark.parametrize("d,r,Hkv,G", [(128, 32, 2, 4), (256, 64, 2, 8), (64, 8, 3, 1)])
def test_calibrated_basis_keeps_the_dominant_joint_energy(d, r, Hkv, G):
    """jssa_calibrate_basis against the oracle's fp64 statement of the same
    reading: the GPU basis is orthonormal and keeps at least 99.9% of the
    joint energy the exact top-r eigen-subspace keeps (tr(P^T M P) with the
    oracle's M; any basis of a dominant subspace does, even where eigenvalues
    of the noise bulk are too close for the iteration to single one out)."""
    from oracle import calib

    w = W(B=3, Hq=G * Hkv, Hkv=Hkv, d=d, r=r, T=3000, k=8, seed=150 + d)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[3000, 2000, 700])
    Pc = ops.calibrate_basis(qd, Kd, sld, Pd, n_keys=512, iters=40)
    torch.cuda.synchronize()
    Pg = host(Pc).double().numpy()
    Pref, lam, M = calib.calibrate(q, K, sl, r, 512)
    for h in range(Hkv):
        np.testing.assert_allclose(Pg[h].T @ Pg[h], np.eye(r), atol=2e-5)
    best = lam[:, :r].sum(1)
    got = calib.captured_energy(M, Pg)
    assert np.all(got >= 0.999 * best), (got, best)


def test_calibrated_basis_recovers_a_planted_subspace():
    """Queries and keys drawn inside a 5-dim subspace U: the calibrated basis
    (r = 16) contains U (||U^T P||_F^2 = 5), from a random start."""
    g = torch.Generator().manual_seed(151)
    d, r0, r, Hkv, G = 128, 5, 16, 2, 4
    U = torch.linalg.qr(torch.randn(Hkv, d, r0, generator=g, dtype=torch.float64))[0]
    q = torch.einsum("nhgz,hdz->nhgd", torch.randn(2, Hkv, G, r0, generator=g, dtype=torch.float64), U)
    K = torch.einsum("bthz,hdz->bthd", torch.randn(2, 600, Hkv, r0, generator=g, dtype=torch.float64), U)
    qd = q.reshape(2, Hkv * G, d).to(torch.bfloat16).contiguous().to(DEV)
    Kd = K.to(torch.bfloat16).contiguous().to(DEV)
    P0 = torch.linalg.qr(torch.randn(Hkv, d, r, generator=g, dtype=torch.float64))[0].float().contiguous().to(DEV)
    sl = torch.tensor([600, 450], dtype=torch.int32, device=DEV)
    Pc = ops.calibrate_basis(qd, Kd, sl, P0, n_keys=256, iters=30)
    torch.cuda.synchronize()
    for h in range(Hkv):
        cap = float((U[h].T @ host(Pc[h]).double()).norm() ** 2)
        assert abs(cap - r0) < 1e-3, cap


# --------------------------------------------- per-query-head selection
@pytest.mark.parametrize("case", ["g4", "g8_r64", "g1", "fp32"])
def test_select_heads_and_decode_heads_match_oracle(case, form):
    """Per-query-head selection (every query head its own top-k) and attention
    over per-head lists: bit-exact top-k on the GPU's own fp32 scores is not
    available here, so the selection follows the tie-window rule against the
    oracle's fp64 per-head scores on the GPU's low-rank cache, and attention
    is compared on the GPU's indices."""
    kt, dtype = torch.bfloat16, torch.bfloat16
    if case == "g4":
        w, sl = W(B=3, Hq=8, Hkv=2, T=7000, k=200, seed=120), [7000, 6999, 150]
    elif case == "g8_r64":
        w, sl = W(B=2, Hq=16, Hkv=2, d=256, r=64, T=5000, k=256, seed=121), [5000, 4096]
    elif case == "g1":
        w, sl = W(B=2, Hq=4, Hkv=4, T=3000, k=64, seed=122), [3000, 1]
    else:
        w, sl, kt, dtype = W(B=2, T=3000, k=100, seed=123), [3000, 2999], torch.float32, torch.float32
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, dtype=dtype, seq_lens=sl)
    Kt = ops.build_lowrank_cache(Kd, Pd, kt_dtype=kt)
    idx, cnt = ops.select_heads(qd, Pd, Kt, sld, w.k, form=form)
    out, lse = ops.indexed_decode_heads(qd, Kd, Vd, idx, cnt, sld, w.scale)
    torch.cuda.synchronize()
    ref_s = oracle.score_heads(q, P, host(Kt), slh)
    check_selection(host(idx).numpy(), host(cnt).numpy(), ref_s, slh.numpy(), w.k)
    ref_o, ref_l = oracle.attend_heads(q, K, V, host(idx), host(cnt), slh, w.scale)
    check_attention(out, lse, ref_o, ref_l, dtype)
    if case == "g1":  # one query head per KV head: the per-KV-head selection itself
        i2, c2 = ops.select(qd, Pd, Kt, sld, w.k, form=form)
        torch.cuda.synchronize()
        assert torch.equal(idx, i2) and torch.equal(cnt, c2)


def test_select_heads_forms_agree_and_group_lists_reduce_to_indexed():
    w, sl = W(B=2, Hq=8, Hkv=2, T=20000, k=256, seed=124), [20000, 9000]
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    a = ops.select_heads(qd, Pd, Kt, sld, w.k, form="cluster")
    b = ops.select_heads(qd, Pd, Kt, sld, w.k, form="scan")
    # every head of a KV head on its group's shared list: equal to the per-KV-head attention
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    G = w.G
    o1, l1 = ops.indexed_decode(qd, Kd, Vd, idx, cnt, sld, w.scale)
    o2, l2 = ops.indexed_decode_heads(qd, Kd, Vd, idx.repeat_interleave(G, 1).contiguous(),
                                      cnt.repeat_interleave(G, 1).contiguous(), sld, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


# ------------------------------------------------------- full-size samples
def _full_size_sampled(w, pairs, ks=None, dense_check=True):
    """The decode step at a full-size workload, in the launch form bench.py
    times (automatic form choice), on sampled (b, h) pairs: stage-isolated
    (the oracle on the GPU's low-rank cache and indices) and end to end (the
    oracle's own low-rank cache, scores, selection and output)."""
    q, K, V, P, sl = make_inputs(w, device=DEV)
    Kt = ops.build_lowrank_cache(K, P)
    pos = (sl - 1).clamp_min(0)
    G = w.G
    s = ops.score(q, P, Kt, sl)
    torch.cuda.synchronize()
    per_pair = []
    for b, h in pairs:
        qs = host(q[b:b + 1, h * G:(h + 1) * G].contiguous())
        Ks = host(K[b:b + 1, :, h:h + 1].contiguous())
        Vs = host(V[b:b + 1, :, h:h + 1].contiguous())
        Ps = host(P[h:h + 1].contiguous())
        slh = sl[b:b + 1].cpu()
        Kt_or = oracle.append_lowrank(Ks, Ps, [0], w.T)  # the oracle's own low-rank cache
        per_pair.append((b, h, qs, Ks, Vs, Ps, slh, Kt_or, oracle.score(qs, Ps, Kt_or, slh)))
    for k in ks or (w.k,):
        out, lse, idx, cnt = ops.decode_step(q, K, V, P, Kt, sl, pos, k, w.scale)
        idx2, cnt2 = ops.topk(s, sl, k)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx2) and torch.equal(cnt, cnt2), "decode step and score + top-k differ (k=%d)" % k
        for b, h, qs, Ks, Vs, Ps, slh, Kt_or, s_or in per_pair:
            Kts = host(Kt[b:b + 1, h:h + 1].contiguous())
            # the newest row was appended by the step: check it, then score the GPU cache
            check_append(Kt[b:b + 1, h:h + 1], Ks, Ps, [int(pos[b])], 1)
            ref_s = oracle.score(qs, Ps, Kts, slh)
            sg = host(s[b:b + 1, h:h + 1]).numpy()
            check_scores(sg, ref_s, score_scale(qs, Ps, Kts, G, 0))
            ig, cg = host(idx[b:b + 1, h:h + 1]).numpy(), host(cnt[b:b + 1, h:h + 1]).numpy()
            check_selection(ig, cg, ref_s, slh.numpy(), k)
            og, lg = out[b:b + 1, h * G:(h + 1) * G], lse[b:b + 1, h * G:(h + 1) * G]
            ref_o, ref_l = oracle.attend(qs, Ks, Vs, ig, cg, slh, w.scale)
            check_attention(og, lg, ref_o, ref_l, torch.bfloat16)
            # end to end against the oracle's own step
            idx_or, cnt_or = oracle.topk(s_or, slh, k)
            out_or, lse_or = oracle.attend(qs, Ks, Vs, idx_or, cnt_or, slh, w.scale)
            check_end_to_end(og, lg, ig, cg, s_or, idx_or, out_or, lse_or, slh, k, G)
    if dense_check:
        do, dl = ops.dense_decode(q, K, V, sl, w.scale, window=w.window)
        torch.cuda.synchronize()
        for b, h, qs, Ks, Vs, Ps, slh, Kt_or, s_or in per_pair[:2]:
            ref_o, ref_l = oracle.dense(qs, Ks, Vs, slh, w.scale, window=w.window)
            check_attention(do[b:b + 1, h * G:(h + 1) * G], dl[b:b + 1, h * G:(h + 1) * G], ref_o, ref_l,
                            torch.bfloat16)
    del q, K, V, Kt, s
    torch.cuda.empty_cache()


def _wl(name, **over):
    from token_level_sparse_kv_b200.inputs import WORKLOADS

    w = WORKLOADS[name]
    return Workload(**{**w.__dict__, **over}) if over else w


def test_full_size_gqa_128k_b16_sampled():
    # the headline workload (k = 256) and the k sweep at B = 16
    _full_size_sampled(_wl("gqa_128k_b16"), [(0, 0), (7, 3), (15, 7), (9, 5)], ks=(256, 128, 1024))


@pytest.mark.parametrize("B", [1, 4])
def test_full_size_gqa_128k_sweep_sampled(B):
    """The 128K sweep points bench.py times with --batch B --topk k (k in
    {128, 256, 1024}): the k = 1024 cases take the three-launch cluster form
    at B = 1 and the fused streaming form at B = 4."""
    pairs = [(0, 0), (0, 5)] if B == 1 else [(0, 0), (3, 7), (2, 4)]
    _full_size_sampled(_wl("gqa_128k_b16", B=B), pairs, ks=(128, 256, 1024), dense_check=False)


def test_full_size_gqa_32k_b4_sampled():
    _full_size_sampled(_wl("gqa_32k_b4"), [(0, 0), (3, 7), (2, 4)])


def test_full_size_hybrid_global_sampled():
    _full_size_sampled(_wl("hybrid_global_128k_b8"), [(0, 0), (7, 1), (4, 0)])


def test_full_size_gqa_4k_b1_all_heads():
    _full_size_sampled(_wl("gqa_4k_b1"), [(0, h) for h in range(8)])


# ------------------------------------------------------- latent cache (MLA)
def MW(**kw):
    base = dict(name="mla", B=2, Hq=128, Hkv=1, d=576, dv=512, T=3000, r=64, k=300, latent=True, seed=60)
    base.update(kw)
    return Workload(**base)


@pytest.mark.parametrize("k,sl", [(100, [3000, 77]), (300, [3000, 2999]), (2048, [3000, 2500]), (128, [128, 0])])
def test_mla_indexed_decode_parity(k, sl):
    w = MW(k=k, seed=61 + k)
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    assert V is None
    g = torch.Generator().manual_seed(7)
    idx = torch.full((w.B, 1, k), -1, dtype=torch.int32)
    cnt = torch.zeros((w.B, 1), dtype=torch.int32)
    for b in range(w.B):
        c = min(k, int(slh[b]))
        cnt[b, 0] = c
        idx[b, 0, :c] = torch.sort(torch.randperm(int(slh[b]), generator=g)[:c])[0].to(torch.int32)
    out, lse = ops.indexed_decode(qd, Kd, None, idx.to(DEV), cnt.to(DEV), sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(q, K, None, idx, cnt, slh, w.scale, dv=512, v_aliases_k=True)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


@pytest.mark.parametrize("B", [3, 12])
def test_mla_split_merge_forms(B):
    """The 16 splits of a k = 2048 latent-cache decode merge inside the
    attention kernel when all its CTAs fit on the GPU at once (B = 3: 48
    CTAs), else in a second kernel (B = 12: 192 CTAs, above the 148 SMs);
    both against the oracle, and twice in a row (the merge counters reset
    themselves)."""
    k = 2048
    w = MW(B=B, T=2200, k=k, seed=70 + B)
    sl = [2200 - 37 * b for b in range(B)]
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    g = torch.Generator().manual_seed(71)
    idx = torch.full((B, 1, k), -1, dtype=torch.int32)
    cnt = torch.zeros((B, 1), dtype=torch.int32)
    for b in range(B):
        c = min(k, int(slh[b]))
        cnt[b, 0] = c
        idx[b, 0, :c] = torch.sort(torch.randperm(int(slh[b]), generator=g)[:c])[0].to(torch.int32)
    dims = ops.make_dims(qd, Kd, None)
    n, _ = ops.plan_info(dims, k, ops.OP_INDEXED_DECODE)
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert n == (1 if 16 * B <= sms else 2), (n, B, sms)
    ws = ops.new_workspace(dims, k, ops.OP_INDEXED_DECODE, DEV)
    res = []
    for _ in range(2):
        out, lse = ops.indexed_decode(qd, Kd, None, idx.to(DEV), cnt.to(DEV), sld, w.scale, ws=ws)
        torch.cuda.synchronize()
        assert ops.device_status(ws) == 0
        res.append((out.clone(), lse.clone()))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    ref_o, ref_l = oracle.attend(q, K, None, idx, cnt, slh, w.scale, dv=512, v_aliases_k=True)
    check_attention(res[0][0], res[0][1], ref_o, ref_l, torch.bfloat16)


@pytest.mark.parametrize("T,sl", [(3000, [3000, 77]), (700, [129, 0]), (5000, [4097, 128])])
def test_mla_dense_decode_parity(T, sl):
    """Full-KV attention over the latent cache (the dense comparison path of
    the latent-cache workload): ragged rows, an empty row, tile edges."""
    w = MW(T=T, seed=63 + T)
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    out, lse = ops.dense_decode(qd, Kd, None, sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.dense(q, K, None, slh, w.scale, dv=512, v_aliases_k=True)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_mla_k_equal_T_equals_dense():
    """The pages' special case for the latent cache: with k = T every token is
    selected and the indexed decode equals dense latent attention."""
    w = MW(T=1900, k=1900, seed=66)
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[1900, 1900])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    o1, l1 = ops.indexed_decode(qd, Kd, None, idx, cnt, sld, w.scale)
    o2, l2 = ops.dense_decode(qd, Kd, None, sld, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx.cpu(), torch.arange(1900, dtype=torch.int32).expand(2, 1, 1900))
    torch.testing.assert_close(o1.float(), o2.float(), rtol=0, atol=2e-2)
    torch.testing.assert_close(l1, l2, rtol=0, atol=1e-3)
    ref_o, ref_l = oracle.dense(q, K, None, slh, w.scale, dv=512, v_aliases_k=True)
    check_attention(o2, l2, ref_o, ref_l, torch.bfloat16)


@pytest.mark.parametrize("k", [300, 2048])
def test_mla_gather_then_dense_matches_indexed_and_oracle(k):
    w = MW(T=4000, k=k, seed=67 + k)
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[4000, 250])
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k)
    o1, l1 = ops.indexed_decode(qd, Kd, None, idx, cnt, sld, w.scale)
    o2, l2 = ops.gather_then_dense(qd, Kd, None, idx, cnt, sld, w.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(q, K, None, host(idx), host(cnt), slh, w.scale, dv=512, v_aliases_k=True)
    check_attention(o1, l1, ref_o, ref_l, torch.bfloat16)
    check_attention(o2, l2, ref_o, ref_l, torch.bfloat16)


def test_mla_decode_step_end_to_end():
    w = MW(T=5000, k=512, kind="spiked", seed=70)
    (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=[5000, 4321])
    pos = (sl - 1).clamp_min(0)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    out, lse, idx, cnt = ops.decode_step(qd, Kd, None, Pd, Kt, sld, pos.to(DEV), w.k, w.scale)
    torch.cuda.synchronize()
    check_append(Kt, K, P, pos.tolist(), 1)
    ref_s = oracle.score(q, P, host(Kt), sl)
    check_selection(host(idx).numpy(), host(cnt).numpy(), ref_s, sl.numpy(), w.k)
    ref_o, ref_l = oracle.attend(q, K, None, host(idx), host(cnt), sl, w.scale, dv=512, v_aliases_k=True)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_full_size_mla_64k_b8_sampled():
    from token_level_sparse_kv_b200.inputs import WORKLOADS

    w = WORKLOADS["mla_64k_b8"]
    q, K, V, P, sl = make_inputs(w, device=DEV)
    Kt = ops.build_lowrank_cache(K, P)
    pos = (sl - 1).clamp_min(0)
    out, lse, idx, cnt = ops.decode_step(q, K, None, P, Kt, sl, pos, w.k, w.scale)
    s = ops.score(q, P, Kt, sl)
    idx2, cnt2 = ops.topk(s, sl, w.k, Hq=w.Hq, d=w.d)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(cnt, cnt2)
    for b in (0, 5):
        qs = host(q[b:b + 1])
        Ks = host(K[b:b + 1])
        slh = sl[b:b + 1].cpu()
        ref_s = oracle.score(qs, host(P), host(Kt[b:b + 1]), slh)
        check_selection(host(idx[b:b + 1]).numpy(), host(cnt[b:b + 1]).numpy(), ref_s, slh.numpy(), w.k)
        ref_o, ref_l = oracle.attend(qs, Ks, None, host(idx[b:b + 1]), host(cnt[b:b + 1]), slh, w.scale, dv=512,
                                     v_aliases_k=True)
        check_attention(out[b:b + 1], lse[b:b + 1], ref_o, ref_l, torch.bfloat16)
    # the dense comparison path at full size, one batch row against the oracle
    do, dl = ops.dense_decode(q, K, None, sl, w.scale)
    torch.cuda.synchronize()
    b = 3
    ref_o, ref_l = oracle.dense(host(q[b:b + 1]), host(K[b:b + 1]), None, sl[b:b + 1].cpu(), w.scale, dv=512,
                                v_aliases_k=True)
    check_attention(do[b:b + 1], dl[b:b + 1], ref_o, ref_l, torch.bfloat16)
    del q, K, Kt, s
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wname", ["gqa_4k_b1", "gqa_32k_b4", "mla_64k_b8", "hybrid_global_128k_b8", "gqa_128k_b16"])
def test_select_forms_agree_full_size(wname):
    """The cluster and the streaming selection give identical index lists on
    the full-size workloads (the shapes where the automatic choice flips)."""
    from token_level_sparse_kv_b200.inputs import WORKLOADS

    w = WORKLOADS[wname]
    q, K, V, P, sl = make_inputs(w, device=DEV)
    Kt = ops.build_lowrank_cache(K, P)
    res = []
    for f in ("cluster", "stream", "scan"):
        res.append(ops.select(q, P, Kt, sl, w.k, form=f))
    torch.cuda.synchronize()
    for r in res[1:]:
        assert torch.equal(res[0][0], r[0]) and torch.equal(res[0][1], r[1])
    del q, K, V, Kt
    torch.cuda.empty_cache()


# ------------------------------------------------- multi-layer decode loop
def _loop_layers(w, L, seed0):
    layers, cpu = [], []
    for l in range(L):
        wl = Workload(**{**w.__dict__, "seed": seed0 + l})
        (q, K, V, P, sl), (qd, Kd, Vd, Pd, sld) = draw(wl, seq_lens=[w.T - 8] * w.B)
        Kt = ops.build_lowrank_cache(Kd, Pd)
        layers.append((Kd, Vd, Pd, Kt))
        cpu.append((q, K, V, P))
    return layers, cpu


def test_decode_loop_graph_matches_eager_and_oracle():
    """An L-layer stack stepped three times eagerly and by CUDA-graph replay
    (the graph holds every layer and the device-side position advance) gives
    bit-identical selections, low-rank rows and outputs; the last step's first
    layer matches the oracle."""
    w = W(B=2, Hq=8, Hkv=2, T=3000, k=64, seed=90)
    L = 3
    layers_a, cpu = _loop_layers(w, L, 900)
    layers_b = [tuple(t.clone() for t in lay) for lay in layers_a]
    q0 = cpu[0][0].to(DEV)
    sl_a = torch.full((w.B,), w.T - 8, dtype=torch.int32, device=DEV)
    pos_a = sl_a - 1
    sl_b, pos_b = sl_a.clone(), pos_a.clone()
    loop_a = ops.DecodeLoop(layers_a, sl_a, pos_a, w.k, w.scale)
    loop_b = ops.DecodeLoop(layers_b, sl_b, pos_b, w.k, w.scale)
    loop_a.set_query(q0)
    loop_b.set_query(q0)
    for _ in range(3):
        loop_a.step()
    loop_b.capture()  # runs one step
    for _ in range(2):
        loop_b.step(graph=True)
    torch.cuda.synchronize()
    assert torch.equal(sl_a, sl_b) and int(sl_a[0]) == w.T - 8 + 3
    for l in range(L):
        assert torch.equal(loop_a.idx[l], loop_b.idx[l])
        assert torch.equal(loop_a.out[l], loop_b.out[l])
        assert torch.equal(layers_a[l][3], layers_b[l][3])
    # oracle: layer 0 of the last step (sequence length T-8+2, position T-8+1)
    q, K, V, P = cpu[0]
    slh = torch.full((w.B,), w.T - 8 + 2, dtype=torch.int32)
    Kt0 = layers_a[0][3]
    check_append(Kt0, K, P, [w.T - 8 + 1] * w.B, 1)
    ref_s = oracle.score(q, P, host(Kt0), slh)
    check_selection(host(loop_a.idx[0]).numpy(), host(loop_a.count[0]).numpy(), ref_s, slh.numpy(), w.k)
    ref_o, ref_l = oracle.attend(q, K, V, host(loop_a.idx[0]), host(loop_a.count[0]), slh, w.scale)
    check_attention(loop_a.out[0], loop_a.lse[0], ref_o, ref_l, torch.bfloat16)


# ------------------------------------------- forced sink / recent tokens
@pytest.mark.parametrize("n_sink,n_recent", [(4, 0), (0, 32), (4, 32), (300, 0)])
def test_forced_tokens_every_form(n_sink, n_recent, form):
    """Always-selected first / last tokens: every selection form, the fused
    pass and score + top-k agree bit for bit, and equal the oracle's forced
    top-k on the GPU's own fp32 scores."""
    w, sl = W(B=3, Hkv=2, Hq=8, T=20000, k=256, seed=95), [20000, 3000, 100]
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    idx, cnt = ops.select(qd, Pd, Kt, sld, w.k, n_sink=n_sink, n_recent=n_recent, form=form)
    s = ops.score(qd, Pd, Kt, sld)
    idx2, cnt2 = ops.topk(s, sld, w.k, n_sink=n_sink, n_recent=n_recent, form=form)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(idx).numpy(), host(idx2).numpy())
    np.testing.assert_array_equal(host(cnt).numpy(), host(cnt2).numpy())
    ref_idx, ref_cnt = oracle.topk(host(s).double().numpy(), slh, w.k, n_sink=n_sink, n_recent=n_recent)
    np.testing.assert_array_equal(host(idx).numpy(), ref_idx)
    np.testing.assert_array_equal(host(cnt).numpy(), ref_cnt)


@pytest.mark.parametrize("fused", ["1", "0"])
def test_forced_tokens_decode_step(fused):
    w, sl = W(B=2, T=30000, k=256, seed=96), [30000, 20001]
    (q, K, V, P, slh), (qd, Kd, Vd, Pd, sld) = draw(w, seq_lens=sl)
    pos = (slh - 1).clamp_min(0)
    Kt = ops.build_lowrank_cache(Kd, Pd)
    out, lse, idx, cnt = ops.decode_step(qd, Kd, Vd, Pd, Kt, sld, pos.to(DEV), w.k, w.scale, n_sink=4, n_recent=64,
                                         form="stream", unfused=fused == "0")
    s = ops.score(qd, Pd, Kt, sld)
    torch.cuda.synchronize()
    ref_idx, ref_cnt = oracle.topk(host(s).double().numpy(), slh, w.k, n_sink=4, n_recent=64)
    np.testing.assert_array_equal(host(idx).numpy(), ref_idx)
    ref_o, ref_l = oracle.attend(q, K, V, host(idx), host(cnt), slh, w.scale)
    check_attention(out, lse, ref_o, ref_l, torch.bfloat16)


def test_decode_step_form_choice():
    """The decode step runs as one fused launch where it plans and k <= 256
    (also on short caches and small batches); a larger k keeps the
    three-launch cluster form where that plans; the latent cache takes three
    launches (prologue, cluster selection, attention with the split merge
    inside: its 128 CTAs fit on the GPU at once), four where they do not."""
    from token_level_sparse_kv_b200.inputs import WORKLOADS, Workload

    def form(w):
        dims = ops.Dims()
        dims.B, dims.Hq, dims.Hkv, dims.d, dims.dv, dims.T_cap, dims.r = w.B, w.Hq, w.Hkv, w.d, w.Dv, w.T, w.r
        dims.kv_dtype, dims.kt_dtype = ops.BF16, ops.BF16
        return ops.plan_info(dims, w.k, ops.OP_DECODE_STEP)

    for name in ("gqa_4k_b1", "gqa_32k_b4", "gqa_128k_b16", "hybrid_global_128k_b8"):
        n, text = form(WORKLOADS[name])
        assert n == 1 and "fused" in text, (name, n, text)
    w = WORKLOADS["gqa_128k_b16"]
    n, text = form(Workload(**{**w.__dict__, "B": 1, "k": 1024}))
    assert n == 3 and "cluster" in text, (n, text)
    n, text = form(WORKLOADS["mla_64k_b8"])
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert n == (3 if 16 * 8 <= sms else 4), (n, text)

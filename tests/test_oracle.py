"""Pins for the fp64 CPU oracle (no GPU).

Each test ties an oracle function to something other than itself: a
hand-worked example, a special case that reduces to a library routine
(numpy matmul / lexsort, torch SDPA in fp64), a closed form, or brute force on
tiny inputs.  The cases are chosen so that a dropped term, a wrong sign, a
wrong head/group index or a transposed operand fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from token_level_sparse_kv_b200.inputs import Workload, make_basis, make_inputs


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t):
    return t.to(torch.float64).numpy()


# ------------------------------------------------------------ worked example
@pytest.fixture(scope="module")
def worked(golden_dir):
    with open(os.path.join(golden_dir, "worked_example_small.json")) as f:
        return json.load(f)


def _worked_tensors(w):
    T, d = w["shapes"]["T"], w["shapes"]["d"]
    K = torch.tensor(w["K_rows"], dtype=torch.float32).reshape(1, T, 1, d).to(torch.bfloat16)
    V = torch.tensor(w["V_rows"], dtype=torch.float32).reshape(1, T, 1, d).to(torch.bfloat16)
    q = torch.tensor(w["q_heads"], dtype=torch.float32).reshape(1, 2, d).to(torch.bfloat16)
    P = torch.tensor(w["P_columns"], dtype=torch.float32).T.reshape(1, d, 2).contiguous()
    return q, K, V, P, torch.tensor([T], dtype=torch.int32)


def test_worked_example_append_score_select(worked):
    q, K, V, P, sl = _worked_tensors(worked)
    T = worked["shapes"]["T"]
    Kt = oracle.append_lowrank(K, P, [0], T, kt_dtype=oracle.BF16)
    np.testing.assert_array_equal(oracle.bf16_bits_to_f64(Kt)[0, 0], np.array(worked["Kt"], dtype=np.float64))
    s_sum = oracle.score(q, P, Kt, sl, agg=oracle.AGG_SUM)[0, 0]
    s_max = oracle.score(q, P, Kt, sl, agg=oracle.AGG_MAX)[0, 0]
    np.testing.assert_array_equal(s_sum, worked["scores_sum"])
    np.testing.assert_array_equal(s_max, worked["scores_max"])
    for key, s, k in (("top2_sum", s_sum, 2), ("top3_sum", s_sum, 3), ("top3_max", s_max, 3)):
        idx, cnt = oracle.topk(s.reshape(1, 1, T), sl, k)
        assert idx[0, 0].tolist() == worked[key]
        assert cnt[0, 0] == k


def test_worked_example_attend(worked):
    q, K, V, P, sl = _worked_tensors(worked)
    idx = np.array([[[0, 3, -1]]], dtype=np.int32)
    cnt = np.array([[2]], dtype=np.int32)
    out, lse = oracle.attend(q, K, V, idx, cnt, sl, scale=1.0)
    e, e4 = math.e, math.exp(4.0)
    np.testing.assert_allclose(out[0, 0], [1 / (1 + e), 0, 0, e / (1 + e)], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out[0, 1], [e4 / (1 + e4), 0, 0, 1 / (1 + e4)], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], [2 + math.log1p(math.exp(-1)), 8 + math.log1p(math.exp(-4))],
                               rtol=0, atol=1e-14)


# ----------------------------------------------------------- bf16 rounding
def test_round_bf16_single_rounding_and_ties():
    # exact grid points and ties-to-even around 1.0 (bf16 ulp at 1 is 2^-7)
    assert oracle.round_bf16(1.0) == 1.0
    assert oracle.round_bf16(1.0 + 2**-8) == 1.0  # tie -> even (mantissa 0)
    assert oracle.round_bf16(1.0 + 3 * 2**-8) == 1.0 + 2**-6  # tie -> even (mantissa 2)
    assert oracle.round_bf16(1.0 + 2**-8 + 2**-40) == 1.0 + 2**-7
    # double rounding trap: x rounds to the bf16 tie point in fp32, but is above it in fp64
    x = 1.0 + 2**-8 + 2**-30
    assert float(np.float32(x)) == 1.0 + 2**-8  # fp32 loses the 2^-30
    assert oracle.round_bf16(x) == 1.0 + 2**-7  # a single rounding from fp64 goes up
    # negative values mirror
    assert oracle.round_bf16(-(1.0 + 2**-8 + 2**-40)) == -(1.0 + 2**-7)
    # overflow and the smallest subnormal
    assert math.isinf(oracle.round_bf16(2.0**128))
    assert oracle.round_bf16(2.0**-133) == 2.0**-133
    assert oracle.round_bf16(2.0**-135) == 0.0


def test_round_bf16_matches_torch_on_fp32_values():
    # For inputs that are exact fp32 values a single rounding fp32 -> bf16 is
    # torch's conversion (round to nearest even).
    g = torch.Generator().manual_seed(1)
    x = torch.randn(4000, generator=g) * torch.exp(torch.randn(4000, generator=g) * 8)
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.round_bf16(float(v)) for v in x.tolist()])
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------------ append
def test_append_identity_basis_is_bitwise_copy():
    g = torch.Generator().manual_seed(2)
    B, T, Hkv, d = 2, 9, 3, 8
    K = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    P = torch.eye(d).expand(Hkv, d, d).contiguous()
    Kt = oracle.append_lowrank(K, P, [0, 0], T)
    np.testing.assert_array_equal(Kt, bits(K.permute(0, 2, 1, 3)))


def test_append_column_permutation_per_head_and_partial_range():
    # P[h] selects columns perm_h (d != r): Kt[...,j] = K[..., perm_h[j]] exactly.
    g = torch.Generator().manual_seed(3)
    B, T, Hkv, d, r = 2, 11, 2, 8, 3
    K = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    perms = [[5, 0, 7], [2, 6, 1]]
    P = torch.zeros(Hkv, d, r)
    for h in range(Hkv):
        for j, i in enumerate(perms[h]):
            P[h, i, j] = 1.0
    pos = [4, 7]
    n_new = 3
    Kt = oracle.append_lowrank(K, P, pos, n_new)
    ref = np.zeros_like(Kt)
    kb = bits(K)
    for b in range(B):
        for h in range(Hkv):
            for t in range(pos[b], pos[b] + n_new):
                ref[b, h, t, :] = kb[b, t, h, perms[h]]
    np.testing.assert_array_equal(Kt, ref)


def test_append_general_basis_within_one_rounding():
    # Unrounded sums equal numpy's fp64 matmul to fp64 accuracy, and the stored
    # bf16 value is the nearest-even bf16 of the exact sum.
    w = Workload("t", B=2, Hq=4, Hkv=2, d=32, T=17, r=8, k=4, kind="plain", seed=5)
    q, K, V, P, sl = make_inputs(w)
    Kt, exact = oracle.append_lowrank(K, P, [0, 0], w.T, want_exact=True)
    ref = np.einsum("bthi,hij->bhtj", f64(K), P.to(torch.float64).numpy())
    np.testing.assert_allclose(exact, ref, rtol=1e-13, atol=1e-13)
    got = oracle.bf16_bits_to_f64(Kt)
    ulp = np.ldexp(1.0, np.frexp(np.abs(exact))[1] - 8)
    assert np.all(np.abs(got - exact) <= 0.5 * ulp + 1e-300)


def test_append_fp32_output_rounds_to_nearest():
    w = Workload("t", B=1, Hq=2, Hkv=1, d=16, T=5, r=4, k=2, kind="plain", seed=6)
    q, K, V, P, sl = make_inputs(w, dtype=torch.float32)
    Kt, exact = oracle.append_lowrank(K, P, [0], w.T, kt_dtype=oracle.FP32, want_exact=True)
    np.testing.assert_array_equal(Kt, exact.astype(np.float32))


def test_append_rejects_out_of_range_positions():
    K = torch.zeros(1, 4, 1, 8, dtype=torch.bfloat16)
    P = torch.zeros(1, 8, 8)
    with pytest.raises(ValueError):
        oracle.append_lowrank(K, P, [2], 3)


# ------------------------------------------------------------------- score
def test_score_identity_basis_equals_exact_group_logits():
    # r = d, P = I: Kt = K exactly, and the SUM score is sum_g q_g . K_t and the
    # MAX score is max_g q_g . K_t with the standard GQA grouping g -> g // G.
    w = Workload("t", B=2, Hq=6, Hkv=2, d=16, T=23, r=16, k=5, kind="plain", seed=7)
    q, K, V, _, sl = make_inputs(w)
    P = torch.eye(w.d).expand(w.Hkv, w.d, w.d).contiguous()
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    logits = np.einsum("bgi,bthi->bght", f64(q), f64(K))  # [B, Hq, Hkv, T]
    G = w.G
    ref_sum = np.stack([logits[:, h * G:(h + 1) * G, h, :].sum(1) for h in range(w.Hkv)], 1)
    ref_max = np.stack([logits[:, h * G:(h + 1) * G, h, :].max(1) for h in range(w.Hkv)], 1)
    np.testing.assert_allclose(oracle.score(q, P, Kt, sl, oracle.AGG_SUM), ref_sum, rtol=1e-12, atol=1e-10)
    np.testing.assert_allclose(oracle.score(q, P, Kt, sl, oracle.AGG_MAX), ref_max, rtol=1e-12, atol=1e-10)


def test_score_general_basis_matches_projected_matmul():
    # general P on the stored (rounded) Kt: s = sum_g (q_g P_h) . Kt_t.
    w = Workload("t", B=2, Hq=8, Hkv=2, d=32, T=40, r=8, k=4, seed=8)
    q, K, V, P, sl = make_inputs(w)
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    ktd = oracle.bf16_bits_to_f64(Kt)
    Pd = P.to(torch.float64).numpy()
    G = w.G
    qt = np.einsum("bhgi,hij->bhgj", f64(q).reshape(w.B, w.Hkv, G, w.d), Pd)
    ref = np.einsum("bhgj,bhtj->bht", qt, ktd)
    np.testing.assert_allclose(oracle.score(q, P, Kt, sl), ref, rtol=1e-12, atol=1e-10)


def test_score_masks_tail_and_respects_bh_list():
    w = Workload("t", B=2, Hq=4, Hkv=2, d=16, T=12, r=4, k=3, seed=9)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([5, 12], dtype=torch.int32)
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    full = oracle.score(q, P, Kt, sl)
    assert np.all(np.isneginf(full[0, :, 5:])) and np.all(np.isfinite(full[0, :, :5]))
    part = oracle.score(q, P, Kt, sl, bh_list=[3])
    np.testing.assert_array_equal(part[1, 1], full[1, 1])
    assert np.all(np.isneginf(part[0])) and np.all(np.isneginf(part[1, 0]))


# -------------------------------------------------------------------- topk
def test_topk_matches_subset_brute_force_with_ties():
    rng = np.random.default_rng(10)
    for trial in range(60):
        n = int(rng.integers(1, 10))
        k = int(rng.integers(1, 5))
        vals = rng.integers(-3, 4, size=n).astype(np.float64)  # many exact ties
        if trial % 3 == 0:
            vals = rng.standard_normal(n)
        if trial % 7 == 0:
            vals[:] = 0.0
            vals[::2] = -0.0  # -0.0 and +0.0 are one value
        idx, cnt = oracle.topk(vals.reshape(1, 1, n), [n], k)
        want = brute.topk_by_subsets(vals.tolist(), k)
        assert cnt[0, 0] == min(k, n)
        assert idx[0, 0, :cnt[0, 0]].tolist() == want
        assert np.all(idx[0, 0, cnt[0, 0]:] == -1)


def test_topk_matches_lexsort_and_is_permutation_equivariant():
    rng = np.random.default_rng(11)
    B, Hkv, T, k = 2, 3, 300, 17
    s = rng.standard_normal((B, Hkv, T))
    sl = [T, 250]
    idx, cnt = oracle.topk(s, sl, k)
    for b in range(B):
        for h in range(Hkv):
            tb = sl[b]
            order = np.lexsort((np.arange(tb), -s[b, h, :tb]))[:k]
            assert idx[b, h].tolist() == sorted(order.tolist())
    perm = rng.permutation(T)
    sp = s[:, :, perm]  # token t' = position of t after permutation
    idx2, _ = oracle.topk(sp, [T, T], k)
    inv = np.argsort(perm)
    for h in range(Hkv):
        assert sorted(perm[idx2[0, h]].tolist()) == idx[0, h].tolist()
    assert inv is not None


def test_topk_edge_cases():
    s = np.arange(6, dtype=np.float64).reshape(1, 1, 6)
    idx, cnt = oracle.topk(s, [0], 3)  # empty sequence
    assert cnt[0, 0] == 0 and idx[0, 0].tolist() == [-1, -1, -1]
    idx, cnt = oracle.topk(s, [4], 8)  # k > T_b
    assert cnt[0, 0] == 4 and idx[0, 0].tolist() == [0, 1, 2, 3, -1, -1, -1, -1]
    idx, cnt = oracle.topk(s, [6], 1)
    assert idx[0, 0].tolist() == [5]


# ------------------------------------------------------------------ attend
def _sdpa_ref(q, K, V, sl, scale, window=0, dv=None, latent=False):
    """torch SDPA in fp64 on CPU, GQA heads mapped by repeat_interleave."""
    B, Hq, d = q.shape
    _, T, Hkv, _ = K.shape
    G = Hq // Hkv
    outs, lses = [], []
    for b in range(B):
        tb = int(sl[b])
        lo = max(0, tb - window) if window > 0 else 0
        kb = K[b, lo:tb].to(torch.float64).permute(1, 0, 2)  # [Hkv, n, d]
        vb = (K[b, lo:tb, :, :dv] if latent else V[b, lo:tb]).to(torch.float64).permute(1, 0, 2)
        kb = kb.repeat_interleave(G, 0)
        vb = vb.repeat_interleave(G, 0)
        qb = q[b].to(torch.float64).unsqueeze(1)  # [Hq, 1, d]
        o = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, scale=scale)
        logits = (qb @ kb.transpose(1, 2)).squeeze(1) * scale
        outs.append(o.squeeze(1))
        lses.append(torch.logsumexp(logits, dim=-1))
    return torch.stack(outs).numpy(), torch.stack(lses).numpy()


def test_dense_matches_torch_sdpa_fp64():
    w = Workload("t", B=2, Hq=8, Hkv=2, d=32, T=37, r=8, k=4, seed=12)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([37, 20], dtype=torch.int32)
    out, lse = oracle.dense(q, K, V, sl, scale=0.3)
    ro, rl = _sdpa_ref(q, K, V, sl, 0.3)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_dense_window_matches_torch_sdpa_fp64():
    w = Workload("t", B=2, Hq=4, Hkv=1, d=16, T=40, r=4, k=4, seed=13)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([40, 9], dtype=torch.int32)
    out, lse = oracle.dense(q, K, V, sl, scale=0.25, window=13)
    ro, rl = _sdpa_ref(q, K, V, sl, 0.25, window=13)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_sparse_with_k_equal_T_is_dense():
    w = Workload("t", B=2, Hq=8, Hkv=2, d=32, T=29, r=8, k=29, seed=14)
    q, K, V, P, sl = make_inputs(w)
    Kt, s, idx, cnt, out, lse = oracle.step(q, K, V, P, oracle.append_lowrank(K, P, [0, 0], w.T), sl,
                                            k=w.T, scale=w.scale)
    assert np.all(cnt == w.T)
    dout, dlse = oracle.dense(q, K, V, sl, scale=w.scale)
    np.testing.assert_array_equal(out, dout)
    np.testing.assert_array_equal(lse, dlse)


def test_attend_closed_forms_single_token_and_equal_logits():
    g = torch.Generator().manual_seed(15)
    B, T, Hkv, d, Hq = 1, 8, 1, 16, 2
    K = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    sl = [T]
    # one selected token: o = V_t, lse = scale * q.K_t
    idx = np.array([[[5, -1, -1]]], dtype=np.int32)
    out, lse = oracle.attend(q, K, V, idx, [[1]], sl, scale=0.5)
    np.testing.assert_array_equal(out[0, 0], f64(V[0, 5, 0]))
    np.testing.assert_allclose(lse[0], 0.5 * f64(q[0]) @ f64(K[0, 5, 0]), rtol=0, atol=1e-13)
    # identical key rows: every weight is 1/n, o = mean of the V rows, lse = l + ln n
    K2 = K.clone()
    K2[0, :, 0, :] = K[0, 2, 0, :]
    idx = np.array([[[1, 3, 4, 6]]], dtype=np.int32)
    out, lse = oracle.attend(q, K2, V, idx, [[4]], sl, scale=0.5)
    mean = f64(V[0, [1, 3, 4, 6], 0]).mean(0)
    np.testing.assert_allclose(out[0, 1], mean, rtol=0, atol=1e-14)
    l0 = 0.5 * f64(q[0, 1]) @ f64(K[0, 2, 0])
    np.testing.assert_allclose(lse[0, 1], l0 + math.log(4), rtol=0, atol=1e-13)


def test_attend_matches_python_loops_and_weights_sum_to_one():
    w = Workload("t", B=1, Hq=4, Hkv=2, d=8, T=10, r=4, k=3, seed=16)
    q, K, V, P, sl = make_inputs(w)
    idx = np.array([[[1, 4, 9], [0, 2, -1]]], dtype=np.int32)
    cnt = np.array([[3, 2]], dtype=np.int32)
    out, lse = oracle.attend(q, K, V, idx, cnt, sl, scale=0.7)
    for h in range(2):
        rows = idx[0, h, :cnt[0, h]].tolist()
        Kr = [f64(K[0, t, h]).tolist() for t in rows]
        Vr = [f64(V[0, t, h]).tolist() for t in rows]
        qs = [f64(q[0, h * 2 + g]).tolist() for g in range(2)]
        bo, bl = brute.attention_loops(qs, Kr, Vr, 0.7)
        np.testing.assert_allclose(out[0, 2 * h:2 * h + 2], bo, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, 2 * h:2 * h + 2], bl, rtol=0, atol=1e-13)
    # softmax weights sum to one: with V = all-ones rows the output is exactly 1
    ones = torch.ones_like(V)
    o1, _ = oracle.attend(q, K, ones, idx, cnt, sl, scale=0.7)
    np.testing.assert_allclose(o1, 1.0, rtol=0, atol=1e-14)


def test_attend_empty_and_bad_index():
    w = Workload("t", B=1, Hq=2, Hkv=1, d=8, T=6, r=4, k=2, seed=17)
    q, K, V, P, sl = make_inputs(w)
    out, lse = oracle.attend(q, K, V, np.full((1, 1, 2), -1, np.int32), [[0]], sl, scale=1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    with pytest.raises(ValueError):
        oracle.attend(q, K, V, np.array([[[2, 6]]], np.int32), [[2]], sl, scale=1.0)


def test_latent_cache_dense_matches_sdpa():
    # latent cache (V = first dv dims of the key row), all heads share one KV head
    w = Workload("t", B=2, Hq=8, Hkv=1, d=24, dv=16, T=19, r=8, k=4, latent=True, seed=18)
    q, K, V, P, sl = make_inputs(w)
    assert V is None
    out, lse = oracle.dense(q, K, None, sl, scale=w.scale, dv=16, v_aliases_k=True)
    ro, rl = _sdpa_ref(q, K, None, sl, w.scale, dv=16, latent=True)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_identity_basis_selection_is_exact_topk_of_full_scores():
    # The pages' defining special case: with r = d and P = I the subspace score is
    # the full q.K score, so selection is the exact top-k of the group logits.
    w = Workload("t", B=2, Hq=8, Hkv=2, d=16, T=64, r=16, k=9, seed=19)
    q, K, V, _, sl = make_inputs(w)
    P = torch.eye(w.d).expand(w.Hkv, w.d, w.d).contiguous()
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    _, s, idx, cnt, _, _ = oracle.step(q, K, V, P, Kt, sl, k=w.k, scale=w.scale)
    logits = np.einsum("bgi,bthi->bght", f64(q), f64(K))
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            full = logits[b, h * G:(h + 1) * G, h, :].sum(0)
            order = np.lexsort((np.arange(w.T), -full))[:w.k]
            assert idx[b, h].tolist() == sorted(order.tolist())


def test_basis_is_orthonormal():
    P = make_basis(3, 64, 16, seed=20).to(torch.float64)
    eye = torch.eye(16, dtype=torch.float64)
    for h in range(3):
        torch.testing.assert_close(P[h].T @ P[h], eye, rtol=0, atol=1e-6)


# ------------------------------------------------ forced sink / recent tokens
def _forced_by_lexsort(s, Tb, k, n_sink, n_recent):
    """Independent statement of the forced selection: order the tokens by
    (forced first; among forced tokens by index; among the others by score
    desc, then index) with numpy's lexsort, keep k_b."""
    t = np.arange(Tb)
    forced = (t < n_sink) | (t >= Tb - n_recent)
    kb = min(k, Tb)
    order = np.lexsort((t, np.where(forced, 0.0, -s[:Tb]), ~forced))
    return np.sort(order[:kb])


@pytest.mark.parametrize("n_sink,n_recent", [(0, 0), (4, 0), (0, 16), (4, 16), (30, 30), (200, 0)])
def test_topk_forced_matches_lexsort_statement(n_sink, n_recent):
    rng = np.random.default_rng(100 + n_sink + n_recent)
    B, Hkv, T = 3, 2, 300
    s = rng.normal(size=(B, Hkv, T))
    s[0, 1] = np.round(s[0, 1] * 2) / 2  # heavy exact ties
    sl = np.array([300, 57, 5], dtype=np.int32)
    for k in (1, 16, 64, 400):
        idx, cnt = oracle.topk(s, sl, k, n_sink=n_sink, n_recent=n_recent)
        for b in range(B):
            for h in range(Hkv):
                ref = _forced_by_lexsort(s[b, h], int(sl[b]), k, n_sink, n_recent)
                assert cnt[b, h] == len(ref)
                np.testing.assert_array_equal(idx[b, h, :len(ref)], ref)
                assert np.all(idx[b, h, len(ref):] == -1)


def test_topk_forced_plain_case_and_invariants():
    rng = np.random.default_rng(7)
    s = rng.normal(size=(1, 1, 500))
    sl = np.array([500], dtype=np.int32)
    i0, c0 = oracle.topk(s, sl, 64)
    i1, c1 = oracle.topk(s, sl, 64, n_sink=0, n_recent=0)
    np.testing.assert_array_equal(i0, i1)
    idx, cnt = oracle.topk(s, sl, 64, n_sink=4, n_recent=8)
    sel = set(idx[0, 0].tolist())
    forced = set(range(4)) | set(range(492, 500))
    assert forced <= sel and cnt[0, 0] == 64
    rest = sorted(sel - forced)
    outside = [t for t in range(500) if t not in sel and t not in forced]
    assert min(s[0, 0, rest]) >= max(s[0, 0, outside])  # the free slots hold the best of the rest
    # forced tokens alone exceed k: the smallest forced indices
    idx, cnt = oracle.topk(s, sl, 6, n_sink=4, n_recent=8)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 492, 493]


# ------------------------------------- per-query-head selection (variant)
def test_score_heads_matches_projected_matmul_and_group_relations():
    # s[b,g,t] = (q_g P_h) . Kt_t with h = g // G, against an independent
    # numpy statement; the SUM / MAX group scores are the sum / max of the
    # group's rows (a dropped head, a wrong group index or a transposed P fails)
    w = Workload("t", B=2, Hq=8, Hkv=2, d=32, T=40, r=8, k=4, seed=108)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([40, 23], dtype=torch.int32)
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    ktd = oracle.bf16_bits_to_f64(Kt)
    G = w.G
    qt = np.einsum("bgi,gij->bgj", f64(q), np.repeat(P.to(torch.float64).numpy(), G, axis=0))
    ref = np.einsum("bgj,bgtj->bgt", qt, np.repeat(ktd, G, axis=1))
    ref[1, :, 23:] = -np.inf
    sh = oracle.score_heads(q, P, Kt, sl)
    np.testing.assert_allclose(sh, ref, rtol=1e-12, atol=1e-10)
    s_sum = oracle.score(q, P, Kt, sl, oracle.AGG_SUM)
    s_max = oracle.score(q, P, Kt, sl, oracle.AGG_MAX)
    fin = np.isfinite(s_sum)
    grp = sh.reshape(w.B, w.Hkv, G, w.T)
    np.testing.assert_allclose(grp.sum(2)[fin], s_sum[fin], rtol=1e-12, atol=1e-10)
    np.testing.assert_array_equal(grp.max(2), s_max)


def test_score_heads_with_one_head_per_kv_head_is_the_group_score():
    w = Workload("t", B=2, Hq=3, Hkv=3, d=16, T=30, r=8, k=4, seed=109)
    q, K, V, P, sl = make_inputs(w)
    Kt = oracle.append_lowrank(K, P, [0, 0], w.T)
    np.testing.assert_array_equal(oracle.score_heads(q, P, Kt, sl), oracle.score(q, P, Kt, sl))


def test_per_head_topk_matches_subset_brute_force():
    # tiny T: each query head's own top-k equals the k-subset optimum of its
    # own scores, and differs from the group's shared set where the heads disagree
    w = Workload("t", B=1, Hq=4, Hkv=1, d=16, T=9, r=16, k=3, kind="plain", seed=110)
    q, K, V, _, sl = make_inputs(w)
    P = torch.eye(w.d).unsqueeze(0).contiguous()
    Kt = oracle.append_lowrank(K, P, [0], w.T)
    sh = oracle.score_heads(q, P, Kt, sl)
    idx, cnt = oracle.topk(sh, sl, w.k)
    for g in range(w.Hq):
        assert idx[0, g].tolist() == brute.topk_by_subsets(sh[0, g].tolist(), w.k)
        assert cnt[0, g] == w.k
    logits = np.einsum("gi,ti->gt", f64(q[0]), f64(K[0, :, 0]))  # P = I: exact q_g . K_t
    np.testing.assert_allclose(sh[0], logits, rtol=1e-12, atol=1e-12)


def test_attend_heads_reduces_to_attend_and_to_loops():
    w = Workload("t", B=2, Hq=6, Hkv=2, d=16, T=25, r=8, k=7, seed=111)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([25, 9], dtype=torch.int32)
    g = np.random.default_rng(5)
    G = w.G
    # shared lists (every head of a KV head on its group's list) equal oracle_attend
    idx = np.full((w.B, w.Hkv, w.k), -1, np.int32)
    cnt = np.zeros((w.B, w.Hkv), np.int32)
    for b in range(w.B):
        for h in range(w.Hkv):
            c = min(w.k, int(sl[b])) - h
            cnt[b, h] = c
            idx[b, h, :c] = np.sort(g.choice(int(sl[b]), c, replace=False))
    o1, l1 = oracle.attend(q, K, V, idx, cnt, sl, w.scale)
    o2, l2 = oracle.attend_heads(q, K, V, np.repeat(idx, G, axis=1), np.repeat(cnt, G, axis=1), sl, w.scale)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # distinct per-head lists against pure-Python loops (head g reads KV head g // G)
    hidx = np.full((w.B, w.Hq, w.k), -1, np.int32)
    hcnt = np.zeros((w.B, w.Hq), np.int32)
    for b in range(w.B):
        for hq in range(w.Hq):
            c = int(g.integers(0, min(w.k, int(sl[b])) + 1))
            hcnt[b, hq] = c
            hidx[b, hq, :c] = np.sort(g.choice(int(sl[b]), c, replace=False))
    o, l = oracle.attend_heads(q, K, V, hidx, hcnt, sl, w.scale)
    Kf, Vf, qf = f64(K), f64(V), f64(q)
    for b in range(w.B):
        for hq in range(w.Hq):
            rows = hidx[b, hq, :hcnt[b, hq]]
            ro, rl = brute.attention_loops([qf[b, hq].tolist()], [Kf[b, t, hq // G].tolist() for t in rows],
                                           [Vf[b, t, hq // G].tolist() for t in rows], w.scale)
            if len(rows):
                np.testing.assert_allclose(o[b, hq], ro[0], rtol=1e-12, atol=1e-13)
                assert abs(l[b, hq] - rl[0]) < 1e-12
            else:
                assert np.all(o[b, hq] == 0) and np.isneginf(l[b, hq])


# ------------------------------------------ calibration of P (NEXT-4 reading)
from oracle import calib  # noqa: E402


def test_calib_key_positions_rule():
    assert calib.key_positions(5, 8).tolist() == [0, 1, 2, 3, 4]
    p = calib.key_positions(1000, 7)
    assert p[0] == 0 and np.all(np.diff(p) > 0) and p[-1] < 1000
    assert p.tolist() == [j * 1000 // 7 for j in range(7)]


def test_calib_moments_match_explicit_loops():
    w = Workload("t", B=2, Hq=4, Hkv=2, d=4, T=9, r=2, k=2, seed=140)
    q, K, V, P, _ = make_inputs(w)
    sl = torch.tensor([9, 5], dtype=torch.int32)
    Sq, Sk = calib.moments(q[:1], K, sl, n_keys=3)
    qf, Kf = f64(q), f64(K)
    for h in range(2):
        ref_q = [[0.0] * 4 for _ in range(4)]
        for g in (2 * h, 2 * h + 1):
            for i in range(4):
                for j in range(4):
                    ref_q[i][j] += qf[0, g, i] * qf[0, g, j]
        np.testing.assert_allclose(Sq[h], ref_q, rtol=1e-15, atol=1e-15)
        ref_k = [[0.0] * 4 for _ in range(4)]
        for b, tb in ((0, 9), (1, 5)):
            for t in ([0, 3, 6] if tb == 9 else [0, 1, 3]):
                for i in range(4):
                    for j in range(4):
                        ref_k[i][j] += Kf[b, t, h, i] * Kf[b, t, h, j]
        np.testing.assert_allclose(Sk[h], ref_k, rtol=1e-15, atol=1e-15)
    M = calib.joint_matrix(Sq, Sk)
    np.testing.assert_allclose([np.trace(M[h]) for h in range(2)], [2.0, 2.0], rtol=1e-14)
    np.testing.assert_allclose(M, np.transpose(M, (0, 2, 1)), rtol=0, atol=0)


def test_calib_recovers_a_planted_subspace():
    # queries and keys drawn inside a 3-dim subspace U of R^16: M has rank 3
    # and the top-r (r = 5) basis contains U exactly (principal angles 0)
    g = torch.Generator().manual_seed(141)
    d, r0, r = 16, 3, 5
    U = torch.linalg.qr(torch.randn(d, r0, generator=g, dtype=torch.float64))[0]
    q = (torch.randn(6, 2, r0, generator=g, dtype=torch.float64) @ U.T).to(torch.float32)
    K = (torch.randn(1, 50, 1, r0, generator=g, dtype=torch.float64) @ U.T).to(torch.float32)
    Pc, lam, M = calib.calibrate(q, K, torch.tensor([50], dtype=torch.int32), r, n_keys=20)
    Ud = U.numpy()
    assert abs(np.linalg.norm(Ud.T @ Pc[0]) ** 2 - r0) < 1e-9
    assert np.all(lam[0, r0:] < 1e-9)
    np.testing.assert_allclose(calib.captured_energy(M, Pc), lam[:, :r].sum(1), rtol=1e-12)

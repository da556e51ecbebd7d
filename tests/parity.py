"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (written here once, used by every GPU test):
  * low-rank append: the stored value is one rounding (<= 1 ulp of the
    storage grid) away from a value within the fp32 accumulation bound
    (d * 2^-24 * sum |terms|) of the exact sum, and equals the oracle's
    round-to-nearest-even value in all but 0.1 % of the elements (fp32
    accumulation moves sums that lie close to a bf16 tie, or close to zero);
  * scores: |gpu - exact| <= 1e-5 * (sum of |terms|) + 1e-6 (fp32 dot products
    of length r after an fp32 projection of length d);
  * selection: exact ties and near-ties may resolve differently in fp32 and
    fp64, so with s_k the oracle's k-th score and tau = 1e-3 * max(|s_k|,
    rms(s)), every token above s_k + tau must be selected, none below
    s_k - tau may be, and the counts are equal;
  * attention output: max |gpu - oracle| <= 2e-2 with bf16 K/V (fp32
    accumulation; the output itself is stored in bf16), 1e-4 with fp32 K/V;
    lse within 1e-3;
  * end to end (the oracle's own low-rank cache, fp64 scores, selection and
    attention against the GPU's step): the selection rule above against the
    oracle's own scores for every (b, h), and the output rule wherever the
    two index sets are identical.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

OUT_TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
LSE_TOL = 1e-3
SEL_REL = 1e-3


def host(t):
    return t.detach().cpu()


def check_append(Kt_gpu: torch.Tensor, K_host, P_host, pos, n_new):
    """Compare GPU low-rank rows with the oracle's (exact sums and RNE values)."""
    kt_code = oracle.BF16 if Kt_gpu.dtype == torch.bfloat16 else oracle.FP32
    ref, exact = oracle.append_lowrank(K_host, P_host, pos, n_new, kt_dtype=kt_code, want_exact=True)
    got, _ = oracle.raw(host(Kt_gpu))
    B = ref.shape[0]
    mask = np.zeros(ref.shape[:3], dtype=bool)
    for b in range(B):
        mask[b, :, pos[b]:pos[b] + n_new] = True
    g, r, e = got[mask], ref[mask], exact[mask]
    # fp32 accumulation error bound of a length-d dot product: d * 2^-24 * sum |terms|
    Pa = np.abs(np.asarray(P_host, np.float64))
    d = Pa.shape[1]
    Kf = oracle.to_f64(K_host)
    absum = np.concatenate([np.einsum("thi,hij->htj", np.abs(Kf[b, pos[b]:pos[b] + n_new]), Pa).reshape(-1, Pa.shape[2])
                            for b in range(B)])
    acc_err = d * 2.0**-24 * absum
    if kt_code == oracle.BF16:
        gv = oracle.bf16_bits_to_f64(g)
        ulp = np.ldexp(1.0, np.maximum(np.frexp(np.abs(e))[1] - 8, -133))
        # one rounding of a value within the fp32 accumulation error of the exact sum
        assert np.all(np.abs(gv - e) <= ulp + acc_err), "a bf16 value is further than one rounding from the sum"
        # the rate of rounding-boundary cases is a statistical bound: a
        # sample of a few hundred elements may hold one
        ndiff = int(np.sum(g != r))
        assert ndiff <= max(1, 1e-3 * g.size), "%d of %d elements differ from round-to-nearest-even" % (ndiff, g.size)
    else:
        assert np.all(np.abs(g.astype(np.float64) - e) <= acc_err + np.abs(e) * 2.0**-24)
    return got


def check_scores(s_gpu: np.ndarray, s_ref: np.ndarray, scale_ref: np.ndarray):
    ok = np.isfinite(s_ref)
    err = np.abs(s_gpu[ok].astype(np.float64) - s_ref[ok])
    bound = 1e-5 * scale_ref[ok] + 1e-6
    assert np.all(err <= bound), "score error %.3g above bound" % float((err - bound).max())


def check_selection(idx_gpu, cnt_gpu, s_ref, seq_lens, k):
    """Tie-window rule against oracle scores s_ref [B,Hkv,T] (fp64)."""
    idx_gpu = np.asarray(idx_gpu)
    cnt_gpu = np.asarray(cnt_gpu)
    B, Hkv, _ = s_ref.shape
    n_diff_sets = 0
    for b in range(B):
        tb = int(seq_lens[b])
        kb = min(k, tb)
        for h in range(Hkv):
            assert int(cnt_gpu[b, h]) == kb, "count %d != %d at (%d,%d)" % (cnt_gpu[b, h], kb, b, h)
            sel = idx_gpu[b, h, :kb]
            assert np.all(idx_gpu[b, h, kb:] == -1)
            if kb == 0:
                continue
            assert np.all(np.diff(sel) > 0), "indices not strictly ascending"
            assert sel.min() >= 0 and sel.max() < tb
            s = s_ref[b, h, :tb]
            order = np.lexsort((np.arange(tb), -s))
            sk = s[order[kb - 1]]
            tau = SEL_REL * max(abs(sk), float(np.sqrt(np.mean(s * s))))
            chosen = np.zeros(tb, dtype=bool)
            chosen[sel] = True
            must = s > sk + tau
            never = s < sk - tau
            assert np.all(chosen[must]), "a token clearly above the k-th score is missing at (%d,%d)" % (b, h)
            assert not np.any(chosen[never]), "a token clearly below the k-th score is selected at (%d,%d)" % (b, h)
            if not np.array_equal(np.sort(order[:kb]), sel):
                n_diff_sets += 1
    return n_diff_sets


def check_attention(out_gpu, lse_gpu, out_ref, lse_ref, dtype):
    o = host(out_gpu).to(torch.float64).numpy()
    err = np.abs(o - out_ref)
    tol = OUT_TOL[dtype]
    assert err.max() <= tol, "max |out - oracle| = %.3g > %.3g" % (err.max(), tol)
    if lse_gpu is not None:
        l = host(lse_gpu).to(torch.float64).numpy()
        both_inf = np.isneginf(l) & np.isneginf(lse_ref)
        assert np.all(np.isneginf(l) == np.isneginf(lse_ref)), "empty-set lse mismatch"
        d = np.abs(np.where(both_inf, 0.0, l - np.where(both_inf, 0.0, lse_ref)))
        assert d.max() <= LSE_TOL, "max |lse - oracle| = %.3g" % d.max()
    return float(err.max())


def check_end_to_end(out_gpu, lse_gpu, idx_gpu, cnt_gpu, s_or, idx_or, out_or, lse_or, seq_lens, k, G):
    """GPU step vs the oracle's own step.  Every (b, h) selection obeys the
    tie-window rule against the oracle's own fp64 scores; every difference
    between the two index sets lies inside the window (rule 4); outputs (and
    lse) agree within the attention tolerance wherever the sets are
    identical.  Returns the number of (b, h) sets that differ."""
    def arr(x):
        return host(x).numpy() if isinstance(x, torch.Tensor) else np.asarray(x)

    ig = arr(idx_gpu)
    n_diff = check_selection(ig, arr(cnt_gpu), s_or, arr(seq_lens), k)
    B, Hkv, _ = ig.shape
    o = host(out_gpu).double().numpy()
    l = host(lse_gpu).double().numpy() if lse_gpu is not None else None
    same = np.all(ig == arr(idx_or), axis=2)
    for b in range(B):
        for h in range(Hkv):
            if not same[b, h]:
                continue
            rows = slice(h * G, (h + 1) * G)
            err = np.abs(o[b, rows] - out_or[b, rows]).max()
            assert err <= OUT_TOL[torch.bfloat16], "end-to-end output error %.3g at (%d,%d)" % (err, b, h)
            if l is not None:
                fin = np.isfinite(lse_or[b, rows])
                assert np.array_equal(np.isfinite(l[b, rows]), fin)
                assert np.abs(l[b, rows][fin] - lse_or[b, rows][fin]).max(initial=0.0) <= LSE_TOL
    assert n_diff == int((~same).sum())
    return n_diff

"""Calibration of the shared query-key basis P (TEST INFRASTRUCTURE ONLY).

The step before the decode path: "Joint Subspace Sparse Attention for
Efficient Long-Context Decoding", Abstract (a spectral solution for a shared
low-dimensional query-key subspace), and the news item "JSSA makes token-level
sparse decoding gather-free", Interpretation para 2 (the subspace preserves
queries and keys jointly).  The pages give neither the objective nor its
closed form; the reading restated here is the plainest spectral one:

    S_q(h) = sum of q q^T over the sampled queries of the G heads of KV head h
    S_k(h) = sum of k k^T over the sampled keys of KV head h
    M(h)   = S_q / tr(S_q) + S_k / tr(S_k)          (each term dropped if its trace is 0)
    P(h)   = an orthonormal basis of the top-r eigenvectors of M(h)

i.e. the r-dimensional subspace that keeps the most of the (trace-normalised)
energy of queries and keys together.  The selection score q^T P P^T k depends
on P only through its span, so any basis of that subspace is equivalent.

Sampled keys (the same rule as the CUDA path): for every batch row b, n tokens
t_j = floor(j * T_b / n), j < n (all t < T_b when T_b <= n).  Sampled queries:
every row of q_cal [N, Hq, d] of the group's heads.

Plain numpy in fp64; numpy.linalg.eigh is the library step.  Nothing here is
shared with the CUDA sources.
"""
from __future__ import annotations

import numpy as np

from . import to_f64


def key_positions(Tb: int, n: int) -> np.ndarray:
    if Tb <= n:
        return np.arange(Tb, dtype=np.int64)
    return (np.arange(n, dtype=np.int64) * Tb) // n


def moments(q_cal, K, seq_lens, n_keys):
    """(S_q, S_k), each [Hkv, d, d] fp64, for q_cal [N, Hq, d] and K [B, T, Hkv, d]."""
    q = to_f64(q_cal)
    Kf = to_f64(K)
    N, Hq, d = q.shape
    B, T, Hkv, _ = Kf.shape
    G = Hq // Hkv
    Sq = np.zeros((Hkv, d, d))
    Sk = np.zeros((Hkv, d, d))
    for h in range(Hkv):
        Qh = q[:, h * G:(h + 1) * G, :].reshape(-1, d)
        Sq[h] = Qh.T @ Qh
        for b in range(B):
            Tb = min(int(seq_lens[b]), T)
            rows = Kf[b, key_positions(Tb, n_keys), h, :]
            Sk[h] += rows.T @ rows
    return Sq, Sk


def joint_matrix(Sq, Sk):
    """M = S_q / tr(S_q) + S_k / tr(S_k) per head (a zero-trace term dropped)."""
    M = np.zeros_like(Sq)
    for h in range(Sq.shape[0]):
        tq, tk = np.trace(Sq[h]), np.trace(Sk[h])
        if tq > 0:
            M[h] += Sq[h] / tq
        if tk > 0:
            M[h] += Sk[h] / tk
    return M


def calibrate(q_cal, K, seq_lens, r, n_keys):
    """(P [Hkv, d, r], eigenvalues [Hkv, d] descending, M [Hkv, d, d])."""
    Sq, Sk = moments(q_cal, K, seq_lens, n_keys)
    M = joint_matrix(Sq, Sk)
    Hkv, d, _ = M.shape
    P = np.zeros((Hkv, d, r))
    lam = np.zeros((Hkv, d))
    for h in range(Hkv):
        w, V = np.linalg.eigh(M[h])  # ascending
        order = np.argsort(w)[::-1]
        lam[h] = w[order]
        P[h] = V[:, order[:r]]
    return P, lam, M


def captured_energy(M, P):
    """tr(P^T M P) per head: the joint energy an orthonormal basis keeps."""
    return np.array([np.trace(P[h].T @ M[h] @ P[h]) for h in range(M.shape[0])])

"""Float64 CPU oracle of the BACKWARD pass of differential attention (numpy).

TEST INFRASTRUCTURE, like the rest of this package: only the test suite, the package smoke
check and the benchmark's CPU-baseline / reference leg may import it.

What it differentiates. The pages present lambda as a learnable per-head scalar, built
from four learnable vectors ("Differential Attention (V2)", Key Terms, "lambda"; Hugging
Face post on the DIFF Transformer, "How?"), inside attention layers that are pre-trained
("Differential Attention (V2)", "V1 vs V2"). Training needs the gradient of the forward
operator with respect to its inputs; that gradient is fixed by the forward definition and
calculus alone. The forward is the one the C oracle computes:

    A_b = softmax(Q_b K_b^T / sqrt(d) + mask)        b = 1, 2 (row-wise)
    O   = A_1 V - lambda A_2 V
    V1: y = (1 - lambda_init) O / sqrt(mean_c O^2 + eps)   (per row and head)
    V2: y = O

Every map is materialised here (no blocking, no online softmax). Given dy = dL/dy:

    V1 norm:  r = sqrt(mean O^2 + eps),  dO = s/r (dy - O (dy . O) / (n r^2)),  s = 1 - lambda_init
    dV      = A_1^T dO - lambda A_2^T dO
    dA_1    = dO V^T,        dA_2 = -lambda dO V^T
    dS_b    = A_b * (dA_b - rowsum(A_b * dA_b))              (softmax backward)
    dQ_b    = dS_b K_b / sqrt(d),  dK_b = dS_b^T Q_b / sqrt(d)
    dlambda = -sum(dO * (A_2 V))
    lambda vectors: dlq1 = dlambda e1 lk1, dlk1 = dlambda e1 lq1, dlq2 = -dlambda e2 lk2,
                    dlk2 = -dlambda e2 lq2, with e_b = exp(lq_b . lk_b)

V2 pairs share a KV head: dK and dV of a KV head sum over every query head that reads it.
Masks follow the forward: queries at the last Nq of Nk positions, causal, optional window.
"""
from __future__ import annotations

import numpy as np


def _mask(Nq: int, Nk: int, causal: bool, window: int) -> np.ndarray:
    """True where query i (at position i + Nk - Nq) attends key j."""
    pos = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    m = np.ones((Nq, Nk), dtype=bool)
    if causal:
        m &= j <= pos
        if window > 0:
            m &= j > pos - window
    return m


def _softmax(s: np.ndarray, mask: np.ndarray) -> np.ndarray:
    s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def _branch_pair_bwd(q1, q2, k1, k2, v, lam, dO, mask):
    """One (batch, head-pair) problem: q_b [Nq,d], k_b [Nk,d], v [Nk,dv], dO [Nq,dv]
    (the gradient reaching O = A_1 V - lam A_2 V). Returns dq1, dq2, dk1, dk2, dv, dlam."""
    d = q1.shape[1]
    sc = 1.0 / np.sqrt(d)
    a1 = _softmax(q1 @ k1.T * sc, mask)
    a2 = _softmax(q2 @ k2.T * sc, mask)
    dv = a1.T @ dO - lam * (a2.T @ dO)
    da1 = dO @ v.T
    da2 = -lam * da1
    ds1 = a1 * (da1 - (a1 * da1).sum(axis=-1, keepdims=True))
    ds2 = a2 * (da2 - (a2 * da2).sum(axis=-1, keepdims=True))
    dq1, dq2 = ds1 @ k1 * sc, ds2 @ k2 * sc
    dk1, dk2 = ds1.T @ q1 * sc, ds2.T @ q2 * sc
    dlam = -float(np.sum(dO * (a2 @ v)))
    return dq1, dq2, dk1, dk2, dv, dlam


def _o_pair(q1, q2, k1, k2, v, lam, mask):
    d = q1.shape[1]
    sc = 1.0 / np.sqrt(d)
    return _softmax(q1 @ k1.T * sc, mask) @ v - lam * (_softmax(q2 @ k2.T * sc, mask) @ v)


def _norm_bwd(o: np.ndarray, dy: np.ndarray, scale: float, eps: float) -> np.ndarray:
    """Gradient through y = scale * o / sqrt(mean(o^2) + eps), row-wise."""
    n = o.shape[-1]
    r = np.sqrt((o * o).mean(axis=-1, keepdims=True) + eps)
    dot = (dy * o).sum(axis=-1, keepdims=True)
    return scale / r * (dy - o * dot / (n * r * r))


def prefill_v1_bwd(q, k, v, lam, lambda_init_value: float, dy, causal=True, apply_norm=True,
                   eps=1e-5, window=0):
    """V1. q [B,Nq,H,2,d]; k [B,Nk,H,2,d]; v [B,Nk,H,2d]; lam [H]; dy [B,Nq,H,2d].
    Returns dq, dk, dv (shapes of q, k, v) and dlam [H]."""
    q, k, v, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dy))
    lam = np.asarray(lam, dtype=np.float64)
    B, Nq, H, _, d = q.shape
    Nk = k.shape[1]
    mask = _mask(Nq, Nk, causal, window)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlam = np.zeros(H)
    for b in range(B):
        for h in range(H):
            q1, q2 = q[b, :, h, 0], q[b, :, h, 1]
            k1, k2 = k[b, :, h, 0], k[b, :, h, 1]
            vv = v[b, :, h]
            g = dy[b, :, h]
            if apply_norm:
                o = _o_pair(q1, q2, k1, k2, vv, lam[h], mask)
                g = _norm_bwd(o, g, 1.0 - lambda_init_value, eps)
            dq1, dq2, dk1, dk2, dvv, dl = _branch_pair_bwd(q1, q2, k1, k2, vv, lam[h], g, mask)
            dq[b, :, h, 0], dq[b, :, h, 1] = dq1, dq2
            dk[b, :, h, 0], dk[b, :, h, 1] = dk1, dk2
            dv[b, :, h] = dvv
            dlam[h] += dl
    return dq, dk, dv, dlam


def prefill_v2_bwd(q, k, v, lam, dy, causal=True, window=0):
    """V2. q [B,Nq,Hq,d]; k, v [B,Nk,Hkv,d]; lam [Hq/2]; dy [B,Nq,Hq/2,d].
    Pair p = query heads 2p, 2p+1 over KV head 2p // (Hq/Hkv). Returns dq, dk, dv, dlam."""
    q, k, v, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dy))
    lam = np.asarray(lam, dtype=np.float64)
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    group = Hq // Hkv
    mask = _mask(Nq, Nk, causal, window)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlam = np.zeros(Hq // 2)
    for b in range(B):
        for p in range(Hq // 2):
            g = (2 * p) // group
            kk, vv = k[b, :, g], v[b, :, g]
            dq1, dq2, dk1, dk2, dvv, dl = _branch_pair_bwd(q[b, :, 2 * p], q[b, :, 2 * p + 1], kk, kk,
                                                         vv, lam[p], dy[b, :, p], mask)
            dq[b, :, 2 * p], dq[b, :, 2 * p + 1] = dq1, dq2
            dk[b, :, g] += dk1 + dk2
            dv[b, :, g] += dvv
            dlam[p] += dl
    return dq, dk, dv, dlam


def lambda_bwd(lq1, lk1, lq2, lk2, dlam):
    """Gradients of the four [H, dim] lambda vectors from dL/dlambda [H]."""
    lq1, lk1, lq2, lk2 = (np.asarray(x, dtype=np.float64) for x in (lq1, lk1, lq2, lk2))
    dlam = np.asarray(dlam, dtype=np.float64)[:, None]
    e1 = np.exp((lq1 * lk1).sum(axis=-1, keepdims=True))
    e2 = np.exp((lq2 * lk2).sum(axis=-1, keepdims=True))
    return dlam * e1 * lk1, dlam * e1 * lq1, -dlam * e2 * lk2, -dlam * e2 * lq2

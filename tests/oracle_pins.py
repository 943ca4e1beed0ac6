"""Pins of the float64 oracle to things other than itself.

Each pin raises AssertionError when the oracle disagrees with what the pages or the
mathematics fix. tests/test_oracle_pins.py runs them against the oracle as built, and
tests/test_oracle_mutants.py runs them against copies of the oracle source with one
planted mistake each, expecting every mutant to fail at least one pin.

Independent references used here (none of them is the oracle's code):
  * torch.nn.functional.scaled_dot_product_attention in float64 on the CPU -- lambda = 0
    reduces differential attention to standard (causal) softmax attention;
  * torch.softmax / matmul / rms_norm in float64 -- the printed operator
    (A_1 - lambda A_2) V ("Attention Variants", Build It, Step 4) evaluated by a library;
  * mpmath at 40 digits, exp / sum without max-subtraction -- brute force on tiny inputs;
  * closed forms: row sums, identical branches, the first causal row, lambda values for
    chosen vectors, the lambda_init schedule's end points;
  * the pages' noise-cancellation claim on a length-1024 signal-plus-noise sequence.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
from differential_attention_05_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa(q, k, v, causal):
    """q [B,H,N,d] f64 -> standard softmax attention (library routine)."""
    d = q.shape[-1]
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal,
        scale=1.0 / math.sqrt(d)).numpy()


def _close(a, b, tol, what):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---- lambda and lambda_init ----------------------------------------------------------

def pin_lambda_init_schedule():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "lambda_init.txt"))
            if ln.strip() and not ln.startswith("#")]
    for depth, value, tol in rows:
        dep = 400 if depth == "inf" else int(depth)
        _close(oracle.lambda_init(dep), float(value), float(tol), f"lambda_init(depth={depth})")
    vals = [oracle.lambda_init(dd) for dd in range(1, 40)]
    assert all(b > a for a, b in zip(vals, vals[1:])), "lambda_init must rise with depth"


def pin_lambda_closed_form():
    """Vectors whose dot products are ln 3 and ln 2 give exp terms 3 and 2 exactly;
    cross products (lq1.lk2, lq2.lk1) are zero, so a swapped pairing gives 0."""
    d = 6
    lq1 = np.zeros((3, d)); lk1 = np.zeros((3, d)); lq2 = np.zeros((3, d)); lk2 = np.zeros((3, d))
    # head 0: lambda = 3 - 2 + li
    lq1[0, 0], lk1[0, 0] = math.log(3.0), 1.0
    lq2[0, 1], lk2[0, 1] = 2.0, math.log(2.0) / 2.0
    # head 1: all zero -> 1 - 1 + li
    # head 2: lambda = 1 - 5 + li  (negative: "can be negative")
    lq2[2, 3], lk2[2, 3] = math.log(5.0), 1.0
    # lambda_init at depths 1 and 2, evaluated by hand from the schedule (tests/golden/lambda_init.txt)
    for depth, li in ((1, 0.2), (2, 0.355509067591)):
        lam = oracle.lambda_(lq1, lk1, lq2, lk2, depth)
        _close(lam, [1.0 + li, li, -4.0 + li], 1e-11, f"lambda closed form (depth {depth})")
        assert lam[2] < 0


# ---- softmax attention special case (lambda = 0) -------------------------------------

def pin_lambda0_is_softmax_attention_v1():
    r = _rng(1)
    B, N, H, d = 2, 37, 3, 8
    q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
    v = r.standard_normal((B, N, H, 2 * d))
    lam = np.zeros(H)
    for causal in (True, False):
        out = oracle.prefill_v1(q, k, v, lam, 0.3, causal=causal, apply_norm=False, threads=2)
        ref = _sdpa(q[:, :, :, 0].transpose(0, 2, 1, 3).copy(), k[:, :, :, 0].transpose(0, 2, 1, 3).copy(),
                    v.transpose(0, 2, 1, 3).copy(), causal).transpose(0, 2, 1, 3)
        _close(out, ref, 1e-12, f"V1 lambda=0 vs SDPA (causal={causal})")


def pin_lambda0_is_softmax_attention_v2():
    r = _rng(2)
    B, N, Hq, Hkv, d = 2, 29, 8, 2, 16
    q = r.standard_normal((B, N, Hq, d)); k = r.standard_normal((B, N, Hkv, d))
    v = r.standard_normal((B, N, Hkv, d))
    lam = np.zeros(Hq // 2)
    group = Hq // Hkv
    for causal in (True, False):
        out = oracle.prefill_v2(q, k, v, lam, causal=causal, threads=2)
        kk = np.repeat(k, group, axis=2)  # query head h reads KV head h // group
        vv = np.repeat(v, group, axis=2)
        ref = _sdpa(q.transpose(0, 2, 1, 3).copy(), kk.transpose(0, 2, 1, 3).copy(),
                    vv.transpose(0, 2, 1, 3).copy(), causal).transpose(0, 2, 1, 3)
        _close(out, ref[:, :, 0::2], 1e-12, f"V2 lambda=0 vs SDPA on heads 2p (causal={causal})")


def pin_lambda0_decode_is_softmax_attention():
    r = _rng(3)
    B, L, Hq, Hkv, d = 3, 41, 8, 2, 16
    q = r.standard_normal((B, Hq, d)); k = r.standard_normal((B, L, Hkv, d))
    v = r.standard_normal((B, L, Hkv, d))
    kv_len = np.array([41, 1, 17], dtype=np.int32)
    out = oracle.decode_v2(q, k, v, np.zeros(Hq // 2), kv_len=kv_len, threads=2)
    group = Hq // Hkv
    for b in range(B):
        n = kv_len[b]
        kk = np.repeat(k[b, :n], group, axis=1).transpose(1, 0, 2)[None].copy()
        vv = np.repeat(v[b, :n], group, axis=1).transpose(1, 0, 2)[None].copy()
        ref = _sdpa(q[b][None, :, None, :].copy(), kk, vv, False)[0, :, 0, :]
        _close(out[b], ref[0::2], 1e-12, f"decode lambda=0 vs SDPA (b={b}, kv_len={n})")


def pin_lambda0_decode_v1_is_softmax_attention():
    """V1 decode with lambda = 0 and no norm: branch 1's softmax attention over the cache
    (K_1 from the first half of each cached key row, V the whole 2d row)."""
    r = _rng(11)
    B, L, H, d = 2, 29, 3, 8
    q = r.standard_normal((B, H, 2, d)); k = r.standard_normal((B, L, H, 2, d))
    v = r.standard_normal((B, L, H, 2 * d))
    kv_len = np.array([29, 5], dtype=np.int32)
    out = oracle.decode_v1(q, k, v, np.zeros(H), 0.3, kv_len=kv_len, apply_norm=False, threads=2)
    for b in range(B):
        n = kv_len[b]
        ref = _sdpa(q[b, :, 0][None, :, None, :].copy(), k[b, :n, :, 0].transpose(1, 0, 2)[None].copy(),
                    v[b, :n].transpose(1, 0, 2)[None].copy(), False)[0, :, 0, :]
        _close(out[b], ref, 1e-12, f"V1 decode lambda=0 vs SDPA (b={b}, kv_len={n})")


def pin_decode_v1_is_last_prefill_row():
    """A V1 decode step for a query at cache position n - 1 equals the last causal prefill
    row over the same n keys, norm and scale included."""
    r = _rng(12)
    B, L, H, d = 2, 24, 2, 8
    k = r.standard_normal((B, L, H, 2, d)); v = r.standard_normal((B, L, H, 2 * d))
    q = r.standard_normal((B, H, 2, d))
    lam = np.array([0.7, -0.4])
    kv_len = np.array([24, 9], dtype=np.int32)
    out = oracle.decode_v1(q, k, v, lam, 0.55, kv_len=kv_len, threads=2)
    for b in range(B):
        n = kv_len[b]
        qq = r.standard_normal((1, n, H, 2, d))
        qq[0, n - 1] = q[b]
        pre = oracle.prefill_v1(qq, k[b:b + 1, :n], v[b:b + 1, :n], lam, 0.55, threads=1)
        _close(out[b], pre[0, n - 1], 1e-13, f"V1 decode vs last prefill row (b={b})")


# ---- invariants of the difference -----------------------------------------------------

def pin_identical_branches_cancel():
    """Q1 = Q2, K1 = K2 and lambda = 1: (A_1 - A_2) V = 0 before the norm."""
    r = _rng(4)
    B, N, H, d = 1, 23, 2, 8
    q1 = r.standard_normal((B, N, H, 1, d)); k1 = r.standard_normal((B, N, H, 1, d))
    q = np.concatenate([q1, q1], axis=3); k = np.concatenate([k1, k1], axis=3)
    v = r.standard_normal((B, N, H, 2 * d))
    out = oracle.prefill_v1(q, k, v, np.ones(H), 0.2, apply_norm=False, threads=1)
    _close(out, 0.0, 1e-15, "V1 identical branches, lambda=1")
    Hq, Hkv = 4, 2
    qv = r.standard_normal((B, N, Hq // 2, d))
    q2 = np.repeat(qv, 2, axis=2)  # heads 2p and 2p+1 equal
    k2 = r.standard_normal((B, N, Hkv, d)); v2 = r.standard_normal((B, N, Hkv, d))
    out2 = oracle.prefill_v2(q2, k2, v2, np.ones(Hq // 2), threads=1)
    _close(out2, 0.0, 1e-15, "V2 identical branches, lambda=1")
    out3 = oracle.decode_v1(q[:, 5], k, v, np.ones(H), 0.2, kv_len=[17], apply_norm=False, threads=1)
    _close(out3, 0.0, 1e-15, "V1 decode identical branches, lambda=1")


def pin_rows_sum_to_one_minus_lambda():
    """Every softmax row sums to 1, so with V = 1 each output channel is 1 - lambda."""
    r = _rng(5)
    B, N, H, d = 1, 19, 3, 4
    q = r.standard_normal((B, N, H, 2, d)) * 3; k = r.standard_normal((B, N, H, 2, d)) * 3
    v = np.ones((B, N, H, 2 * d))
    lam = np.array([0.0, 0.8, -1.7])
    for causal in (True, False):
        out = oracle.prefill_v1(q, k, v, lam, 0.2, causal=causal, apply_norm=False, threads=1)
        _close(out, np.broadcast_to((1.0 - lam)[None, None, :, None], out.shape), 1e-13,
               f"V1 rows sum to 1 - lambda (causal={causal})")
    Hq, Hkv = 8, 4
    q2 = r.standard_normal((B, N, Hq, d)); k2 = r.standard_normal((B, N, Hkv, d))
    lam2 = np.array([0.5, 1.0, 0.2, -0.3])
    out2 = oracle.prefill_v2(q2, k2, np.ones((B, N, Hkv, d)), lam2, threads=1)
    _close(out2, np.broadcast_to((1.0 - lam2)[None, None, :, None], out2.shape), 1e-13,
           "V2 rows sum to 1 - lambda")
    out3 = oracle.decode_v2(q2[:, 0], k2, np.ones((B, N, Hkv, d)), lam2, kv_len=[7], threads=1)
    _close(out3, np.broadcast_to((1.0 - lam2)[None, :, None], out3.shape), 1e-13,
           "decode rows sum to 1 - lambda")
    out4 = oracle.decode_v1(q[:, 3], q, v, lam, 0.2, kv_len=[11], apply_norm=False, threads=1)
    _close(out4, np.broadcast_to((1.0 - lam)[None, :, None], out4.shape), 1e-13,
           "V1 decode rows sum to 1 - lambda")


def pin_norm_first_row_closed_form():
    """Causal row 0 sees only key 0: o = (1-lambda) v0, then RMSNorm and (1 - lambda_init):
    out_0 = (1-lambda) v0 / sqrt((1-lambda)^2 mean(v0^2) + eps) * (1 - lambda_init).
    The second case makes mean(o^2) comparable to eps so a dropped eps shows."""
    r = _rng(6)
    B, N, H, d = 1, 5, 2, 8
    q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
    lam = np.array([0.35, -0.6])
    li, eps = 0.43, 1e-5
    for vscale in (1.0, 2e-3):
        v = r.standard_normal((B, N, H, 2 * d)) * vscale
        out = oracle.prefill_v1(q, k, v, lam, li, apply_norm=True, eps=eps, threads=1)
        for h in range(H):
            v0 = v[0, 0, h]
            o = (1 - lam[h]) * v0
            ref = o / np.sqrt(np.mean(o * o) + eps) * (1 - li)
            _close(out[0, 0, h], ref, 1e-13, f"first-row norm closed form (scale {vscale})")


def pin_printed_operator_with_library_ops():
    """(A_1 - lambda A_2) V with A_b from torch.softmax over the causal mask, then
    torch's rms_norm and the (1 - lambda_init) factor -- for V1 with distinct branches."""
    r = _rng(7)
    B, N, H, d = 1, 33, 2, 8
    q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
    v = r.standard_normal((B, N, H, 2 * d))
    lam = np.array([0.7, 0.25]); li, eps = 0.6, 1e-5
    T = torch.from_numpy
    mask = torch.ones(N, N, dtype=torch.bool).tril()
    ref = np.zeros((B, N, H, 2 * d))
    for h in range(H):
        def amap(b):
            s = T(q[0, :, h, b]) @ T(k[0, :, h, b]).T / math.sqrt(d)
            return torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
        o = (amap(0) - lam[h] * amap(1)) @ T(v[0, :, h])
        o = torch.nn.functional.rms_norm(o, (2 * d,), eps=eps) * (1 - li)
        ref[0, :, h] = o.numpy()
    out = oracle.prefill_v1(q, k, v, lam, li, apply_norm=True, eps=eps, threads=2)
    _close(out, ref, 1e-12, "printed operator via torch ops")
    rows = [0, 5, 32, 17]
    out_rows = oracle.prefill_v1(q, k, v, lam, li, apply_norm=True, eps=eps, rows=rows, threads=1)
    _close(out_rows, ref[:, rows], 1e-12, "row-sampled oracle")


def pin_brute_force_tiny():
    """N <= 8, d in {1, 2, 4}: 40-digit mpmath, exp and sums taken directly (no maximum
    subtracted), weights A_1 - lambda A_2 formed explicitly."""
    import mpmath
    mpmath.mp.dps = 40
    r = _rng(8)
    for (N, d) in ((1, 1), (2, 1), (5, 2), (8, 4)):
        B, H = 1, 1
        q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
        v = r.standard_normal((B, N, H, 2 * d))
        lam = np.array([0.77])
        out = oracle.prefill_v1(q, k, v, lam, 0.1, apply_norm=False, threads=1)
        for i in range(N):
            def row(b):
                e = [mpmath.e ** (mpmath.fsum(mpmath.mpf(q[0, i, 0, b, c]) * mpmath.mpf(k[0, j, 0, b, c])
                                              for c in range(d)) / mpmath.sqrt(d)) for j in range(i + 1)]
                s = mpmath.fsum(e)
                return [x / s for x in e]
            a1, a2 = row(0), row(1)
            w = [a1[j] - mpmath.mpf(lam[0]) * a2[j] for j in range(i + 1)]
            ref = [float(mpmath.fsum(w[j] * mpmath.mpf(v[0, j, 0, c]) for j in range(i + 1)))
                   for c in range(2 * d)]
            _close(out[0, i, 0], ref, 1e-14, f"brute force N={N} d={d} row {i}")


# ---- noise cancellation (the pages' measurement) --------------------------------------

def _snr_gains(lam, stride=37):
    """Median SNR gain (differential over plain softmax) over query rows past the planted
    key. SNR = weight on the signal key / mean |weight| on unrelated keys."""
    cfg = {ln.split()[0]: ln.split()[1] for ln in open(os.path.join(GOLDEN, "snr_claim.txt"))
           if ln.strip() and not ln.startswith("#")}
    N = int(cfg["length"])
    inp = synth.signal_plus_noise(N=N, Hq=8, Hkv=1, d=128, seed=5)
    q = inp.as_f64("q")[0]; k = inp.as_f64("k")[0]
    pos = inp.extra["planted_pos"]
    gains, plain_mass, diff_mass = [], [], []
    for p in range(4):
        s = int(pos[0, p])
        for i in range(s + 1, N, stride):
            a1, a2 = oracle.map_row_v2(q, k, p, i)
            w = a1 - lam * a2
            n = i  # unrelated keys visible to row i
            plain = a1[s] / ((a1.sum() - a1[s]) / n)
            diff = w[s] / ((np.abs(w).sum() - abs(w[s])) / n)
            gains.append(diff / plain)
            plain_mass.append(a1.sum() - a1[s])
            diff_mass.append(w.sum() - w[s])
    return float(np.median(gains)), float(np.mean(plain_mass)), float(np.mean(diff_mass)), cfg


def pin_noise_cancellation():
    g0, plain_mass, _, cfg = _snr_gains(0.0)
    assert abs(g0 - 1.0) < 1e-12, "lambda = 0 must be plain softmax"
    assert plain_mass > 0.5, f"plain softmax noise mass {plain_mass:.3f} should be O(1)"
    lam = float(cfg["lambda"])
    g, _, diff_mass, _ = _snr_gains(lam)
    assert float(cfg["gain_min"]) <= g <= float(cfg["gain_max"]), f"SNR gain {g:.2f} outside claim"
    assert abs(diff_mass) < 0.25 * plain_mass, (
        f"differential noise mass {diff_mass:.3f} not well below plain {plain_mass:.3f}")
    sweep = [_snr_gains(x)[0] for x in (0.0, 0.5, 0.8, 0.9)]
    assert all(b > a for a, b in zip(sweep, sweep[1:])), f"lambda ablation not rising: {sweep}"


ALL_PINS = [
    pin_lambda_init_schedule,
    pin_lambda_closed_form,
    pin_lambda0_is_softmax_attention_v1,
    pin_lambda0_is_softmax_attention_v2,
    pin_lambda0_decode_is_softmax_attention,
    pin_lambda0_decode_v1_is_softmax_attention,
    pin_decode_v1_is_last_prefill_row,
    pin_identical_branches_cancel,
    pin_rows_sum_to_one_minus_lambda,
    pin_norm_first_row_closed_form,
    pin_printed_operator_with_library_ops,
    pin_brute_force_tiny,
    pin_noise_cancellation,
]


def pin_compact_query_rows():
    """Sampled rows given as a compact query array equal the same rows of the full run
    (bookkeeping check of the row-sampling path used at full sizes)."""
    r = _rng(9)
    B, N, H, d = 2, 40, 2, 8
    q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
    v = r.standard_normal((B, N, H, 2 * d))
    lam = np.array([0.4, 0.9])
    rows = [39, 0, 17]
    full = oracle.prefill_v1(q, k, v, lam, 0.5, threads=1)
    comp = oracle.prefill_v1(None, k, v, lam, 0.5, rows=rows, q_rows=q[:, rows], threads=1)
    _close(comp, full[:, rows], 0.0, "V1 compact rows")
    Hq, Hkv = 8, 2
    q2 = r.standard_normal((B, N, Hq, d)); k2 = r.standard_normal((B, N, Hkv, d))
    v2 = r.standard_normal((B, N, Hkv, d)); lam2 = r.standard_normal(Hq // 2)
    full2 = oracle.prefill_v2(q2, k2, v2, lam2, threads=1)
    comp2 = oracle.prefill_v2(None, k2, v2, lam2, rows=rows, q_rows=q2[:, rows], threads=1)
    _close(comp2, full2[:, rows], 0.0, "V2 compact rows")


ALL_PINS.append(pin_compact_query_rows)


def pin_chunked_prefill_is_last_rows():
    """Nq < Nk queries (a chunk after Nk - Nq cached positions) equal the last Nq rows of
    the full causal prefill whose last Nq queries are the chunk's (V1 and V2)."""
    r = _rng(13)
    B, Nk, Nq, H, d = 2, 45, 17, 2, 8
    qf = r.standard_normal((B, Nk, H, 2, d)); k = r.standard_normal((B, Nk, H, 2, d))
    v = r.standard_normal((B, Nk, H, 2 * d)); lam = np.array([0.6, -0.2])
    full = oracle.prefill_v1(qf, k, v, lam, 0.4, threads=1)
    part = oracle.prefill_v1(qf[:, Nk - Nq:].copy(), k, v, lam, 0.4, threads=1)
    _close(part, full[:, Nk - Nq:], 1e-13, "V1 chunk = last rows")
    Hq, Hkv = 8, 2
    qf2 = r.standard_normal((B, Nk, Hq, d)); k2 = r.standard_normal((B, Nk, Hkv, d))
    v2 = r.standard_normal((B, Nk, Hkv, d)); lam2 = r.standard_normal(Hq // 2)
    full2 = oracle.prefill_v2(qf2, k2, v2, lam2, threads=1)
    part2 = oracle.prefill_v2(qf2[:, Nk - Nq:].copy(), k2, v2, lam2, threads=1)
    _close(part2, full2[:, Nk - Nq:], 1e-13, "V2 chunk = last rows")


def pin_window_lambda0_is_banded_attention():
    """lambda = 0 with a causal sliding window of W keys: softmax attention under the band
    mask pos - W < j <= pos (torch SDPA with an explicit boolean mask), chunked queries
    included."""
    r = _rng(14)
    B, Nk, Nq, H, d, W = 1, 40, 25, 2, 8, 7
    q = r.standard_normal((B, Nq, H, 2, d)); k = r.standard_normal((B, Nk, H, 2, d))
    v = r.standard_normal((B, Nk, H, 2 * d))
    out = oracle.prefill_v1(q, k, v, np.zeros(H), 0.3, apply_norm=False, window=W, threads=1)
    pos = np.arange(Nq)[:, None] + (Nk - Nq)
    j = np.arange(Nk)[None, :]
    mask = torch.from_numpy((j <= pos) & (j > pos - W))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[:, :, :, 0].transpose(0, 2, 1, 3).copy()),
        torch.from_numpy(k[:, :, :, 0].transpose(0, 2, 1, 3).copy()),
        torch.from_numpy(v.transpose(0, 2, 1, 3).copy()), attn_mask=mask,
        scale=1.0 / math.sqrt(d)).numpy().transpose(0, 2, 1, 3)
    _close(out, ref, 1e-12, "V1 window lambda=0 vs banded SDPA")
    Hq, Hkv = 4, 2
    q2 = r.standard_normal((B, Nq, Hq, d)); k2 = r.standard_normal((B, Nk, Hkv, d))
    v2 = r.standard_normal((B, Nk, Hkv, d))
    out2 = oracle.prefill_v2(q2, k2, v2, np.zeros(Hq // 2), window=W, threads=1)
    kk = np.repeat(k2, 2, axis=2).transpose(0, 2, 1, 3).copy()
    vv = np.repeat(v2, 2, axis=2).transpose(0, 2, 1, 3).copy()
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q2.transpose(0, 2, 1, 3).copy()), torch.from_numpy(kk),
        torch.from_numpy(vv), attn_mask=mask, scale=1.0 / math.sqrt(d)).numpy().transpose(0, 2, 1, 3)
    _close(out2, ref2[:, :, 0::2], 1e-12, "V2 window lambda=0 vs banded SDPA")


def pin_window_extremes():
    """A window as long as the sequence changes nothing; a window of one key leaves
    o = (1 - lambda) v_pos (then the V1 norm and scale)."""
    r = _rng(15)
    B, N, H, d = 1, 21, 2, 8
    q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
    v = r.standard_normal((B, N, H, 2 * d)); lam = np.array([0.3, 0.9])
    plain = oracle.prefill_v1(q, k, v, lam, 0.5, threads=1)
    _close(oracle.prefill_v1(q, k, v, lam, 0.5, window=N, threads=1), plain, 0.0, "window = N")
    one = oracle.prefill_v1(q, k, v, lam, 0.5, apply_norm=False, window=1, threads=1)
    _close(one, (1.0 - lam)[None, None, :, None] * v, 1e-14, "window = 1")


ALL_PINS += [pin_chunked_prefill_is_last_rows, pin_window_lambda0_is_banded_attention,
             pin_window_extremes]


# ---- paged KV cache ------------------------------------------------------------------

def pin_paged_decode_is_contiguous_decode():
    """A paged cache is a storage layout: decoding it over a shuffled page pool gives, bit
    for bit, the contiguous cache's result. Rows past kv_len and spare pages hold NaN, so a
    read outside the entry's own keys would show."""
    r = _rng(16)
    B, L, Hq, Hkv, d = 3, 37, 8, 2, 4
    q = r.standard_normal((B, Hq, d)); k = r.standard_normal((B, L, Hkv, d))
    v = r.standard_normal((B, L, Hkv, d)); lam = r.uniform(-0.5, 1.0, Hq // 2)
    kv_len = np.array([37, 1, 20], dtype=np.int32)
    kn, vn = k.copy(), v.copy()
    for b in range(B):
        kn[b, kv_len[b]:] = np.nan
        vn[b, kv_len[b]:] = np.nan
    for ps in (1, 4, 16, 64):
        (kp, vp), bt = synth.paginate([kn, vn], ps, seed=ps)
        got = oracle.decode_v2_paged(q, kp, vp, bt, lam, kv_len, threads=1)
        _close(got, oracle.decode_v2(q, k, v, lam, kv_len=kv_len, threads=1), 0.0, f"V2 page {ps}")
    H = 2
    q1 = r.standard_normal((B, H, 2, d)); k1 = r.standard_normal((B, L, H, 2, d))
    v1 = r.standard_normal((B, L, H, 2 * d)); lam1 = np.array([0.2, 0.7])
    k1n, v1n = k1.copy(), v1.copy()
    for b in range(B):
        k1n[b, kv_len[b]:] = np.nan
        v1n[b, kv_len[b]:] = np.nan
    (kp, vp), bt = synth.paginate([k1n, v1n], 8, seed=3)
    got = oracle.decode_v1_paged(q1, kp, vp, bt, lam1, 0.4, kv_len, threads=1)
    want = oracle.decode_v1(q1, k1, v1, lam1, 0.4, kv_len=kv_len, threads=1)
    _close(got, want, 0.0, "V1 paged")


ALL_PINS += [pin_paged_decode_is_contiguous_decode]


# ---- variable-length batch -----------------------------------------------------------

def pin_varlen_equal_lengths_is_batched():
    """Packing B sequences of one length back to back gives the fixed-length batch's rows,
    for plain prompts (nq = nk) and for chunks (nq < nk), V1 and V2."""
    r = _rng(17)
    B, Nq, Nk, H, d = 3, 5, 9, 2, 4
    lam = np.array([0.4, -0.2])
    cu_q = np.arange(B + 1) * Nq
    cu_k = np.arange(B + 1) * Nk
    q = r.standard_normal((B, Nq, H, 2, d)); k = r.standard_normal((B, Nk, H, 2, d))
    v = r.standard_normal((B, Nk, H, 2 * d))
    got = oracle.prefill_v1_varlen(q.reshape(B * Nq, H, 2, d), k.reshape(B * Nk, H, 2, d),
                                   v.reshape(B * Nk, H, 2 * d), cu_q, cu_k, lam, 0.3, threads=1)
    want = oracle.prefill_v1(q, k, v, lam, 0.3, threads=1)
    _close(got, want.reshape(B * Nq, H, 2 * d), 0.0, "V1 packed")
    Hq, Hkv = 4, 2
    q2 = r.standard_normal((B, Nq, Hq, d)); k2 = r.standard_normal((B, Nk, Hkv, d))
    v2 = r.standard_normal((B, Nk, Hkv, d))
    got = oracle.prefill_v2_varlen(q2.reshape(B * Nq, Hq, d), k2.reshape(B * Nk, Hkv, d),
                                   v2.reshape(B * Nk, Hkv, d), cu_q, cu_k, lam, window=3, threads=1)
    want = oracle.prefill_v2(q2, k2, v2, lam, window=3, threads=1)
    _close(got, want.reshape(B * Nq, Hq // 2, d), 0.0, "V2 packed")


ALL_PINS += [pin_varlen_equal_lengths_is_batched]


# ---- backward ------------------------------------------------------------------------

from oracle import backward as OB  # noqa: E402


def _fd(f, x, h=1e-5):
    """Central differences of the scalar function f at every element of array x."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        x0 = x[i]
        x[i] = x0 + h
        fp = f()
        x[i] = x0 - h
        fm = f()
        x[i] = x0
        g[i] = (fp - fm) / (2 * h)
    return g


def pin_backward_finite_differences():
    """The backward oracle against central differences of the FORWARD C oracle (a separate
    code base) on tiny inputs: V1 with the norm and a chunk (Nq < Nk), V2 with GQA and a
    window; then the lambda vectors through the lambda oracle."""
    r = _rng(18)
    B, Nq, Nk, H, d = 1, 3, 5, 2, 3
    q = r.standard_normal((B, Nq, H, 2, d)); k = r.standard_normal((B, Nk, H, 2, d))
    v = r.standard_normal((B, Nk, H, 2 * d)); lam = np.array([0.35, -0.2]); li = 0.3
    R = r.standard_normal((B, Nq, H, 2 * d))
    loss = lambda: float(np.sum(oracle.prefill_v1(q, k, v, lam, li, eps=1e-3, threads=1) * R))
    dq, dk, dv, dl = OB.prefill_v1_bwd(q, k, v, lam, li, R, eps=1e-3)
    for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv), ("dlambda", lam, dl)):
        _close(g, _fd(loss, x), 2e-7, f"V1 {name}")
    Hq, Hkv, Nq2, Nk2 = 4, 1, 4, 6
    q = r.standard_normal((B, Nq2, Hq, d)); k = r.standard_normal((B, Nk2, Hkv, d))
    v = r.standard_normal((B, Nk2, Hkv, d)); lam = np.array([0.6, 0.1])
    R = r.standard_normal((B, Nq2, Hq // 2, d))
    loss = lambda: float(np.sum(oracle.prefill_v2(q, k, v, lam, window=3, threads=1) * R))
    dq, dk, dv, dl = OB.prefill_v2_bwd(q, k, v, lam, R, window=3)
    for name, x, g in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv), ("dlambda", lam, dl)):
        _close(g, _fd(loss, x), 2e-7, f"V2 {name}")
    vecs = [0.3 * r.standard_normal((Hq // 2, 4)) for _ in range(4)]
    dlam = r.standard_normal(Hq // 2)
    lossl = lambda: float(np.sum(oracle.lambda_(*vecs, depth=2) * dlam))
    for x, g in zip(vecs, OB.lambda_bwd(*vecs, dlam)):
        _close(g, _fd(lossl, x), 2e-7, "lambda vectors")


def pin_backward_autograd():
    """The backward oracle against torch autograd (float64) through the printed operator
    (softmax, matmul, rms_norm), causal and full, V1 and V2 with GQA."""
    r = _rng(19)
    B, N, H, d = 2, 7, 2, 4
    for causal in (True, False):
        q = r.standard_normal((B, N, H, 2, d)); k = r.standard_normal((B, N, H, 2, d))
        v = r.standard_normal((B, N, H, 2 * d)); lam = np.array([0.8, -0.3]); li = 0.45
        dy = r.standard_normal((B, N, H, 2 * d))
        tq, tk, tv, tl = (torch.tensor(x, requires_grad=True) for x in (q, k, v, lam))
        mask = torch.ones(N, N, dtype=torch.bool).tril() if causal else torch.ones(N, N, dtype=torch.bool)
        def attn(qb, kb):
            s = torch.einsum("bihd,bjhd->bhij", qb, kb) / math.sqrt(d)
            return torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
        a1, a2 = attn(tq[:, :, :, 0], tk[:, :, :, 0]), attn(tq[:, :, :, 1], tk[:, :, :, 1])
        vv = tv.permute(0, 2, 1, 3)
        o = (a1 @ vv - tl[None, :, None, None] * (a2 @ vv)).permute(0, 2, 1, 3)
        y = torch.nn.functional.rms_norm(o, (2 * d,), eps=1e-5) * (1 - li)
        (y * torch.tensor(dy)).sum().backward()
        got = OB.prefill_v1_bwd(q, k, v, lam, li, dy, causal=causal)
        for g, t, name in zip(got, (tq, tk, tv, tl), ("dq", "dk", "dv", "dlambda")):
            _close(g, t.grad.numpy(), 1e-11, f"V1 autograd {name} causal={causal}")
        Hq, Hkv = 8, 2
        q = r.standard_normal((B, N, Hq, d)); k = r.standard_normal((B, N, Hkv, d))
        v = r.standard_normal((B, N, Hkv, d)); lam = r.uniform(-0.5, 1, Hq // 2)
        dy = r.standard_normal((B, N, Hq // 2, d))
        tq, tk, tv, tl = (torch.tensor(x, requires_grad=True) for x in (q, k, v, lam))
        kr = tk.repeat_interleave(Hq // Hkv, dim=2)
        vr = tv.repeat_interleave(Hq // Hkv, dim=2)
        a = attn(tq, kr)                                   # [B, Hq, N, N]
        o = a @ vr.permute(0, 2, 1, 3)                     # [B, Hq, N, d]
        y = (o[:, 0::2] - tl[None, :, None, None] * o[:, 1::2]).permute(0, 2, 1, 3)
        (y * torch.tensor(dy)).sum().backward()
        got = OB.prefill_v2_bwd(q, k, v, lam, dy, causal=causal)
        for g, t, name in zip(got, (tq, tk, tv, tl), ("dq", "dk", "dv", "dlambda")):
            _close(g, t.grad.numpy(), 1e-11, f"V2 autograd {name} causal={causal}")


ALL_PINS += [pin_backward_finite_differences, pin_backward_autograd]

"""Float64 CPU oracle for differential attention (ctypes wrapper over diffattn_oracle.c).

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's
CPU-baseline / reference leg may import this module. The product package never imports
it, and nothing here is shared with the CUDA path.

The C source states, function by function, which passage of the pages each step
follows. This wrapper only converts numpy arrays to contiguous float64 and calls it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "diffattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_libs: dict = {}
_active = None


def compile_source(src: str, out: str) -> str:
    """gcc, IEEE float64, no fast-math, no FMA contraction."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
         "-fno-fast-math", "-o", tmp, src, "-lm", "-lpthread"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile diffattn_oracle.c into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


class use_library:
    """Context manager that points this module at another build of the oracle source
    (used by the tests that plant a mistake in a copy of the oracle)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _active
        self._prev = _active
        _active = self.path
        return self

    def __exit__(self, *exc):
        global _active
        _active = self._prev
        return False


def _load():
    path = _active or build()
    lib = _libs.get(path)
    if lib is None:
        lib = ctypes.CDLL(os.path.abspath(path))
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_lambda_init.restype = ctypes.c_double
        lib.oracle_lambda_init.argtypes = [ctypes.c_int]
        lib.oracle_lambda.restype = ctypes.c_int
        lib.oracle_lambda.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp]
        lib.oracle_prefill_v1.restype = ctypes.c_int
        lib.oracle_prefill_v1.argtypes = [dp, dp, dp, dp, ctypes.c_double] + [ctypes.c_int] * 6 + [
            ctypes.c_double, ip, ctypes.c_int, ctypes.c_int, dp, ctypes.c_int]
        lib.oracle_prefill_v2.restype = ctypes.c_int
        lib.oracle_prefill_v2.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 6 + [
            ip, ctypes.c_int, ctypes.c_int, dp, ctypes.c_int]
        lib.oracle_prefill_v1_range.restype = ctypes.c_int
        lib.oracle_prefill_v1_range.argtypes = [dp, dp, dp, dp, ctypes.c_double] + [ctypes.c_int] * 8 + [
            ctypes.c_double, ip, ctypes.c_int, ctypes.c_int, dp, ctypes.c_int]
        lib.oracle_prefill_v2_range.restype = ctypes.c_int
        lib.oracle_prefill_v2_range.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 8 + [
            ip, ctypes.c_int, ctypes.c_int, dp, ctypes.c_int]
        lib.oracle_decode_v2.restype = ctypes.c_int
        lib.oracle_decode_v2.argtypes = [dp, dp, dp, ip, dp] + [ctypes.c_int] * 5 + [dp, ctypes.c_int]
        lib.oracle_decode_v1.restype = ctypes.c_int
        lib.oracle_decode_v1.argtypes = [dp, dp, dp, ip, dp, ctypes.c_double] + [ctypes.c_int] * 5 + [
            ctypes.c_double, dp, ctypes.c_int]
        lib.oracle_map_row_v2.restype = ctypes.c_int
        lib.oracle_map_row_v2.argtypes = [dp, dp] + [ctypes.c_int] * 6 + [dp, dp]
        _libs[path] = lib
    return lib


def _f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        raise TypeError("bf16 bit patterns must be converted to values before the oracle sees them")
    return np.ascontiguousarray(a, dtype=np.float64)


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def lambda_init(depth: int) -> float:
    return float(_load().oracle_lambda_init(int(depth)))


def lambda_(lq1, lk1, lq2, lk2, depth: int) -> np.ndarray:
    """lambda per head from the four [H, d] re-parameterisation vectors."""
    a = [_f64(x) for x in (lq1, lk1, lq2, lk2)]
    H, d = a[0].shape
    out = np.zeros(H, dtype=np.float64)
    rc = _load().oracle_lambda(*[_dp(x) for x in a], H, d, int(depth), _dp(out))
    if rc != 0:
        raise ValueError(f"oracle_lambda failed: {rc}")
    return out


def _rows(rows, N):
    if rows is None:
        return None, N
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    return r, int(r.size)


def prefill_v1(q, k, v, lam, lambda_init_value: float, causal=True, apply_norm=True,
               eps=1e-5, rows=None, threads=None, q_rows=None, window=0,
               n_queries=None) -> np.ndarray:
    """V1 prefill. q: [B,Nq,H,2,d]; k: [B,Nk,H,2,d]; v: [B,Nk,H,2d]; lam: [H]
    -> out [B,R,H,2d]. Nq <= Nk queries are the last Nq positions (chunked prefill); a
    causal sliding window of `window` keys when window > 0. With rows and q_rows
    ([B,R,H,2,d], the queries at those positions), q may be None (then Nq = n_queries,
    default Nk)."""
    k, v, lam = _f64(k), _f64(v), _f64(lam)
    B, Nk, H, two, d = k.shape
    assert two == 2 and v.shape == (B, Nk, H, 2 * d) and lam.shape == (H,)
    compact = q_rows is not None
    if compact:
        Nq = int(n_queries or Nk)
        r, R = _rows(rows, Nq)
        assert r is not None
        q = _f64(q_rows)
        assert q.shape == (B, R, H, 2, d)
    else:
        q = _f64(q)
        Nq = q.shape[1]
        r, R = _rows(rows, Nq)
        assert q.shape == (B, Nq, H, 2, d)
    out = np.zeros((B, R, H, 2 * d), dtype=np.float64)
    rc = _load().oracle_prefill_v1_range(_dp(q), _dp(k), _dp(v), _dp(lam), float(lambda_init_value),
                                         B, Nq, Nk, H, d, int(bool(causal)), int(window),
                                         int(bool(apply_norm)), float(eps), _ip(r), R, int(compact),
                                         _dp(out), int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_prefill_v1_range failed: {rc}")
    return out


def prefill_v2(q, k, v, lam, causal=True, rows=None, threads=None, q_rows=None, window=0,
               n_queries=None) -> np.ndarray:
    """V2 prefill. q: [B,Nq,Hq,d]; k,v: [B,Nk,Hkv,d]; lam: [Hq/2] -> out [B,R,Hq/2,d].
    Nq <= Nk, window as for prefill_v1. With rows and q_rows ([B,R,Hq,d]), q may be None."""
    k, v, lam = _f64(k), _f64(v), _f64(lam)
    B, Nk, Hkv, d = k.shape
    assert v.shape == k.shape
    compact = q_rows is not None
    if compact:
        Nq = int(n_queries or Nk)
        r, R = _rows(rows, Nq)
        assert r is not None
        q = _f64(q_rows)
        assert q.shape[:2] == (B, R) and q.shape[3] == d
    else:
        q = _f64(q)
        Nq = q.shape[1]
        r, R = _rows(rows, Nq)
        assert q.shape[0] == B and q.shape[3] == d
    Hq = q.shape[2]
    assert lam.shape == (Hq // 2,)
    out = np.zeros((B, R, Hq // 2, d), dtype=np.float64)
    rc = _load().oracle_prefill_v2_range(_dp(q), _dp(k), _dp(v), _dp(lam), B, Nq, Nk, Hq, Hkv, d,
                                         int(bool(causal)), int(window), _ip(r), R, int(compact),
                                         _dp(out), int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_prefill_v2_range failed: {rc}")
    return out


def _varlen(run, q, k, v, cu_q, cu_k, out_width):
    """A variable-length batch is its sequences run one by one: sequence s is rows
    cu_q[s]..cu_q[s+1] of q (and of the result) over rows cu_k[s]..cu_k[s+1] of k, v."""
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.zeros((q.shape[0],) + out_width, dtype=np.float64)
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        if q1 > q0:
            out[q0:q1] = run(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1])[0]
    return out


def prefill_v1_varlen(q, k, v, cu_q, cu_k, lam, lambda_init_value: float, causal=True,
                      apply_norm=True, eps=1e-5, window=0, threads=None) -> np.ndarray:
    """V1 prefill of packed sequences. q: [Tq,H,2,d]; k: [Tk,H,2,d]; v: [Tk,H,2d]
    -> [Tq,H,2d] (rows of no sequence stay 0)."""
    H, d = q.shape[1], q.shape[3]
    run = lambda qq, kk, vv: prefill_v1(qq, kk, vv, lam, lambda_init_value, causal=causal,
                                        apply_norm=apply_norm, eps=eps, window=window,
                                        threads=threads)
    return _varlen(run, q, k, v, cu_q, cu_k, (H, 2 * d))


def prefill_v2_varlen(q, k, v, cu_q, cu_k, lam, causal=True, window=0, threads=None) -> np.ndarray:
    """V2 prefill of packed sequences. q: [Tq,Hq,d]; k,v: [Tk,Hkv,d] -> [Tq,Hq/2,d]."""
    Hq, d = q.shape[1], q.shape[2]
    run = lambda qq, kk, vv: prefill_v2(qq, kk, vv, lam, causal=causal, window=window,
                                        threads=threads)
    return _varlen(run, q, k, v, cu_q, cu_k, (Hq // 2, d))


def decode_v2(q, k, v, lam, kv_len=None, threads=None) -> np.ndarray:
    """V2 decode. q: [B,Hq,d]; k,v: [B,L,Hkv,d]; kv_len: [B] or None -> out [B,Hq/2,d]."""
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    B, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    assert k.shape == (B, L, Hkv, d) and v.shape == k.shape and lam.shape == (Hq // 2,)
    kl = None if kv_len is None else np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32))
    out = np.zeros((B, Hq // 2, d), dtype=np.float64)
    rc = _load().oracle_decode_v2(_dp(q), _dp(k), _dp(v), _ip(kl), _dp(lam), B, L, Hq, Hkv, d,
                                  _dp(out), int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_decode_v2 failed: {rc}")
    return out


def decode_v1(q, k, v, lam, lambda_init_value: float, kv_len=None, apply_norm=True, eps=1e-5,
              threads=None) -> np.ndarray:
    """V1 decode. q: [B,H,2,d]; k: [B,L,H,2,d]; v: [B,L,H,2d]; kv_len: [B] or None
    -> out [B,H,2d] (per-head RMSNorm and (1 - lambda_init) scale when apply_norm)."""
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    B, H, two, d = q.shape
    L = k.shape[1]
    assert two == 2 and k.shape == (B, L, H, 2, d) and v.shape == (B, L, H, 2 * d)
    assert lam.shape == (H,)
    kl = None if kv_len is None else np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32))
    out = np.zeros((B, H, 2 * d), dtype=np.float64)
    rc = _load().oracle_decode_v1(_dp(q), _dp(k), _dp(v), _ip(kl), _dp(lam), float(lambda_init_value),
                                  B, L, H, d, int(bool(apply_norm)), float(eps), _dp(out),
                                  int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_decode_v1 failed: {rc}")
    return out


def gather_pages(pool, block_table) -> np.ndarray:
    """A paged cache read back as a contiguous one: entry b's token t is row t % page_size
    of page block_table[b, t // page_size]. pool [P, page_size, ...] -> [B, n*page_size, ...]."""
    pool = np.asarray(pool)
    bt = np.asarray(block_table, dtype=np.int64)
    B, n = bt.shape
    assert bt.min() >= 0 and bt.max() < pool.shape[0]
    return pool[bt].reshape((B, n * pool.shape[1]) + pool.shape[2:])


def decode_v2_paged(q, k_pool, v_pool, block_table, lam, kv_len, threads=None) -> np.ndarray:
    """V2 decode over a paged cache: the contiguous decode of the gathered cache."""
    return decode_v2(q, gather_pages(k_pool, block_table), gather_pages(v_pool, block_table), lam,
                     kv_len=kv_len, threads=threads)


def decode_v1_paged(q, k_pool, v_pool, block_table, lam, lambda_init_value: float, kv_len,
                    apply_norm=True, eps=1e-5, threads=None) -> np.ndarray:
    """V1 decode over a paged cache: the contiguous decode of the gathered cache."""
    return decode_v1(q, gather_pages(k_pool, block_table), gather_pages(v_pool, block_table), lam,
                     lambda_init_value, kv_len=kv_len, apply_norm=apply_norm, eps=eps,
                     threads=threads)


def map_row_v2(q, k, p: int, i: int):
    """The two softmax rows (A_1[i, :i+1], A_2[i, :i+1]) of pair p, one batch entry.
    q: [N,Hq,d]; k: [N,Hkv,d]."""
    q, k = _f64(q), _f64(k)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    a1 = np.zeros(i + 1, dtype=np.float64)
    a2 = np.zeros(i + 1, dtype=np.float64)
    rc = _load().oracle_map_row_v2(_dp(q), _dp(k), N, Hq, Hkv, d, int(p), int(i), _dp(a1), _dp(a2))
    if rc != 0:
        raise ValueError(f"oracle_map_row_v2 failed: {rc}")
    return a1, a2

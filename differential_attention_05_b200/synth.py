"""Seeded synthetic inputs for the differential attention operator.

This module only draws random numbers and arranges them into the operator's input
layouts; it holds none of the operator's arithmetic. Both the CUDA path (tests and
benchmark) and the float64 oracle read their inputs from here, so the two sides always
see the same bits.

Streams: numpy PCG64 seeded from SeedSequence([1000 + config_index, tensor_id, slice]).
Each tensor (and, for the decode cache, each batch entry) has its own stream, so a
slice can be regenerated without drawing the rest. Values are drawn in float32 and, for
bf16 configurations, rounded to bf16 with round-to-nearest-even; bf16 tensors are
returned as uint16 bit patterns.

Layouts (row-major, last dimension contiguous):
  V1: q, k [B, N, H, 2, d] (index 0 of the branch axis is branch 1); v [B, N, H, 2d]
  V2 prefill: q [B, N, Hq, d] (heads 2p, 2p+1 = branches 1, 2 of pair p);
              k, v [B, N, Hkv, d]
  V2 decode: q [B, Hq, d]; k, v [B, L, Hkv, d]
  lambda vectors: four float32 arrays [n_units, d_lambda]
"""
from __future__ import annotations

import concurrent.futures as _cf
import math
import os
from dataclasses import dataclass, field

import numpy as np

# tensor ids inside one configuration's seed space
_T_Q, _T_K, _T_V, _T_LQ1, _T_LK1, _T_LQ2, _T_LK2, _T_PLANT, _T_Q2 = range(9)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even.
    Inputs here are finite draws, so no NaN/Inf handling is needed."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tensor: int, slice_: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, slice_])))


def _normal(seed, tensor, shape, std=1.0, slice_=0) -> np.ndarray:
    x = _rng(seed, tensor, slice_).standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x.reshape(shape)


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return 4


def _normal_sliced(seed, tensor, shape, std=1.0, bf16=True) -> np.ndarray:
    """Draw along axis 0 in independent per-slice streams (slice = index on axis 0), in a
    thread pool; numpy's generators release the GIL while filling."""
    out = np.empty(shape, dtype=np.uint16 if bf16 else np.float32)

    def work(b):
        x = _normal(seed, tensor, shape[1:], std, slice_=b)
        out[b] = bf16_bits(x) if bf16 else x

    with _cf.ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(shape[0])))
    return out


@dataclass
class Inputs:
    """One configuration's inputs. bf16 tensors are uint16 bit arrays."""
    name: str
    variant: int                 # 1 = V1, 2 = V2
    mode: str                    # "prefill" or "decode"
    dtype: str                   # "f32" or "bf16"
    B: int
    N: int                       # sequence length (prefill) / cache capacity L (decode)
    H: int                       # V1: differential heads; V2: query heads Hq
    Hkv: int
    d: int                       # branch width
    depth: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    lq1: np.ndarray
    lk1: np.ndarray
    lq2: np.ndarray
    lk2: np.ndarray
    causal: bool = True
    apply_norm: bool = False
    eps: float = 1e-5
    kv_len: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def n_units(self) -> int:
        """number of lambda scalars: V1 heads or V2 pairs"""
        return self.H if self.variant == 1 else self.H // 2

    def as_f64(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        if a.dtype == np.uint16:
            return bf16_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def _lambda_vectors(seed, n_units, dim):
    # "lambda vectors N(0, 0.1)": read as standard deviation 0.1
    return tuple(_normal(seed, t, (n_units, dim), 0.1) for t in (_T_LQ1, _T_LK1, _T_LQ2, _T_LK2))


def lambda_vectors(seed: int, n_units: int, dim: int):
    """The four lambda vectors (lq1, lk1, lq2, lk2) float32 [n_units, dim] that the workload
    with this seed uses, drawn without its other tensors."""
    return _lambda_vectors(seed, n_units, dim)


# ---------------------------------------------------------------------------------------
# The five workloads of the operator (seed = 1000 + index)


def config1() -> Inputs:
    """V1 single head, fp32, causal: B=1, N=128, d=64; Q1,Q2,K1,K2 [128,64], V [128,128]
    iid N(0,1); lambda vectors N(0, 0.1) [1,64]; depth 1; RMSNorm eps 1e-5."""
    s, B, N, H, d = 1000, 1, 128, 1, 64
    q = _normal(s, _T_Q, (B, N, H, 2, d))
    k = _normal(s, _T_K, (B, N, H, 2, d))
    v = _normal(s, _T_V, (B, N, H, 2 * d))
    return Inputs("v1_f32_single_head", 1, "prefill", "f32", B, N, H, H, d, 1, q, k, v,
                  *_lambda_vectors(s, H, d), causal=True, apply_norm=True)


def config2() -> Inputs:
    """V1 layer, bf16, causal: B=2, 16 heads, N=4096, d=64, V width 128; Q/K/V iid N(0,1)
    times 1/sqrt(d), rounded to bf16; lambda vectors N(0, 0.1) [16,64]; depth 12."""
    s, B, N, H, d = 1001, 2, 4096, 16, 64
    sc = 1.0 / math.sqrt(d)
    q = _normal_sliced(s, _T_Q, (B, N, H, 2, d), sc)
    k = _normal_sliced(s, _T_K, (B, N, H, 2, d), sc)
    v = _normal_sliced(s, _T_V, (B, N, H, 2 * d), sc)
    return Inputs("v1_bf16_layer_b2_h16_n4096_d64", 1, "prefill", "bf16", B, N, H, H, d, 12,
                  q, k, v, *_lambda_vectors(s, H, d), causal=True, apply_norm=True)


def v2_prefill(B=1, N=16384, Hq=64, Hkv=8, d=128, depth=24, seed=1002, name=None) -> Inputs:
    """V2 prefill, bf16, causal GQA: q [B,N,Hq,d], k,v [B,N,Hkv,d] iid N(0,1)."""
    q = _normal_sliced(seed, _T_Q, (B * N, Hq, d)).reshape(B, N, Hq, d)
    k = _normal_sliced(seed, _T_K, (B * N, Hkv, d)).reshape(B, N, Hkv, d)
    v = _normal_sliced(seed, _T_V, (B * N, Hkv, d)).reshape(B, N, Hkv, d)
    return Inputs(name or f"v2_bf16_prefill_b{B}_n{N}_hq{Hq}_hkv{Hkv}_d{d}", 2, "prefill", "bf16",
                  B, N, Hq, Hkv, d, depth, q, k, v, *_lambda_vectors(seed, Hq // 2, d))


def grad_out(shape, seed: int) -> np.ndarray:
    """A seeded incoming gradient dL/dy of the given shape, N(0,1), as bf16 bits."""
    return _normal_sliced(seed, _T_V + 17, tuple(shape))


def v1_backward() -> Inputs:
    """Backward of the V1 layer: the config2 inputs plus dy [B,N,H,2d] N(0,1) in
    extra["dy"] (seed 1001)."""
    inp = config2()
    inp.name = "v1_bf16_backward_b2_h16_n4096_d64"
    inp.extra["dy"] = grad_out((inp.B, inp.N, inp.H, 2 * inp.d), 1001)
    return inp


def v2_backward(B=1, N=4096, Hq=64, Hkv=8, d=128, depth=24, seed=1007, name=None) -> Inputs:
    """Backward of a V2 prefill: the V2 prefill inputs (iid N(0,1)) plus dy [B,N,Hq/2,d]
    N(0,1) in extra["dy"]."""
    inp = v2_prefill(B=B, N=N, Hq=Hq, Hkv=Hkv, d=d, depth=depth, seed=seed,
                     name=name or f"v2_bf16_backward_b{B}_n{N}_hq{Hq}_hkv{Hkv}_d{d}")
    inp.extra["dy"] = grad_out((B, N, Hq // 2, d), seed)
    return inp


def config3() -> Inputs:
    """V2 prefill, bf16, causal, GQA: B=1, 64 query heads (32 pairs) over 8 KV heads,
    d=128, N=16384; iid N(0,1); per-pair lambda at depth 24; no norm."""
    return v2_prefill(seed=1002, name="v2_bf16_prefill_b1_n16384_hq64_hkv8_d128")


def v2_decode(B=64, L=32768, Hq=64, Hkv=8, d=128, depth=24, seed=1003, kv_len=None,
              name=None) -> Inputs:
    """V2 decode, bf16: q [B,Hq,d]; cache k,v [B,L,Hkv,d] iid N(0,1), one stream per batch
    entry so sampled entries can be redrawn alone (see decode_cache_slice)."""
    q = _normal_sliced(seed, _T_Q, (B, Hq, d))
    k = _normal_sliced(seed, _T_K, (B, L, Hkv, d))
    v = _normal_sliced(seed, _T_V, (B, L, Hkv, d))
    kl = None if kv_len is None else np.asarray(kv_len, dtype=np.int32)
    return Inputs(name or f"v2_bf16_decode_b{B}_l{L}_hq{Hq}_hkv{Hkv}_d{d}", 2, "decode", "bf16",
                  B, L, Hq, Hkv, d, depth, q, k, v, *_lambda_vectors(seed, Hq // 2, d),
                  causal=False, kv_len=kl)


def config4() -> Inputs:
    """V2 decode, bf16: batch 64, one new query each, cache length 32768, 64 query heads
    over 8 KV heads, d=128; cache and queries iid N(0,1)."""
    return v2_decode(name="v2_bf16_decode_b64_l32768_hq64_hkv8_d128")


def decode_cache_slice(b: int, L=32768, Hkv=8, d=128, seed=1003):
    """Batch entry b of the decode cache (k, v) as bf16 bits, identical to v2_decode's."""
    k = bf16_bits(_normal(seed, _T_K, (L, Hkv, d), slice_=b))
    v = bf16_bits(_normal(seed, _T_V, (L, Hkv, d), slice_=b))
    return k, v


def v1_decode(B=32, L=32768, H=16, d=64, depth=12, seed=1006, kv_len=None, name=None,
              scale=None) -> Inputs:
    """V1 decode, bf16: q [B,H,2,d]; cache k [B,L,H,2,d], v [B,L,H,2d]; the V1 layer's
    heads and widths (C2: 16 heads, d = 64, depth 12) over a decode cache holding the same
    bytes as the V2 decode workload (8.6 GB at B=32, L=32768). Values N(0,1) scaled by
    1/sqrt(d) like the V1 layer inputs; one stream per batch entry (see
    decode_cache_slice_v1)."""
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    q = _normal_sliced(seed, _T_Q, (B, H, 2, d), sc)
    k = _normal_sliced(seed, _T_K, (B, L, H, 2, d), sc)
    v = _normal_sliced(seed, _T_V, (B, L, H, 2 * d), sc)
    kl = None if kv_len is None else np.asarray(kv_len, dtype=np.int32)
    return Inputs(name or f"v1_bf16_decode_b{B}_l{L}_h{H}_d{d}", 1, "decode", "bf16",
                  B, L, H, H, d, depth, q, k, v, *_lambda_vectors(seed, H, d),
                  causal=False, apply_norm=True, kv_len=kl)


def decode_cache_slice_v1(b: int, L=32768, H=16, d=64, seed=1006, scale=None):
    """Batch entry b of the V1 decode cache (k, v) as bf16 bits, identical to v1_decode's."""
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    k = bf16_bits(_normal(seed, _T_K, (L, H, 2, d), sc, slice_=b))
    v = bf16_bits(_normal(seed, _T_V, (L, H, 2 * d), sc, slice_=b))
    return k, v


def paginate(caches, page_size: int, seed: int, spare_pages: int = 3, fill: str = "nan"):
    """Scatter contiguous caches [B, L, ...] (all with the same B and L) into one page pool
    per cache, in a seeded shuffled page order, as a serving system's paged cache holds
    them. Returns (pools [P, page_size, ...] per cache, block_table int32 [B, ceil(L /
    page_size)]). The rows past L in each entry's last page and the spare pages hold NaN
    (fill="nan") or N(0,1) noise (fill="noise"), so a reader that strays shows it. Inputs
    and pools are bf16 bit arrays (uint16) or float arrays."""
    B, L = caches[0].shape[:2]
    n = -(-L // page_size) if L else 1
    P = B * n + spare_pages
    perm = np.random.default_rng(np.random.PCG64(seed)).permutation(P)
    table = perm[:B * n].reshape(B, n).astype(np.int32)
    pools = []
    for ci, c in enumerate(caches):
        assert c.shape[:2] == (B, L)
        shape = (P, page_size) + c.shape[2:]
        if fill == "nan":
            pool = (np.full(shape, 0x7FC0, dtype=np.uint16) if c.dtype == np.uint16
                    else np.full(shape, np.nan, dtype=c.dtype))
        else:
            noise = _normal(seed, 100 + ci, shape)
            pool = bf16_bits(noise) if c.dtype == np.uint16 else noise.astype(c.dtype)
        for b in range(B):
            for i in range(n):
                rows = c[b, i * page_size:(i + 1) * page_size]
                pool[table[b, i], :rows.shape[0]] = rows
        pools.append(pool)
    return pools, table


def signal_plus_noise(N=65536, Hq=64, Hkv=8, d=128, depth=24, seed=1004, name=None) -> Inputs:
    """Long-context signal-plus-noise workload (bf16, causal, B=1).

    For each KV head g and each of its pairs i (pair p = g*(Hq/Hkv/2) + i):
      * a seeded unit signal direction u[g,i] and a seeded planted position s[g,i];
      * the planted key k[s, g] = 3 * sqrt(d) * u[g,i] (the signal query direction scaled
        to norm 3*sqrt(d)); every other key is N(0,1) noise;
      * per position t, a noise query n ~ N(0, I): branch 2 (head 2p+1) sees n, branch 1
        (head 2p) sees n + u[g,i]  (two microphones sharing one noise source);
      * v is N(0,1) with channels 0..pairs_per_group-1 zeroed, and the planted row of pair i
        is the one-hot vector e_i, so out[t, p, i] is exactly the differential weight on
        the planted key.
    """
    B = 1
    ppg = Hq // Hkv // 2  # pairs per KV group
    r = _rng(seed, _T_PLANT)
    u = r.standard_normal((Hkv, ppg, d)).astype(np.float64)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    pos = np.empty((Hkv, ppg), dtype=np.int64)
    for g in range(Hkv):
        pos[g] = r.choice(np.arange(N // 8, N // 2), size=ppg, replace=False)
    kf = _normal(seed, _T_K, (N, Hkv, d))
    vf = _normal(seed, _T_V, (N, Hkv, d))
    vf[:, :, :ppg] = 0.0
    for g in range(Hkv):
        for i in range(ppg):
            kf[pos[g, i], g] = (3.0 * math.sqrt(d) * u[g, i]).astype(np.float32)
            vf[pos[g, i], g] = 0.0
            vf[pos[g, i], g, i] = 1.0
    noise = _normal_sliced(seed, _T_Q, (N, Hq // 2, d), bf16=False)
    q = np.empty((N, Hq, d), dtype=np.uint16)
    for p in range(Hq // 2):
        g, i = divmod(p, ppg)
        q[:, 2 * p + 1] = bf16_bits(noise[:, p])
        q[:, 2 * p] = bf16_bits(noise[:, p] + u[g, i].astype(np.float32))
    del noise
    inp = Inputs(name or f"v2_bf16_signal_plus_noise_n{N}_hq{Hq}_hkv{Hkv}_d{d}", 2, "prefill",
                 "bf16", B, N, Hq, Hkv, d, depth, q.reshape(B, N, Hq, d),
                 bf16_bits(kf).reshape(B, N, Hkv, d), bf16_bits(vf).reshape(B, N, Hkv, d),
                 *_lambda_vectors(seed, Hq // 2, d))
    inp.extra = {"planted_pos": pos, "signal_dir": u, "pairs_per_group": ppg}
    return inp


def config5() -> Inputs:
    """V2 long-context signal-plus-noise, bf16, causal: N=65536, 64 query heads over 8 KV
    heads, d=128; 4 planted keys per KV head; lambda at depth 24."""
    return signal_plus_noise(name="v2_bf16_signal_plus_noise_n65536_hq64_hkv8_d128")


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}


def v1_small(B=1, N=300, H=2, d=64, depth=3, seed=77, dtype="bf16", causal=True,
             apply_norm=True, scale=None) -> Inputs:
    """Small V1 case (ragged N, several tiles) for parity tests."""
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    conv = bf16_bits if dtype == "bf16" else (lambda x: x)
    q = conv(_normal(seed, _T_Q, (B, N, H, 2, d), sc))
    k = conv(_normal(seed, _T_K, (B, N, H, 2, d), sc))
    v = conv(_normal(seed, _T_V, (B, N, H, 2 * d), sc))
    return Inputs(f"v1_{dtype}_b{B}_n{N}_h{H}_d{d}", 1, "prefill", dtype, B, N, H, H, d, depth,
                  q, k, v, *_lambda_vectors(seed, H, d), causal=causal, apply_norm=apply_norm)


def v2_small(B=1, N=300, Hq=16, Hkv=2, d=128, depth=5, seed=78, dtype="bf16", causal=True) -> Inputs:
    """Small V2 prefill case (ragged N) for parity tests."""
    conv = bf16_bits if dtype == "bf16" else (lambda x: x)
    q = conv(_normal(seed, _T_Q, (B, N, Hq, d)))
    k = conv(_normal(seed, _T_K, (B, N, Hkv, d)))
    v = conv(_normal(seed, _T_V, (B, N, Hkv, d)))
    return Inputs(f"v2_{dtype}_b{B}_n{N}_hq{Hq}_hkv{Hkv}_d{d}", 2, "prefill", dtype, B, N, Hq, Hkv,
                  d, depth, q, k, v, *_lambda_vectors(seed, Hq // 2, d), causal=causal)

"""GPU parity: the V1 split-KV decode (diffattn_fwd_decode_v1) against the float64 oracle."""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, dev_tensor, lambda_on_device, out_f64

pytestmark = pytest.mark.gpu


def _lam(inp):
    return oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)


def _decode_v1(inp, kv_len=None, num_splits=0, apply_norm=True, q=None, lam=None):
    qd = dev_tensor(inp.q if q is None else q)
    k, v = dev_tensor(inp.k), dev_tensor(inp.v)
    lam_d, li = lambda_on_device(inp)
    if lam is not None:
        lam_d = torch.tensor(lam, dtype=torch.float32, device="cuda")
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out = da.diffattn_fwd_decode_v1(qd, k, v, lam_d, li, kv_len=kl, apply_norm=apply_norm,
                                    norm_eps=inp.eps, num_splits=num_splits)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("L,kv_len,splits,norm", [(1000, [1000, 1, 513], 0, True),
                                                  (4096, None, 3, True),
                                                  (200, [200, 64, 65], 7, False),
                                                  (65, [1, 64, 65], 2, True)])
def test_decode_v1_small(L, kv_len, splits, norm):
    inp = synth.v1_decode(B=3, L=L, H=4, seed=95)
    out = out_f64(_decode_v1(inp, kv_len, splits, norm))
    ref = oracle.decode_v1(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _lam(inp),
                           oracle.lambda_init(inp.depth), kv_len=kv_len, apply_norm=norm,
                           eps=inp.eps)
    assert_parity(out, ref, "bf16", f"V1 decode L={L} splits={splits} norm={norm}")


def test_decode_v1_kv_len_zero_is_zero():
    inp = synth.v1_decode(B=2, L=128, H=2, seed=96)
    out = _decode_v1(inp, [0, 0])
    assert torch.all(out.float() == 0).item()


def test_decode_v1_identical_branches_cancel_exactly():
    """Branch 2 a copy of branch 1 (query and cached keys) and lambda = 1: both branches run
    the same arithmetic, so the difference is exactly zero before the norm."""
    inp = synth.v1_decode(B=2, L=700, H=4, seed=97)
    q = inp.q.copy()
    q[:, :, 1] = q[:, :, 0]
    k = inp.k.copy()
    k[:, :, :, 1] = k[:, :, :, 0]
    inp.k = k
    out = _decode_v1(inp, q=q, lam=np.ones(4), apply_norm=False)
    assert torch.all(out.float() == 0).item()


def test_decode_v1_lambda0_is_branch1_attention():
    """lambda = 0, no norm: branch 1's softmax attention over the cache (torch SDPA on the
    same bf16 values in fp32)."""
    inp = synth.v1_decode(B=2, L=333, H=3, seed=98)
    out = _decode_v1(inp, lam=np.zeros(3), apply_norm=False).float()
    q = dev_tensor(inp.q).float()[:, :, 0]                      # [B, H, d]
    k = dev_tensor(inp.k).float()[:, :, :, 0].transpose(1, 2)   # [B, H, L, d]
    v = dev_tensor(inp.v).float().transpose(1, 2)               # [B, H, L, 2d]
    ref = torch.nn.functional.scaled_dot_product_attention(q[:, :, None], k, v)[:, :, 0]
    err = (out - ref).abs().max().item()
    assert err <= 2e-2, err


@pytest.mark.slow
def test_decode_v1_full_size_sampled():
    """The V1 decode workload the benchmark times (batch 32, cache 32768, 16 heads, d = 64),
    in the same launch configuration; the oracle checks every head of 4 sampled entries."""
    inp = synth.v1_decode()
    out = out_f64(_decode_v1(inp))
    lam, li = _lam(inp), oracle.lambda_init(inp.depth)
    for b in (0, 9, 21, 31):
        k, v = (synth.bf16_to_f32(x[b:b + 1]) for x in (inp.k, inp.v))
        ref = oracle.decode_v1(synth.bf16_to_f32(inp.q[b:b + 1]), k, v, lam, li, eps=inp.eps)
        assert_parity(out[b:b + 1], ref, "bf16", f"V1 decode batch {b}")

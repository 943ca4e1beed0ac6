"""GPU parity: lambda kernel, exact-fp32 prefill and the split-KV decode against the oracle."""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, dev_tensor, lambda_on_device, out_f64, run_prefill

pytestmark = pytest.mark.gpu


def _oracle_lambda(inp):
    return oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)


@pytest.mark.parametrize("make", [synth.config1, lambda: synth.v1_small(H=16, depth=12),
                                  lambda: synth.v2_small(Hq=64, Hkv=8, depth=24)])
def test_lambda_kernel(make):
    inp = make()
    lam, li = lambda_on_device(inp)
    torch.cuda.synchronize()
    ref = _oracle_lambda(inp)
    np.testing.assert_allclose(lam.cpu().numpy(), ref, rtol=0, atol=2e-6)
    assert abs(float(li.item()) - oracle.lambda_init(inp.depth)) < 1e-6


def test_lambda_init_depth1_is_02():
    inp = synth.config1()
    _, li = lambda_on_device(inp)
    assert abs(float(li.item()) - 0.2) < 1e-7


def test_config1_fp32_v1_single_head():
    """V1, fp32, causal, B=1, N=128, d=64, depth 1: max abs error <= 1e-5."""
    inp = synth.config1()
    out = out_f64(run_prefill(inp))
    ref = oracle.prefill_v1(inp.q, inp.k, inp.v, _oracle_lambda(inp), oracle.lambda_init(inp.depth),
                            causal=True, apply_norm=True, eps=inp.eps)
    assert_parity(out, ref, "f32", "config 1")


@pytest.mark.parametrize("N,causal,norm", [(1, True, True), (300, True, True), (77, False, True),
                                           (200, True, False)])
def test_fp32_v1_ragged(N, causal, norm):
    inp = synth.v1_small(B=2, N=N, H=3, d=64, dtype="f32", causal=causal, apply_norm=norm, scale=1.0)
    out = out_f64(run_prefill(inp))
    ref = oracle.prefill_v1(inp.q, inp.k, inp.v, _oracle_lambda(inp), oracle.lambda_init(inp.depth),
                            causal=causal, apply_norm=norm, eps=inp.eps)
    assert_parity(out, ref, "f32", f"fp32 V1 N={N}")


@pytest.mark.parametrize("N,causal,d", [(130, True, 128), (65, False, 64), (3, True, 32)])
def test_fp32_v2(N, causal, d):
    inp = synth.v2_small(B=2, N=N, Hq=8, Hkv=2, d=d, dtype="f32", causal=causal)
    out = out_f64(run_prefill(inp))
    ref = oracle.prefill_v2(inp.q, inp.k, inp.v, _oracle_lambda(inp), causal=causal)
    assert_parity(out, ref, "f32", f"fp32 V2 N={N}")


def _decode(inp, kv_len=None, num_splits=0):
    q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
    lam, _ = lambda_on_device(inp)
    kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out = da.diffattn_fwd_decode(q, k, v, lam, kv_len=kl, num_splits=num_splits)
    torch.cuda.synchronize()
    return out_f64(out)


@pytest.mark.parametrize("L,kv_len,splits", [(1000, [1000, 1, 0, 513], 0), (4096, None, 3),
                                             (200, [200, 64, 65, 127], 7)])
def test_decode_small(L, kv_len, splits):
    inp = synth.v2_decode(B=4, L=L, Hq=16, Hkv=2, seed=91)
    out = _decode(inp, kv_len, splits)
    ref = oracle.decode_v2(inp.as_f64('q'), inp.as_f64('k'), inp.as_f64('v'), _oracle_lambda(inp),
                           kv_len=kv_len)
    assert_parity(out, ref, "bf16", f"decode L={L}")


def test_decode_kv_len_zero_is_zero():
    inp = synth.v2_decode(B=2, L=128, Hq=8, Hkv=1, seed=92)
    out = _decode(inp, [0, 0])
    assert np.all(out == 0.0)


def test_decode_identical_branches_cancel_exactly():
    """Both heads of every pair equal and lambda = 1: the two branches run the same
    arithmetic, so the GPU result is exactly zero."""
    inp = synth.v2_decode(B=2, L=700, Hq=16, Hkv=2, seed=93)
    q = inp.q.copy()
    q[:, 1::2] = q[:, 0::2]
    qd, k, v = dev_tensor(q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam = torch.ones(8, dtype=torch.float32, device="cuda")
    out = da.diffattn_fwd_decode(qd, k, v, lam)
    torch.cuda.synchronize()
    assert torch.all(out.float() == 0).item()


@pytest.mark.slow
def test_config4_decode_full_size_sampled():
    """Config 4 (batch 64, cache 32768, 64/8 heads) in the launch configuration the
    benchmark times; the oracle checks every pair of 4 sampled batch entries."""
    inp = synth.config4()
    out = _decode(inp)
    lam = _oracle_lambda(inp)
    for b in (0, 17, 42, 63):
        k, v = (synth.bf16_to_f32(x[b:b + 1]) for x in (inp.k, inp.v))
        ref = oracle.decode_v2(synth.bf16_to_f32(inp.q[b:b + 1]), k, v, lam)
        assert_parity(out[b:b + 1], ref, "bf16", f"config 4 batch {b}")

"""GPU parity of the variable-length prefill (diffattn_fwd_prefill_varlen): sequences of
different lengths packed back to back, plain prompts (nq = nk) and chunks after cached
tokens (nq < nk), against the float64 oracle; each sequence bit-identical to the
fixed-length call on it alone; inconsistent offsets reported through dev_status."""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, dev_tensor, lambda_on_device, out_f64

pytestmark = pytest.mark.gpu


def _packed(variant, nq, nk, dtype="bf16", seed=0):
    """Packed q [Tq, ...], k and v [Tk, ...] drawn like the fixed-length inputs."""
    Tq, Tk = int(sum(nq)), int(sum(nk))
    if variant == 1:
        inp = synth.v1_small(B=1, N=max(Tq, Tk, 1), H=2, seed=500 + seed, dtype=dtype)
    else:
        inp = synth.v2_small(B=1, N=max(Tq, Tk, 1), Hq=8, Hkv=2, seed=600 + seed, dtype=dtype)
    inp.q, inp.k, inp.v = inp.q[0, :Tq], inp.k[0, :Tk], inp.v[0, :Tk]
    cu_q = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(nk)]).astype(np.int32)
    return inp, cu_q, cu_k


def _run(inp, cu_q, cu_k, window=0, causal=True, dev_status=None):
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam, li = lambda_on_device(inp)
    out = da.diffattn_fwd_prefill_varlen(
        q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
        int(np.max(np.diff(cu_q))) if len(cu_q) > 1 else 0, lam, li, causal=causal,
        apply_norm=inp.apply_norm, norm_eps=inp.eps, window=window, dev_status=dev_status)
    torch.cuda.synchronize()
    return out


def _ref(inp, cu_q, cu_k, window=0, causal=True):
    lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    q, k, v = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v")
    if inp.variant == 1:
        return oracle.prefill_v1_varlen(q, k, v, cu_q, cu_k, lam, oracle.lambda_init(inp.depth),
                                        causal=causal, apply_norm=inp.apply_norm, eps=inp.eps,
                                        window=window)
    return oracle.prefill_v2_varlen(q, k, v, cu_q, cu_k, lam, causal=causal, window=window)


# (query counts, key counts): an empty sequence, one-token sequences, tile edges, chunks
CASES = [([300, 1, 129, 0, 513], [300, 1, 129, 0, 513]),
         ([64, 200, 1, 77], [500, 200, 90, 77]),
         ([128], [1000])]


@pytest.mark.parametrize("nq,nk", CASES)
@pytest.mark.parametrize("variant", [1, 2])
def test_varlen_bf16(variant, nq, nk):
    inp, cu_q, cu_k = _packed(variant, nq, nk, seed=len(nq))
    assert_parity(out_f64(_run(inp, cu_q, cu_k)), _ref(inp, cu_q, cu_k), "bf16",
                  f"V{variant} varlen {nq}/{nk}")


@pytest.mark.parametrize("variant", [1, 2])
def test_varlen_window_and_non_causal(variant):
    inp, cu_q, cu_k = _packed(variant, [300, 45, 260], [300, 400, 260], seed=9)
    assert_parity(out_f64(_run(inp, cu_q, cu_k, window=100)), _ref(inp, cu_q, cu_k, window=100),
                  "bf16", f"V{variant} varlen window")
    assert_parity(out_f64(_run(inp, cu_q, cu_k, causal=False)), _ref(inp, cu_q, cu_k, causal=False),
                  "bf16", f"V{variant} varlen non-causal")


@pytest.mark.parametrize("variant", [1, 2])
def test_varlen_f32(variant):
    inp, cu_q, cu_k = _packed(variant, [70, 1, 33], [70, 90, 33], dtype="f32", seed=3)
    assert_parity(out_f64(_run(inp, cu_q, cu_k)), _ref(inp, cu_q, cu_k), "f32", f"V{variant} varlen f32")


@pytest.mark.parametrize("variant", [1, 2])
def test_each_sequence_equals_its_own_call(variant):
    """Every row's arithmetic depends only on its own sequence: the packed call equals,
    bit for bit, the fixed-length call on each sequence alone."""
    nq, nk = [257, 1, 640, 100], [257, 130, 640, 700]
    inp, cu_q, cu_k = _packed(variant, nq, nk, seed=21)
    packed = _run(inp, cu_q, cu_k)
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam, li = lambda_on_device(inp)
    for s in range(len(nq)):
        one = da.diffattn_fwd_prefill(q[None, cu_q[s]:cu_q[s + 1]].contiguous(),
                                      k[None, cu_k[s]:cu_k[s + 1]].contiguous(),
                                      v[None, cu_k[s]:cu_k[s + 1]].contiguous(), lam, li,
                                      apply_norm=inp.apply_norm, norm_eps=inp.eps)
        torch.cuda.synchronize()
        assert torch.equal(one[0], packed[cu_q[s]:cu_q[s + 1]]), s


def test_inconsistent_offsets_are_reported():
    """A sequence with more queries than keys is skipped (its rows keep their prior
    contents) and DIFFATTN_ERR_INVALID_ARG lands in dev_status; the others are computed."""
    inp, cu_q, cu_k = _packed(2, [100, 50, 80], [100, 60, 80], seed=30)
    cu_k_bad = cu_k.copy()
    cu_k_bad[2] = cu_k_bad[1] + 40              # sequence 1: 50 queries over 40 keys
    cu_k_bad[3] = cu_k[3]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam, _ = lambda_on_device(inp)
    out = torch.full((q.shape[0], 4, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    da.diffattn_fwd_prefill_varlen(q, k, v, torch.from_numpy(cu_q).cuda(),
                                   torch.from_numpy(cu_k_bad).cuda(), 100, lam, out=out,
                                   dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == -1
    assert torch.all(out[100:150].float() == 7.0).item()
    ref = _ref(inp, cu_q, cu_k)
    assert_parity(out_f64(out[:100]), ref[:100], "bf16", "sequence 0")
    # sequence 2 reads keys 140.. of the packed tensor under the bad offsets
    ref2 = _ref(inp, np.array([0, 80], np.int32) + 150, np.array([cu_k_bad[2], cu_k_bad[3]], np.int32))
    assert_parity(out_f64(out[150:230]), ref2[150:230], "bf16", "sequence 2")


def test_varlen_rejects():
    inp, cu_q, cu_k = _packed(2, [10, 20], [10, 20], seed=31)
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam, _ = lambda_on_device(inp)
    with pytest.raises(da.DiffattnError):
        da.diffattn_fwd_prefill_varlen(q, k, v, torch.from_numpy(cu_q).cuda(),
                                       torch.from_numpy(cu_k[:2]).cuda(), 20, lam)
    with pytest.raises(da.DiffattnError):
        da.diffattn_fwd_prefill_varlen(q, k, v, torch.from_numpy(cu_q).cuda(),
                                       torch.from_numpy(cu_k).cuda(), -1, lam)

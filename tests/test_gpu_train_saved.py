"""The training forward (diffattn_fwd_prefill_train) and the backward from its saved output
(diffattn_bwd_prefill_saved), V2 bf16 with d = 128.

  * out is the inference forward's, bit for bit (same kernel arithmetic);
  * o2 = A_2 V of every (query, pair) matches the float64 oracle run with branch 1's
    queries replaced by branch 2's and lambda = 0 (the output is then A_2 V), within the
    bf16 bounds;
  * lse_b = log2 sum_j exp(s_b,j) matches the same quantity in float64 from the inputs
    (raw scores s = q . k / sqrt(d)) to 2e-3 absolute (fp32 sums of ex2.approx terms);
  * the gradients match the float64 backward oracle within the tensor-core tolerance of
    tests/test_gpu_backward.py (rel RMS <= 5e-3, max abs <= 2% of each tensor's scale) and
    come out deterministic.
"""
import math

import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from oracle import backward as OB
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, dev_tensor, lambda_on_device, out_f64

pytestmark = pytest.mark.gpu


def _check_tc(got, ref, what):
    got = got.detach().float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)), what
    scale = float(np.max(np.abs(ref)))
    err = float(np.max(np.abs(got - ref)))
    rms = float(np.sqrt(np.mean((got - ref) ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))
    assert rms <= 5e-3, f"{what}: rel RMS {rms:.3e}"
    assert err <= 2e-2 * scale + 1e-6, f"{what}: max abs {err:.3e} vs scale {scale:.3e}"


def _lse_ref(q, k, Nq, Nk, group, causal, window):
    """log2 sum_j exp(q_h . k_g(h),j / sqrt(d)) over the visible keys, float64 [B, Hq, Nq]."""
    B, _, Hq, d = q.shape
    out = np.empty((B, Hq, Nq))
    pos = np.arange(Nq) + (Nk - Nq)
    j = np.arange(Nk)
    vis = np.ones((Nq, Nk), dtype=bool)
    if causal:
        vis &= j[None, :] <= pos[:, None]
        if window > 0:
            vis &= j[None, :] > pos[:, None] - window
    for b in range(B):
        for h in range(Hq):
            s = q[b, :, h] @ k[b, :, h // group].T / math.sqrt(d)
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            out[b, h] = (np.log(np.exp(s - m).sum(axis=1)) + m[:, 0]) / math.log(2.0)
    return out


@pytest.mark.parametrize("Nq,Nk,causal,window,seed", [(300, 300, True, 0, 900), (97, 97, False, 0, 901),
                                                      (60, 201, True, 0, 902), (130, 130, True, 33, 903)])
def test_train_forward_and_saved_backward(Nq, Nk, causal, window, seed):
    Hq, Hkv = 16, 2
    inp = synth.v2_small(B=2, N=Nk, Hq=Hq, Hkv=Hkv, seed=seed, causal=causal)
    q = dev_tensor(inp.q)[:, Nk - Nq:].contiguous()
    k, v = dev_tensor(inp.k), dev_tensor(inp.v)
    lam, _ = lambda_on_device(inp)
    out, o2, lse = da.diffattn_fwd_prefill_train(q, k, v, lam, causal=causal, window=window)
    ref_out = da.diffattn_fwd_prefill(q, k, v, lam, causal=causal, window=window)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)

    q64 = inp.as_f64("q")[:, Nk - Nq:]
    k64, v64 = inp.as_f64("k"), inp.as_f64("v")
    q2only = q64.copy()
    q2only[:, :, 0::2] = q64[:, :, 1::2]  # branch 1 sees branch 2's queries
    o2_ref = oracle.prefill_v2(q2only, k64, v64, np.zeros(Hq // 2), causal=causal, window=window)
    assert_parity(out_f64(o2), o2_ref, "bf16", f"o2 Nq={Nq} Nk={Nk}")
    lse_ref = _lse_ref(q64, k64, Nq, Nk, Hq // Hkv, causal, window)  # [B, Hq, Nq]
    got = lse.cpu().numpy().astype(np.float64)                      # [B, Hq/2, Nq, 2]
    np.testing.assert_allclose(got[..., 0], lse_ref[:, 0::2], atol=2e-3)
    np.testing.assert_allclose(got[..., 1], lse_ref[:, 1::2], atol=2e-3)

    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(out.shape, generator=g).bfloat16().cuda()
    grads = da.diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dy, causal=causal, window=window)
    again = da.diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dy, causal=causal, window=window)
    torch.cuda.synchronize()
    for x, y in zip(grads, again):
        assert torch.equal(x, y)
    lam64 = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    ref = OB.prefill_v2_bwd(q64, k64, v64, lam64, dy.float().cpu().numpy().astype(np.float64),
                            causal=causal, window=window)
    for name, t, r in zip(("dq", "dk", "dv", "dlambda"), grads, ref):
        _check_tc(t, r, f"saved {name} Nq={Nq} Nk={Nk} causal={causal} window={window}")


def test_train_rejects_other_variants():
    inp = synth.v1_small(B=1, N=64, H=2, seed=910)
    q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
    lam, li = lambda_on_device(inp)
    out = torch.empty((1, 64, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Exception):
        da.diffattn_fwd_prefill_train(q, k, v, lam, out=out)


def test_backward_graph_capture_and_side_stream():
    """The tensor-core backward runs its dQ kernel on a library-owned second stream, forked
    from and joined back to the caller's stream. Captured into a CUDA graph on a non-default
    stream and replayed, it gives the eager call's gradients bit for bit, and work queued on
    the caller's stream after it sees the finished gradients."""
    Nq = Nk = 520
    inp = synth.v2_small(B=1, N=Nk, Hq=16, Hkv=2, seed=920, causal=True)
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    lam, _ = lambda_on_device(inp)
    out, o2, lse = da.diffattn_fwd_prefill_train(q, k, v, lam)
    g = torch.Generator().manual_seed(921)
    dy = torch.randn(out.shape, generator=g).bfloat16().cuda()
    eager = da.diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dy)
    p = da._binding.prefill_params(q, k, v, out, causal=True)
    ws = torch.empty(max(da._binding.diffattn_bwd_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
    grads = tuple(torch.full(t.shape, float("nan"), dtype=torch.float32, device="cuda") for t in eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        da.diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dy, workspace=ws, grads=grads)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        da.diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dy, workspace=ws, grads=grads)
    for t in grads:
        t.fill_(float("nan"))
    graph.replay()
    # read on the replay stream's successor: the copy is ordered after the joined graph
    copies = [t.clone() for t in grads]
    torch.cuda.synchronize()
    for name, x, y in zip(("dq", "dk", "dv", "dlambda"), copies, eager):
        assert torch.equal(x, y), name
    del graph

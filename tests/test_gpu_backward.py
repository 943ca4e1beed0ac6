"""GPU parity of the backward pass (diffattn_bwd_prefill, diffattn_lambda_bwd) against the
float64 backward oracle (itself pinned to finite differences of the forward oracle and to
torch autograd).

Tolerances, per tensor:
  * exact-fp32 kernels (fp32 inputs, other head widths): the kernels compute in fp32 from
    the same input values the oracle reads (bf16 inputs are widened exactly), so the only
    error is fp32 rounding of sums over at most a few thousand terms and of expf/logf:
    max abs error <= 2e-5 x max|reference| + 1e-6;
  * tensor-core kernels (bf16 V2 with d = 128, bf16 V1 with d = 64): the MMA operands
    P_1 - lambda P_2 and dS_b (and V1's dO) are rounded to bf16 (relative 2^-9 each,
    independent across terms), as in the forward: relative RMS error <= 5e-3 and max abs
    error <= 2e-2 x max|reference|. V1's statistics pass forms O and the norm's backward
    from probabilities split into two bf16 parts (error ~2^-18), so dlambda, which keeps
    only the small part of O_2 orthogonal to O, meets the same bound."""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from oracle import backward as OB
from differential_attention_05_b200 import synth

from gpu_helpers import dev_tensor, lambda_on_device

pytestmark = pytest.mark.gpu

REL = 2e-5
ABS = 1e-6


def _check(got, ref, what, tensor_core=False, zero_bound=1e-5):
    got = got.detach().float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if tensor_core:
        if scale == 0.0:
            # every query sees a single key, so the score gradient cancels exactly
            # (dQ = dK = 0); what is left is the residue of dP - delta (see _zero_bound)
            assert err <= zero_bound, f"{what}: {err:.3e} against an all-zero reference"
            return
        rms = float(np.sqrt(np.mean((got - ref) ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))
        assert rms <= 5e-3, f"{what}: rel RMS {rms:.3e} > 5e-3"
        assert err <= 2e-2 * scale + 1e-6, f"{what}: max abs err {err:.3e} > {2e-2 * scale:.3e}"
        return
    bound = REL * scale + ABS
    assert err <= bound, f"{what}: max abs err {err:.3e} > {bound:.3e}"


def _zero_bound(variant, q64, k64, v64, dO64, group):
    """Residue of a one-key query's dS = P (dP - delta) on the tensor-core path. V1's
    statistics pass forms O from split operands (error ~2^-18), leaving fp32 rounding. V2's
    keeps the forward's bf16 operand p_1 - c p_2 = 1 - lambda, so O_1 and delta_1 are off by
    up to 2^-9 relative and |dS| <= 2^-8 |dO . V|; dQ and dK multiply that by a q or k row
    / sqrt(d), and a KV head's dK adds the group's query heads."""
    if variant == 1:
        return 1e-5
    d = q64.shape[-1]
    dp = float(np.max(np.abs(np.einsum("bihc,bjgc->bhgij", dO64, v64)))) if dO64.size else 0.0
    return 2.0 ** -8 * dp * max(np.max(np.abs(q64)), np.max(np.abs(k64))) / np.sqrt(d) * group + 1e-6


def _case(variant, Nq, Nk, dtype, seed, causal=True, window=0, norm=True, Hq=8, Hkv=2, H=2, d=None):
    if variant == 1:
        inp = synth.v1_small(B=2, N=Nk, H=H, d=d or 64, seed=seed, dtype=dtype, causal=causal,
                             apply_norm=norm)
    else:
        inp = synth.v2_small(B=2, N=Nk, Hq=Hq, Hkv=Hkv, seed=seed, dtype=dtype, causal=causal)
    q = dev_tensor(inp.q)[:, Nk - Nq:].contiguous()
    k, v = dev_tensor(inp.k), dev_tensor(inp.v)
    lam, li = lambda_on_device(inp)
    oshape = (2, Nq, H, 2 * inp.d) if variant == 1 else (2, Nq, Hq // 2, inp.d)
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(oshape, generator=g).to(q.dtype).cuda()
    dq, dk, dv, dl = da.diffattn_bwd_prefill(q, k, v, lam, dy, li, causal=causal,
                                             apply_norm=inp.apply_norm, norm_eps=inp.eps,
                                             window=window)
    torch.cuda.synchronize()
    lam64 = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    q64 = inp.as_f64("q")[:, Nk - Nq:]
    k64, v64 = inp.as_f64("k"), inp.as_f64("v")
    dy64 = dy.float().cpu().numpy().astype(np.float64)
    if variant == 1:
        ref = OB.prefill_v1_bwd(q64, k64, v64, lam64, oracle.lambda_init(inp.depth), dy64,
                                causal=causal, apply_norm=inp.apply_norm, eps=inp.eps, window=window)
    else:
        ref = OB.prefill_v2_bwd(q64, k64, v64, lam64, dy64, causal=causal, window=window)
    tag = f"V{variant} {dtype} Nq={Nq} Nk={Nk} causal={causal} window={window}"
    tc = dtype == "bf16" and inp.d == (64 if variant == 1 else 128)
    zb = _zero_bound(variant, q64, k64, v64, dy64, Hq // Hkv) if tc else 1e-5
    for name, t, r in zip(("dq", "dk", "dv", "dlambda"), (dq, dk, dv, dl), ref):
        _check(t, r, f"{tag} {name}", tensor_core=tc, zero_bound=zb)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", [1, 2])
def test_backward_causal(variant, dtype):
    _case(variant, 150, 150, dtype, seed=700 + variant)


@pytest.mark.parametrize("variant", [1, 2])
def test_backward_full_chunk_window(variant):
    _case(variant, 97, 97, "bf16", seed=710 + variant, causal=False)
    _case(variant, 60, 201, "bf16", seed=720 + variant)
    _case(variant, 130, 130, "bf16", seed=730 + variant, window=33)
    _case(variant, 41, 170, "f32", seed=740 + variant, window=50)


def test_backward_v1_without_norm():
    _case(1, 120, 120, "bf16", seed=750, norm=False)


@pytest.mark.parametrize("variant", [1, 2])
def test_backward_tiny_and_ragged(variant):
    """Edge sizes of the tensor-core paths: one query over one key, a few queries over a
    ragged key count (chunk), and a window of one key (every query sees only itself)."""
    _case(variant, 1, 1, "bf16", seed=800 + variant)
    _case(variant, 3, 70, "bf16", seed=810 + variant)
    _case(variant, 65, 65, "bf16", seed=820 + variant, window=1)


def test_backward_v1_other_width_exact():
    """bf16 V1 with d != 64 runs the exact-fp32 kernels (and meets their bound)."""
    _case(1, 90, 90, "bf16", seed=752, d=32)


def test_backward_v1_layer_full_size():
    """The V1 layer at full size (B=2, 16 heads, N=4096, d=64, the seeded synth.config2
    tensors, the norm on), as the bench runs its backward. The float64 oracle covers one
    seeded head over both batch entries: its dQ, dK, dV and dlambda."""
    inp = synth.config2()
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    dy_bits = synth.grad_out((inp.B, inp.N, inp.H, 2 * inp.d), 1001)
    dy = dev_tensor(dy_bits)
    lam, li = lambda_on_device(inp)
    dq, dk, dv, dl = da.diffattn_bwd_prefill(q, k, v, lam, dy, li, apply_norm=True, norm_eps=inp.eps)
    torch.cuda.synchronize()
    h = int(np.random.default_rng(1001).integers(inp.H))
    lam64 = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)[h:h + 1]
    dy64 = synth.bf16_to_f32(dy_bits).astype(np.float64)[:, :, h:h + 1]
    ref = OB.prefill_v1_bwd(inp.as_f64("q")[:, :, h:h + 1], inp.as_f64("k")[:, :, h:h + 1],
                            inp.as_f64("v")[:, :, h:h + 1], lam64, oracle.lambda_init(inp.depth), dy64,
                            apply_norm=True, eps=inp.eps)
    got = (dq[:, :, h:h + 1], dk[:, :, h:h + 1], dv[:, :, h:h + 1], dl[h:h + 1])
    for name, t, r in zip(("dq", "dk", "dv", "dlambda"), got, ref):
        _check(t, r, f"V1 layer N=4096 head {h} {name}", tensor_core=True)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (8, 1), (16, 2)])
def test_backward_v2_group_sizes(Hq, Hkv):
    """dK and dV of a KV head sum both branches of every pair in its GQA group."""
    _case(2, 80, 80, "bf16", seed=760 + Hq, Hq=Hq, Hkv=Hkv)


def test_backward_v2_medium():
    """2048 tokens, 16 query heads over 2 KV heads, d = 128: several hundred keys per
    row, so rounding of long sums is exercised."""
    _case(2, 2048, 2048, "bf16", seed=770, Hq=16, Hkv=2)


@pytest.mark.parametrize("path", ["recompute", "saved"])
def test_backward_v2_full_size_one_kv_group(path):
    """The bench's backward workload at full size (B=1, N=4096, 64 query heads over 8 KV
    heads, d=128, the seeded synth.v2_backward tensors), run as the bench runs it (the
    recomputing backward, and the training forward + the backward from its saved outputs).
    The float64 oracle covers one seeded KV group: the dQ of its 8 query heads, its dK and
    dV (summed over the group's 4 pairs) and its 4 dlambda."""
    inp = synth.v2_backward()
    q, k, v = dev_tensor(inp.q), dev_tensor(inp.k), dev_tensor(inp.v)
    dy = dev_tensor(inp.extra["dy"])
    lam, _ = lambda_on_device(inp)
    if path == "recompute":
        dq, dk, dv, dl = da.diffattn_bwd_prefill(q, k, v, lam, dy)
    else:
        o, o2, lse = da.diffattn_fwd_prefill_train(q, k, v, lam)
        dq, dk, dv, dl = da.diffattn_bwd_prefill_saved(q, k, v, lam, o, o2, lse, dy)
    torch.cuda.synchronize()
    g = int(np.random.default_rng(1007).integers(inp.Hkv))
    group = inp.H // inp.Hkv
    h0, p0 = g * group, g * group // 2
    lam64 = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)[p0:p0 + group // 2]
    dy64 = synth.bf16_to_f32(inp.extra["dy"]).astype(np.float64)[:, :, p0:p0 + group // 2]
    ref = OB.prefill_v2_bwd(inp.as_f64("q")[:, :, h0:h0 + group], inp.as_f64("k")[:, :, g:g + 1],
                            inp.as_f64("v")[:, :, g:g + 1], lam64, dy64)
    tag = f"V2 N=4096 {path} KV group {g}"
    got = (dq[:, :, h0:h0 + group], dk[:, :, g:g + 1], dv[:, :, g:g + 1], dl[p0:p0 + group // 2])
    for name, t, r in zip(("dq", "dk", "dv", "dlambda"), got, ref):
        _check(t, r, f"{tag} {name}", tensor_core=True)


def test_lambda_bwd():
    inp = synth.v2_small(B=1, N=4, Hq=64, Hkv=8, seed=780)
    vecs = [dev_tensor(getattr(inp, n)) for n in ("lq1", "lk1", "lq2", "lk2")]
    dl = torch.randn(32, generator=torch.Generator().manual_seed(1)).cuda()
    got = da.diffattn_lambda_bwd(*vecs, dl)
    torch.cuda.synchronize()
    ref = OB.lambda_bwd(inp.lq1, inp.lk1, inp.lq2, inp.lk2, dl.cpu().numpy())
    for name, t, r in zip(("dlq1", "dlk1", "dlq2", "dlk2"), got, ref):
        _check(t, r, name)


@pytest.mark.parametrize("variant", [1, 2])
def test_backward_deterministic(variant):
    """No atomics: two calls give identical bits."""
    if variant == 1:
        inp = synth.v1_small(B=1, N=300, H=4, seed=791)
        oshape = (1, 300, 4, 128)
    else:
        inp = synth.v2_small(B=1, N=300, Hq=16, Hkv=2, seed=790)
        oshape = (1, 300, 8, 128)
    q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
    lam, li = lambda_on_device(inp)
    dy = torch.randn(oshape, generator=torch.Generator().manual_seed(2)).bfloat16().cuda()
    kw = dict(apply_norm=True) if variant == 1 else {}
    a = da.diffattn_bwd_prefill(q, k, v, lam, dy, li, **kw)
    b = da.diffattn_bwd_prefill(q, k, v, lam, dy, li, **kw)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)

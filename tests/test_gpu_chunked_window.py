"""GPU parity of chunked prefill (Nq < Nk queries at the last positions) and of the causal
sliding window, for the bf16 tcgen05 kernels (V1, V2) and the fp32 kernel, against the
float64 oracle; plus two properties that hold exactly on the device: a chunk's output is
bit-identical to the last rows of the full prefill, and window = Nk reproduces plain causal
attention bit-identically (the check the "Attention variants" page names for sliding-window
attention, Sliding window section)."""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, dev_tensor, lambda_on_device, out_f64

pytestmark = pytest.mark.gpu


def _inputs(variant, Nk, dtype="bf16", B=2, seed=0, causal=True):
    if variant == 1:
        return synth.v1_small(B=B, N=Nk, H=2, seed=300 + seed, dtype=dtype, causal=causal)
    return synth.v2_small(B=B, N=Nk, Hq=8, Hkv=2, seed=400 + seed, dtype=dtype, causal=causal)


def _run(inp, Nq, window=0, causal=True):
    q = dev_tensor(inp.q)[:, inp.N - Nq:].contiguous()
    k, v = dev_tensor(inp.k), dev_tensor(inp.v)
    lam, li = lambda_on_device(inp)
    out = da.diffattn_fwd_prefill(q, k, v, lam, li, causal=causal, apply_norm=inp.apply_norm,
                                  norm_eps=inp.eps, window=window)
    torch.cuda.synchronize()
    return out


def _ref(inp, Nq, window=0, causal=True):
    q = inp.as_f64("q")[:, inp.N - Nq:]
    k, v = inp.as_f64("k"), inp.as_f64("v")
    lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    if inp.variant == 1:
        return oracle.prefill_v1(q, k, v, lam, oracle.lambda_init(inp.depth), causal=causal,
                                 apply_norm=inp.apply_norm, eps=inp.eps, window=window)
    return oracle.prefill_v2(q, k, v, lam, causal=causal, window=window)


# (Nk, Nq, window): chunks that start inside a tile, a one-query chunk, windows narrower
# than a key tile, spanning several, equal to one, of one key, and the whole sequence
CASES = [(513, 100, 0), (513, 129, 0), (700, 1, 0), (300, 300, 64), (700, 257, 64),
         (640, 200, 128), (700, 300, 1), (1000, 390, 300), (333, 333, 333)]


@pytest.mark.parametrize("Nk,Nq,window", CASES)
@pytest.mark.parametrize("variant", [1, 2])
def test_bf16_chunk_window(variant, Nk, Nq, window):
    inp = _inputs(variant, Nk, seed=Nk + Nq + window)
    assert_parity(out_f64(_run(inp, Nq, window)), _ref(inp, Nq, window), "bf16",
                  f"V{variant} bf16 Nk={Nk} Nq={Nq} window={window}")


@pytest.mark.parametrize("Nk,Nq,window", [(300, 77, 0), (300, 300, 40), (257, 100, 1)])
@pytest.mark.parametrize("variant", [1, 2])
def test_f32_chunk_window(variant, Nk, Nq, window):
    inp = _inputs(variant, Nk, dtype="f32", seed=Nk + Nq + window)
    assert_parity(out_f64(_run(inp, Nq, window)), _ref(inp, Nq, window), "f32",
                  f"V{variant} f32 Nk={Nk} Nq={Nq} window={window}")


@pytest.mark.parametrize("variant", [1, 2])
def test_non_causal_chunk(variant):
    """causal = 0: every query of the chunk attends all Nk keys."""
    inp = _inputs(variant, 450, seed=7, causal=False)
    assert_parity(out_f64(_run(inp, 130, causal=False)), _ref(inp, 130, causal=False), "bf16",
                  f"V{variant} non-causal chunk")


@pytest.mark.parametrize("window", [0, 96])
@pytest.mark.parametrize("variant", [1, 2])
def test_chunk_is_last_rows_of_full_prefill(variant, window):
    """Each row's arithmetic depends only on its own scores and the keys it sees, so the
    rows of a chunk equal, bit for bit, the same rows of the full prefill."""
    inp = _inputs(variant, 900, seed=11)
    full = _run(inp, 900, window)
    for Nq in (1, 200, 451):
        part = _run(inp, Nq, window)
        assert torch.equal(part, full[:, 900 - Nq:]), (variant, window, Nq)


@pytest.mark.parametrize("variant", [1, 2])
def test_window_of_whole_sequence_is_causal(variant):
    inp = _inputs(variant, 611, seed=12)
    assert torch.equal(_run(inp, 611, window=611), _run(inp, 611, window=0))
    assert torch.equal(_run(inp, 200, window=5000), _run(inp, 200, window=0))


def test_rejects():
    inp = _inputs(2, 256)
    q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
    lam, _ = lambda_on_device(inp)
    with pytest.raises(da.DiffattnError):
        da.diffattn_fwd_prefill(q, k[:, :100], v[:, :100], lam)          # Nk < Nq
    with pytest.raises(da.DiffattnError):
        da.diffattn_fwd_prefill(q, k, v, lam, causal=False, window=16)   # window needs causal
    with pytest.raises(da.DiffattnError):
        da.diffattn_fwd_prefill(q, k, v, lam, window=-1)

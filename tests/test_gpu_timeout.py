"""The bounded-wait path, driven on purpose: a wait that nothing completes must end in
DIFFATTN_ERR_TIMEOUT within its bound, and the CUDA context must stay usable afterwards
(a prefill run right after it still matches the oracle). No fault, trap or hang is
involved: the wait gives up after a few hundred milliseconds."""
import time

import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
import oracle
from differential_attention_05_b200 import synth

from gpu_helpers import assert_parity, out_f64, run_prefill

pytestmark = pytest.mark.gpu

TIMEOUT = -6  # DIFFATTN_ERR_TIMEOUT


def test_wait_runs_out_and_reports():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    da.diffattn_selftest_timeout(st, timeout_ms=200)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == TIMEOUT
    assert 0.15 < dt < 5.0


def test_status_word_keeps_the_first_code():
    st = torch.full((1,), -3, dtype=torch.int32, device="cuda")
    da.diffattn_selftest_timeout(st, timeout_ms=50)
    torch.cuda.synchronize()
    assert int(st.item()) == -3


def test_context_usable_after_timeout():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    da.diffattn_selftest_timeout(st, timeout_ms=50)
    torch.cuda.synchronize()
    assert int(st.item()) == TIMEOUT
    inp = synth.v2_small(B=1, N=300, Hq=8, Hkv=2, seed=31)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = out_f64(run_prefill(inp, dev_status=st2))
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    ref = oracle.prefill_v2(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), lam, causal=inp.causal)
    assert_parity(out, ref, "bf16", "prefill after a timed-out wait")

"""diffattn_fwd_decode_static: the decode for callers that cannot allocate device memory
when they call (a serving loop on a budget fixed at start-up, a plugin whose host owns all
device memory). It must give what diffattn_fwd_decode gives with a caller workspace, on
consecutive calls that share the library's static array.

This file is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da
from differential_attention_05_b200 import _binding as B
from differential_attention_05_b200 import synth

from gpu_helpers import BF16_ATOL, BF16_REL_RMS, dev_tensor, errors, lambda_on_device, out_f64


def _too_big_params():
    p = B.DecodeParams()
    p.variant, p.dtype = B.DIFFATTN_V2, B.DIFFATTN_BF16
    p.batch, p.max_kv_len, p.n_q_heads, p.n_kv_heads, p.head_dim = 1024, 4096, 64, 8, 128
    p.q_strides[:] = (64 * 128, 128)
    p.kv_strides[:] = (4096 * 8 * 128, 8 * 128, 128)
    p.o_strides[:] = (32 * 128, 128)
    return p


def test_rejects_problems_larger_than_the_static_array():
    """Checked on the host before any CUDA call, so this runs without a GPU too."""
    lib = da.load_library()
    p = _too_big_params()
    rc = lib.diffattn_fwd_decode_static(ctypes.byref(p), None, None, None, None, None, None,
                                        None, None)
    assert rc == -4  # DIFFATTN_ERR_WORKSPACE
    p.batch, p.num_splits = 16, 4096 // 64  # fits unsplit, not with this explicit split count
    p.max_kv_len = 4096
    n = ctypes.c_size_t(0)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    assert n.value > (16 << 20), "the case must exceed the static array to test the rejection"
    assert lib.diffattn_fwd_decode_static(ctypes.byref(p), None, None, None, None, None, None,
                                          None, None) == -4


@pytest.mark.gpu
def test_matches_the_workspace_entry_point_on_consecutive_calls():
    outs = []
    for seed, kv in ((201, [4096, 17, 0, 2048, 1, 4000, 300, 4095]), (202, None)):
        inp = synth.v2_decode(B=8, L=4096, Hq=64, Hkv=8, seed=seed)
        q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
        lam, _ = lambda_on_device(inp)
        kl = None if kv is None else torch.tensor(kv, dtype=torch.int32, device="cuda")
        ref = da.diffattn_fwd_decode(q, k, v, lam, kv_len=kl)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = da.diffattn_fwd_decode_static(q, k, v, lam, kv_len=kl, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        g, r = out_f64(got), out_f64(ref)
        max_abs, rel_rms = errors(g, r)
        assert max_abs <= BF16_ATOL and rel_rms <= BF16_REL_RMS, (seed, max_abs, rel_rms)
        outs.append(g)
    # the second call did not inherit the first call's results
    assert not np.array_equal(outs[0], outs[1])


@pytest.mark.gpu
def test_full_size_decode_fits_with_fewer_splits():
    """Batch 64, cache 32768, 64/8 heads: the automatic split count is reduced until the
    partial states fit the 16 MiB array; the result still matches the workspace path."""
    g = torch.Generator(device="cuda")
    g.manual_seed(203)
    q = torch.randn((64, 64, 128), generator=g, device="cuda").bfloat16()
    k = torch.randn((64, 32768, 8, 128), generator=g, device="cuda").bfloat16()
    v = torch.randn((64, 32768, 8, 128), generator=g, device="cuda").bfloat16()
    lam = torch.full((32,), 0.8, dtype=torch.float32, device="cuda")
    ref = da.diffattn_fwd_decode(q, k, v, lam)
    got = da.diffattn_fwd_decode_static(q, k, v, lam)
    torch.cuda.synchronize()
    max_abs, rel_rms = errors(out_f64(got), out_f64(ref))
    assert max_abs <= BF16_ATOL and rel_rms <= BF16_REL_RMS, (max_abs, rel_rms)


@pytest.mark.gpu
def test_calls_after_the_first_take_no_device_memory():
    """After one warm-up call (which loads the library's module and so commits the static
    array), further calls leave the device's free memory unchanged: nothing is allocated,
    stream-ordered allocations included."""
    inp = synth.v2_decode(B=4, L=2048, Hq=64, Hkv=8, seed=204)
    q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
    lam, _ = lambda_on_device(inp)
    out = torch.empty((4, 32, 128), dtype=torch.bfloat16, device="cuda")
    da.diffattn_fwd_decode_static(q, k, v, lam, out=out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        da.diffattn_fwd_decode_static(q, k, v, lam, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)

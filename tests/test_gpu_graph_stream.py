"""Serving-style use of the boundary: calls captured into CUDA graphs and calls from several
host threads at once.

  * The lambda kernel, the V2 prefill, the V2 decode over a contiguous cache and over a
    paged one, captured into one CUDA graph on a non-default stream and replayed, give the
    eager calls' outputs bit for bit (the kernels are deterministic and allocate nothing).
  * Two host threads, each on its own stream, run the tensor-core backward (which forks its
    dQ kernel onto a library-owned second stream) over different inputs at the same time,
    several times; every result equals the same call made alone.
"""
import threading

import pytest
import torch

import differential_attention_05_b200 as da
from differential_attention_05_b200 import synth

from gpu_helpers import dev_tensor

pytestmark = pytest.mark.gpu


def test_forward_paths_in_one_cuda_graph():
    pre = synth.v2_small(B=1, N=300, Hq=16, Hkv=2, seed=930, causal=True)
    q, k, v = (dev_tensor(getattr(pre, n)) for n in ("q", "k", "v"))
    vecs = [dev_tensor(getattr(pre, n)) for n in ("lq1", "lk1", "lq2", "lk2")]
    dec = synth.v2_decode(B=3, L=700, Hq=64, Hkv=8, seed=931)
    dq_, dk_, dv_ = (dev_tensor(getattr(dec, n)) for n in ("q", "k", "v"))
    dvecs = [dev_tensor(getattr(dec, n)) for n in ("lq1", "lk1", "lq2", "lk2")]
    (kp, vp), bt = synth.paginate([dec.k, dec.v], 16, seed=932)
    kp, vp, bt = dev_tensor(kp), dev_tensor(vp), torch.from_numpy(bt).cuda()

    lam = torch.empty(8, dtype=torch.float32, device="cuda")
    li = torch.empty(1, dtype=torch.float32, device="cuda")
    dlam = torch.empty(32, dtype=torch.float32, device="cuda")
    dli = torch.empty(1, dtype=torch.float32, device="cuda")
    out = torch.empty((1, 300, 8, 128), dtype=torch.bfloat16, device="cuda")
    dout = torch.empty((3, 32, 128), dtype=torch.bfloat16, device="cuda")
    pout = torch.empty((3, 32, 128), dtype=torch.bfloat16, device="cuda")
    p = da._binding.decode_params(dq_, dk_, dv_, dout)
    ws = torch.empty(da._binding.diffattn_decode_workspace_size(p), dtype=torch.uint8, device="cuda")
    pws = torch.empty(2 * ws.numel(), dtype=torch.uint8, device="cuda")

    def run():
        da.diffattn_lambda(*vecs, depth=pre.depth, lambda_out=lam, lambda_init_out=li)
        da.diffattn_fwd_prefill(q, k, v, lam, li, out=out)
        da.diffattn_lambda(*dvecs, depth=dec.depth, lambda_out=dlam, lambda_init_out=dli)
        da.diffattn_fwd_decode(dq_, dk_, dv_, dlam, out=dout, workspace=ws)
        da.diffattn_fwd_decode_paged(dq_, kp, vp, bt, dlam, out=pout, workspace=pws,
                                     max_kv_len=dec.N)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (lam, out, dlam, dout, pout)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for t in (out, dout, pout):
        t.fill_(float("nan"))
    lam.fill_(float("nan"))
    dlam.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for name, x, y in zip(("lambda", "prefill", "lambda (decode)", "decode", "paged decode"),
                          (lam, out, dlam, dout, pout), eager):
        assert torch.equal(x, y), name
    # the paged and contiguous decodes read the same cache rows
    assert torch.equal(dout, pout)
    del graph


def test_backward_from_two_host_threads():
    cases = []
    for i in range(2):
        inp = synth.v2_small(B=1, N=400 + 64 * i, Hq=16, Hkv=2, seed=940 + i, causal=True)
        q, k, v = (dev_tensor(getattr(inp, n)) for n in ("q", "k", "v"))
        vecs = [dev_tensor(getattr(inp, n)) for n in ("lq1", "lk1", "lq2", "lk2")]
        lam, _ = da.diffattn_lambda(*vecs, depth=inp.depth)
        g = torch.Generator().manual_seed(950 + i)
        dy = torch.randn((1, inp.N, 8, 128), generator=g).bfloat16().cuda()
        cases.append((q, k, v, lam, dy))
    torch.cuda.synchronize()
    alone = []
    for q, k, v, lam, dy in cases:
        alone.append([t.clone() for t in da.diffattn_bwd_prefill(q, k, v, lam, dy)])
    torch.cuda.synchronize()

    results, errors = [[], []], []

    def worker(i):
        try:
            q, k, v, lam, dy = cases[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(6):
                    results[i].append([t.clone() for t in da.diffattn_bwd_prefill(q, k, v, lam, dy)])
            s.synchronize()
        except Exception as e:  # surfaced in the main thread below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a backward thread did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    for i in range(2):
        assert len(results[i]) == 6
        for r in results[i]:
            for name, x, y in zip(("dq", "dk", "dv", "dlambda"), r, alone[i]):
                assert torch.equal(x, y), f"thread {i} {name}"

"""Shared helpers of the GPU parity tests: move seeded inputs to the device, run the
library through its C ABI binding, and compare with the oracle."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import differential_attention_05_b200 as da
from differential_attention_05_b200 import synth

F32_ATOL = 1e-5            # fp32 configurations: max abs error
BF16_ATOL = 2e-2           # bf16 configurations: max abs error ...
BF16_REL_RMS = 5e-3        # ... and relative RMS error


def dev_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def lambda_on_device(inp: synth.Inputs, device="cuda"):
    vecs = [dev_tensor(getattr(inp, n), device) for n in ("lq1", "lk1", "lq2", "lk2")]
    lam, li = da.diffattn_lambda(*vecs, depth=inp.depth)
    return lam, li


def run_prefill(inp: synth.Inputs, device="cuda", dev_status=None):
    q, k, v = (dev_tensor(getattr(inp, n), device) for n in ("q", "k", "v"))
    lam, li = lambda_on_device(inp, device)
    out = da.diffattn_fwd_prefill(q, k, v, lam, li, causal=inp.causal,
                                  apply_norm=inp.apply_norm, norm_eps=inp.eps,
                                  dev_status=dev_status)
    torch.cuda.synchronize()
    return out


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def errors(gpu: np.ndarray, ref: np.ndarray):
    diff = gpu - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rms_ref = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    rel_rms = float(np.sqrt(np.mean(diff * diff)) / rms_ref) if rms_ref > 0 else 0.0
    return max_abs, rel_rms


def _log(what, max_abs, rel_rms):
    path = os.environ.get("DIFFATTN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, "max_abs": max_abs, "rel_rms": rel_rms}) + "\n")


def assert_parity(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    max_abs, rel_rms = errors(gpu, ref)
    _log(what, max_abs, rel_rms)
    if dtype == "f32":
        assert max_abs <= F32_ATOL, f"{what}: max abs {max_abs:.3e} > {F32_ATOL}"
    else:
        assert max_abs <= BF16_ATOL, f"{what}: max abs {max_abs:.3e} > {BF16_ATOL}"
        assert rel_rms <= BF16_REL_RMS, f"{what}: rel RMS {rel_rms:.3e} > {BF16_REL_RMS}"
    return max_abs, rel_rms

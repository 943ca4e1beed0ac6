"""GPU parity of the split-KV decode over a paged KV cache (diffattn_fwd_decode_paged),
V2 and V1, against the float64 oracle; bit-identity with the contiguous decode (only the
row addresses differ); an out-of-pool block-table entry reported through dev_status."""
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


def _paged(inp, page_size, kv_len, fill="nan", seed=5):
    """Device copies of the query, the shuffled page pools and the block table. The rows
    past kv_len[b] are set to NaN in the pool too, so any read of them would show."""
    k, v = inp.k.copy(), inp.v.copy()
    if fill == "nan":
        for b, n in enumerate(kv_len):
            k[b, n:] = 0x7FC0
            v[b, n:] = 0x7FC0
    (kp, vp), bt = synth.paginate([k, v], page_size, seed=seed, fill=fill)
    return dev_tensor(kp), dev_tensor(vp), torch.from_numpy(bt).cuda()


@pytest.mark.parametrize("page_size", [1, 4, 8, 16, 64, 256])
def test_v2_paged(page_size):
    L = 1000
    kv_len = [1000, 1, 513]
    inp = synth.v2_decode(B=3, L=L, Hq=16, Hkv=2, seed=120 + page_size)
    kp, vp, bt = _paged(inp, page_size, kv_len)
    lam, _ = lambda_on_device(inp)
    kl = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    q = dev_tensor(inp.q)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, kv_len=kl, max_kv_len=L, num_splits=3,
                                       dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.decode_v2(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _lam(inp), kv_len=kv_len)
    assert_parity(out_f64(out), ref, "bf16", f"V2 paged page={page_size}")
    # same kernel, same splits: bit-identical to the contiguous cache
    cont = da.diffattn_fwd_decode(q, dev_tensor(inp.k), dev_tensor(inp.v), lam, kv_len=kl, num_splits=3)
    torch.cuda.synchronize()
    assert torch.equal(out, cont)


@pytest.mark.parametrize("page_size", [1, 32, 128])
def test_v1_paged(page_size):
    L = 700
    kv_len = [700, 65, 64]
    inp = synth.v1_decode(B=3, L=L, H=4, seed=130 + page_size)
    kp, vp, bt = _paged(inp, page_size, kv_len)
    lam, li = lambda_on_device(inp)
    kl = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    q = dev_tensor(inp.q)
    out = da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, kv_len=kl, lambda_init=li, max_kv_len=L,
                                       norm_eps=inp.eps, num_splits=2)
    torch.cuda.synchronize()
    ref = oracle.decode_v1(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _lam(inp),
                           oracle.lambda_init(inp.depth), kv_len=kv_len, eps=inp.eps)
    assert_parity(out_f64(out), ref, "bf16", f"V1 paged page={page_size}")
    cont = da.diffattn_fwd_decode_v1(q, dev_tensor(inp.k), dev_tensor(inp.v), lam, li, kv_len=kl,
                                     norm_eps=inp.eps, num_splits=2)
    torch.cuda.synchronize()
    assert torch.equal(out, cont)


def test_paged_default_length_and_spare_pages():
    """kv_len NULL: every entry holds max_kv_len = page_size x table width keys; the pool
    has unused noise pages that the table never names."""
    inp = synth.v2_decode(B=2, L=512, Hq=8, Hkv=1, seed=140)
    kp, vp, bt = _paged(inp, 64, [512, 512], fill="noise")
    lam, _ = lambda_on_device(inp)
    out = da.diffattn_fwd_decode_paged(dev_tensor(inp.q), kp, vp, bt, lam)
    torch.cuda.synchronize()
    ref = oracle.decode_v2(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _lam(inp))
    assert_parity(out_f64(out), ref, "bf16", "V2 paged, full length")


@pytest.mark.parametrize("bad", [-1, 10 ** 6])
def test_out_of_pool_page_is_reported(bad):
    """A block-table entry outside the pool is not followed: its rows read as zeros and
    DIFFATTN_ERR_INVALID_ARG lands in dev_status; other entries are unaffected."""
    inp = synth.v2_decode(B=2, L=256, Hq=8, Hkv=1, seed=141)
    kp, vp, bt = _paged(inp, 16, [256, 256], fill="noise")
    bt[1, 3] = bad
    lam, _ = lambda_on_device(inp)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = da.diffattn_fwd_decode_paged(dev_tensor(inp.q), kp, vp, bt, lam, num_splits=1, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == -1
    ref = oracle.decode_v2(inp.as_f64("q")[:1], inp.as_f64("k")[:1], inp.as_f64("v")[:1], _lam(inp))
    assert_parity(out_f64(out[:1]), ref, "bf16", "entry with a valid table")
    assert torch.isfinite(out.float()).all()


def test_paged_rejects():
    inp = synth.v2_decode(B=1, L=128, Hq=8, Hkv=1, seed=142)
    kp, vp, bt = _paged(inp, 16, [128], fill="noise")
    lam, _ = lambda_on_device(inp)
    q = dev_tensor(inp.q)
    with pytest.raises(da.DiffattnError):  # capacity below max_kv_len
        da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, max_kv_len=129)
    with pytest.raises(da.DiffattnError):  # V2 has no norm
        da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, apply_norm=True)
    kp3, vp3, bt3 = _paged(inp, 16, [128], fill="noise")
    with pytest.raises(da.DiffattnError):  # page size not a power of two
        da.diffattn_fwd_decode_paged(q, kp3[:, :12], vp3[:, :12], bt3, lam, max_kv_len=96)

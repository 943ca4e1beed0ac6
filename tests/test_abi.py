"""The C-ABI library (no GPU needed): it loads, exports every entry point the header
declares, and rejects bad arguments on the host before launching anything. No call here
reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import differential_attention_05_b200 as da
from differential_attention_05_b200 import _binding as B
from differential_attention_05_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "diffattn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return da.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w[\w\s\*]*?\b(diffattn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    assert set(declared_functions()) == set(B.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from {da.library_path()}"


def test_version_and_status_strings(lib):
    assert lib.diffattn_version() == 100
    for code in range(-6, 1):
        assert da.diffattn_status_string(code)
    assert da.diffattn_status_string(-99) == "unknown status"


def _prefill_params(**kw):
    p = B.PrefillParams()
    p.variant, p.dtype, p.batch, p.seqlen = B.DIFFATTN_V2, B.DIFFATTN_BF16, 1, 256
    p.n_q_heads, p.n_kv_heads, p.head_dim = 16, 2, 128
    p.causal, p.apply_norm, p.norm_eps = 1, 0, 1e-5
    N = p.seqlen
    p.q_strides[:] = (N * 16 * 128, 16 * 128, 128)
    p.k_strides[:] = (N * 2 * 128, 2 * 128, 128)
    p.v_strides[:] = (N * 2 * 128, 2 * 128, 128)
    p.o_strides[:] = (N * 8 * 128, 8 * 128, 128)
    for k_, v_ in kw.items():
        setattr(p, k_, v_)
    return p


GOOD = 1 << 20  # a 16-byte-aligned stand-in address; validation never dereferences it


def _call_prefill(lib, p, q=GOOD, k=GOOD + 4096, v=GOOD + 8192, lam=GOOD + 12288, li=None,
                  out=GOOD + 16384):
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.diffattn_fwd_prefill(ctypes.byref(p), vp(q), vp(k), vp(v), vp(lam), vp(li), vp(out),
                                    None, None)


@pytest.mark.parametrize("field,value,code", [
    ("variant", 3, -1), ("dtype", 7, -1), ("batch", -1, -1), ("seqlen", -5, -1),
    ("n_kv_heads", 3, -1),    # 16 % 3 != 0
    ("n_kv_heads", 16, -1),   # group of 1 cannot hold a pair
    ("apply_norm", 1, -1),    # V2 has no per-head norm
    ("causal", 2, -1),
    ("head_dim", 96, -2),     # bf16 V2 needs d = 128
    ("kv_seqlen", 255, -1),   # fewer keys than queries
    ("window", -1, -1),
])
def test_prefill_rejects(lib, field, value, code):
    assert _call_prefill(lib, _prefill_params(**{field: value})) == code


def test_prefill_rejects_null_and_alias_and_misalignment(lib):
    p = _prefill_params()
    assert lib.diffattn_fwd_prefill(None, None, None, None, None, None, None, None, None) == -1
    assert _call_prefill(lib, p, q=None) == -1
    assert _call_prefill(lib, p, out=GOOD) == -1                 # out aliases q
    assert _call_prefill(lib, p, k=GOOD + 4098) == -3            # not 16-byte aligned
    p2 = _prefill_params()
    p2.q_strides[1] = 16 * 128 + 4                               # token stride not 16 B multiple
    assert _call_prefill(lib, p2) == -3


def test_prefill_window_needs_causal(lib):
    assert _call_prefill(lib, _prefill_params(causal=0, window=16)) == -1


def test_prefill_params_layout():
    """The two chunked-prefill fields sit after the stride arrays (ABI append-only)."""
    assert B.PrefillParams.kv_seqlen.offset == B.PrefillParams.o_strides.offset + 24
    assert B.PrefillParams.window.offset == B.PrefillParams.kv_seqlen.offset + 4


def test_prefill_empty_problem_launches_nothing(lib):
    assert _call_prefill(lib, _prefill_params(batch=0), q=None, k=None, v=None, out=None) == 0
    assert _call_prefill(lib, _prefill_params(seqlen=0), q=None, k=None, v=None, out=None) == 0


def test_v1_requires_lambda_init_when_normalising(lib):
    p = _prefill_params(variant=B.DIFFATTN_V1, n_q_heads=4, n_kv_heads=4, head_dim=64, apply_norm=1)
    assert _call_prefill(lib, p, li=None) == -1


def _decode_params(B_=4, L=1000, Hq=64, Hkv=8, d=128, splits=0):
    p = B.DecodeParams()
    p.variant, p.dtype = B.DIFFATTN_V2, B.DIFFATTN_BF16
    p.batch, p.max_kv_len, p.n_q_heads, p.n_kv_heads, p.head_dim, p.num_splits = B_, L, Hq, Hkv, d, splits
    p.q_strides[:] = (Hq * d, d)
    p.kv_strides[:] = (L * Hkv * d, Hkv * d, d)
    p.o_strides[:] = (Hq // 2 * d, d)
    return p


def test_decode_workspace_size(lib):
    n = ctypes.c_size_t(0)
    p = _decode_params(B_=4, L=1000, splits=3)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    # 3 splits of 384 keys (rounded up to the 64-key chunk): 4 * 64 heads * 3 records
    recs = 4 * 64 * 3
    assert n.value == ((recs * 128 * 4 + 255) // 256) * 256 + recs * 2 * 4
    p = _decode_params(Hq=64, Hkv=16)  # group of 4: not this build's decode shape
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == -2
    p = _decode_params()
    p.variant = B.DIFFATTN_V1  # V1 needs one cache per head (Hq == Hkv)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == -1


def _decode_params_v1(B_=4, L=1000, H=16, d=64, splits=0):
    p = B.DecodeParams()
    p.variant, p.dtype = B.DIFFATTN_V1, B.DIFFATTN_BF16
    p.batch, p.max_kv_len, p.n_q_heads, p.n_kv_heads, p.head_dim, p.num_splits = B_, L, H, H, d, splits
    p.q_strides[:] = (H * 2 * d, 2 * d)
    p.kv_strides[:] = (L * H * 2 * d, H * 2 * d, 2 * d)
    p.o_strides[:] = (H * 2 * d, 2 * d)
    return p


def test_decode_v1_workspace_size(lib):
    n = ctypes.c_size_t(0)
    p = _decode_params_v1(B_=4, L=1000, H=16, splits=3)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    # 3 splits; per (b, h, split) two branch records of 2d = 128 floats and (max, sum)
    recs = 4 * 16 * 3 * 2
    assert n.value == ((recs * 128 * 4 + 255) // 256) * 256 + recs * 2 * 4
    p = _decode_params_v1(d=128)  # this build's V1 decode takes d = 64
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == -2


def test_decode_v1_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_fwd_decode_v1
    p = _decode_params_v1(B_=2, L=512, H=4)
    n = ctypes.c_size_t(0)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    ptrs = [vp(GOOD), vp(GOOD + 4096), vp(GOOD + 8192), None, vp(GOOD + 12288)]
    ws = vp(GOOD * 4)
    # V2 parameters through the V1 entry point
    p2 = _decode_params(B_=2, L=512)
    assert f(ctypes.byref(p2), *ptrs, vp(GOOD), 1, 1e-5, vp(GOOD + 16384), ws, n.value, None, None) == -1
    # apply_norm without lambda_init, a bad flag, a bad eps
    assert f(ctypes.byref(p), *ptrs, None, 1, 1e-5, vp(GOOD + 16384), ws, n.value, None, None) == -1
    assert f(ctypes.byref(p), *ptrs, vp(GOOD), 2, 1e-5, vp(GOOD + 16384), ws, n.value, None, None) == -1
    assert f(ctypes.byref(p), *ptrs, vp(GOOD), 1, -1.0, vp(GOOD + 16384), ws, n.value, None, None) == -1
    # workspace too small / missing / misaligned; misaligned query
    assert f(ctypes.byref(p), *ptrs, vp(GOOD), 1, 1e-5, vp(GOOD + 16384), ws, n.value - 1, None, None) == -4
    assert f(ctypes.byref(p), *ptrs, vp(GOOD), 1, 1e-5, vp(GOOD + 16384), None, n.value, None, None) == -4
    assert f(ctypes.byref(p), *ptrs, vp(GOOD), 1, 1e-5, vp(GOOD + 16384), vp(GOOD * 4 + 16), n.value, None, None) == -3
    bad = [vp(GOOD + 2)] + ptrs[1:]
    assert f(ctypes.byref(p), *bad, vp(GOOD), 1, 1e-5, vp(GOOD + 16384), ws, n.value, None, None) == -3


def test_decode_rejects_small_workspace(lib):
    p = _decode_params(B_=2, L=512)
    n = ctypes.c_size_t(0)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    vp = ctypes.c_void_p
    args = [vp(GOOD), vp(GOOD + 4096), vp(GOOD + 8192), None, vp(GOOD + 12288), vp(GOOD + 16384)]
    assert lib.diffattn_fwd_decode(ctypes.byref(p), *args, vp(GOOD * 4), n.value - 1, None, None) == -4
    assert lib.diffattn_fwd_decode(ctypes.byref(p), *args, None, n.value, None, None) == -4
    assert lib.diffattn_fwd_decode(ctypes.byref(p), *args, vp(GOOD * 4 + 16), n.value, None, None) == -3


def test_lambda_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_lambda
    assert f(None, vp(GOOD), vp(GOOD), vp(GOOD), 4, 64, 1, vp(GOOD), None, None) == -1
    assert f(vp(GOOD), vp(GOOD), vp(GOOD), vp(GOOD), 0, 64, 1, vp(GOOD), None, None) == -1
    assert f(vp(GOOD), vp(GOOD), vp(GOOD), vp(GOOD), 4, 64, 0, vp(GOOD), None, None) == -1
    assert f(vp(GOOD + 4), vp(GOOD), vp(GOOD), vp(GOOD), 4, 64, 1, vp(GOOD), None, None) == -3


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setenv("DIFFATTN_LIBRARY", str(tmp_path / "nope.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        B.load_library()


def test_selftest_timeout_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_selftest_timeout
    assert f(None, 100, None) == -1
    assert f(vp(GOOD), 0, None) == -1
    assert f(vp(GOOD), 10001, None) == -1


def test_selftest_exp2_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_selftest_exp2
    assert f(vp(GOOD), vp(GOOD), vp(GOOD), -1, None) == -1
    assert f(None, vp(GOOD), vp(GOOD), 8, None) == -1
    assert f(vp(GOOD), vp(GOOD), None, 8, None) == -1
    assert f(None, None, None, 0, None) == 0  # nothing to do, nothing launched


def test_train_and_saved_backward_reject(lib):
    vp = ctypes.c_void_p
    assert lib.diffattn_fwd_prefill_train(None, *([None] * 9)) == -1
    assert lib.diffattn_bwd_prefill_saved(None, *([None] * 13), 0, None, None) == -1
    p = B.PrefillParams()
    p.variant, p.dtype, p.batch, p.seqlen, p.n_q_heads, p.n_kv_heads, p.head_dim = 1, 1, 1, 8, 2, 2, 64
    p.causal = 1
    assert lib.diffattn_fwd_prefill_train(ctypes.byref(p), *([vp(GOOD)] * 7), None, None) == -2  # V1
    p.variant, p.n_q_heads, p.n_kv_heads, p.head_dim = 2, 4, 2, 64
    assert lib.diffattn_fwd_prefill_train(ctypes.byref(p), *([vp(GOOD)] * 7), None, None) == -2  # d != 128


def test_debug_bounds_violations_normal_build(lib):
    f = lib.diffattn_debug_bounds_violations
    assert f(None) == -1
    n = ctypes.c_int32(7)
    assert f(ctypes.byref(n)) == -2 and n.value == 0  # the normal build counts nothing


def _paged(page_size=16, num_pages=64, max_pages=8, strides=(16 * 8 * 128, 8 * 128, 128)):
    pk = B.PagedKV()
    pk.page_size, pk.num_pages, pk.max_pages_per_seq = page_size, num_pages, max_pages
    pk.page_strides[:] = strides
    return pk


def test_decode_paged_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_fwd_decode_paged
    p = _decode_params(B_=2, L=128)
    n = ctypes.c_size_t(0)
    assert lib.diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    ws = vp(GOOD * 4)

    def call(pk, bt=vp(GOOD + 20480), norm=0, params=p):
        return f(ctypes.byref(params), ctypes.byref(pk), vp(GOOD), vp(GOOD + 4096), vp(GOOD + 8192),
                 bt, None, vp(GOOD + 12288), None, norm, 1e-5, vp(GOOD + 16384), ws, n.value, None, None)

    assert f(ctypes.byref(p), None, vp(GOOD), vp(GOOD), vp(GOOD), vp(GOOD), None, vp(GOOD), None, 0,
             1e-5, vp(GOOD), ws, n.value, None, None) == -1             # no pool geometry
    assert call(_paged(page_size=12)) == -1                             # not a power of two
    assert call(_paged(page_size=0)) == -1
    assert call(_paged(max_pages=7)) == -1                               # 7 x 16 < 128 keys
    assert call(_paged(num_pages=0)) == -1
    bad = _paged()
    bad.reserved = 1
    assert call(bad) == -1
    assert call(_paged(), bt=None) == -1                                 # no block table
    assert call(_paged(), norm=1) == -1                                  # V2 has no norm
    assert call(_paged(strides=(16 * 8 * 128, 8 * 128 + 4, 128))) == -3  # token stride
    pv1 = _decode_params_v1(B_=2, L=128, H=4)
    assert call(_paged(), params=pv1, norm=1) == -1                      # V1 norm needs lambda_init


def test_prefill_varlen_rejects(lib):
    vp = ctypes.c_void_p
    f = lib.diffattn_fwd_prefill_varlen
    p = _prefill_params()
    p.batch, p.seqlen, p.kv_seqlen = 3, 256, 300
    for st in (p.q_strides, p.k_strides, p.v_strides, p.o_strides):
        st[0] = 0
    args = [vp(GOOD), vp(GOOD + 4096), vp(GOOD + 8192), vp(GOOD + 12288), None, vp(GOOD + 16384)]
    cu_q, cu_k = vp(GOOD + 20480), vp(GOOD + 24576)
    assert f(ctypes.byref(p), None, cu_k, 128, *args, None, None) == -1      # no offsets
    assert f(ctypes.byref(p), cu_q, None, 128, *args, None, None) == -1
    assert f(ctypes.byref(p), cu_q, cu_k, -1, *args, None, None) == -1       # bad max length
    assert f(ctypes.byref(p), vp(GOOD + 20482), cu_k, 128, *args, None, None) == -3  # misaligned
    p.window, p.causal = 8, 0
    assert f(ctypes.byref(p), cu_q, cu_k, 128, *args, None, None) == -1      # window needs causal
    p.window, p.causal = 0, 1
    assert f(ctypes.byref(p), cu_q, cu_k, 0, *args, None, None) == 0         # nothing to launch


def test_backward_workspace_and_rejects(lib):
    vp = ctypes.c_void_p
    p = _prefill_params()  # V2, B=1, N=256, Hq=16, Hkv=2, d=128: tensor-core backward
    n = ctypes.c_size_t(0)
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    rows = 1 * 256 * 8
    up = lambda x: (x + 255) // 256 * 256
    # per (entry, pair): N + 64 rows of (lse_1, lse_2, delta_1, delta_2), then N dlambda shares
    assert n.value == up(8 * (256 + 64) * 16) + up(rows * 4)
    pf = _prefill_params(dtype=B.DIFFATTN_F32)  # exact-fp32 kernels: dO rows as well
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(pf), ctypes.byref(n)) == 0
    assert n.value == up(rows * 128 * 4) + up(rows * 16) + up(rows * 4)
    big = _prefill_params(head_dim=256)
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(big), ctypes.byref(n)) == -2
    # V1 (H = 4 heads): bf16 with d = 64 takes the tensor-core path, whose workspace adds
    # the bf16 dO through the norm [B, N, H, 2d]; bf16 with another d and fp32 take the
    # exact kernels (fp32 dO rows of width 2d)
    v1 = lambda **kw: _prefill_params(variant=B.DIFFATTN_V1, n_q_heads=4, n_kv_heads=4, apply_norm=1, **kw)
    r1 = 256 * 4
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(v1(head_dim=64)), ctypes.byref(n)) == 0
    assert n.value == up(4 * (256 + 64) * 16) + up(r1 * 4) + up(r1 * 128 * 2)
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(v1(head_dim=32)), ctypes.byref(n)) == 0
    assert n.value == up(r1 * 64 * 4) + up(r1 * 16) + up(r1 * 4)
    assert lib.diffattn_bwd_workspace_size(ctypes.byref(v1(head_dim=64, dtype=B.DIFFATTN_F32)),
                                           ctypes.byref(n)) == 0
    assert n.value == up(r1 * 128 * 4) + up(r1 * 16) + up(r1 * 4)
    f = lib.diffattn_bwd_prefill
    ptr = [vp(GOOD), vp(GOOD + 4096), vp(GOOD + 8192), vp(GOOD + 12288), None, vp(GOOD + 16384)]
    outs = [vp(GOOD + 20480), vp(GOOD + 24576), vp(GOOD + 28672), vp(GOOD + 32768)]
    need = up(8 * (256 + 64) * 16) + up(rows * 4)
    assert f(ctypes.byref(p), *ptr, *outs, vp(GOOD * 4), need - 1, None, None) == -4
    assert f(ctypes.byref(p), *ptr, *outs, None, need, None, None) == -4
    assert f(ctypes.byref(p), *ptr, vp(GOOD + 20484), *outs[1:], vp(GOOD * 4), need, None, None) == -3
    assert f(ctypes.byref(p), *ptr, None, *outs[1:], vp(GOOD * 4), need, None, None) == -1
    assert lib.diffattn_lambda_bwd(None, vp(GOOD), vp(GOOD), vp(GOOD), 4, 64, vp(GOOD),
                                   vp(GOOD), vp(GOOD), vp(GOOD), vp(GOOD), None) == -1


def _declared_arity():
    """Number of parameters of every entry point as include/diffattn.h declares it."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(diffattn_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    """The binding's ctypes signatures have the header's parameter counts (catches an entry
    point whose C signature changed without its binding)."""
    arity = _declared_arity()
    assert set(arity) == set(B.EXPORTS)
    for name in B.EXPORTS:
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, f"{name}: no argtypes"
        assert len(argtypes) == arity[name], f"{name}: binding {len(argtypes)} vs header {arity[name]}"


def test_plain_c_program(lib, tmp_path):
    """A plain C program compiled against include/diffattn.h and linked to the library runs
    the host-side paths (no GPU): the boundary is a C ABI, not a Python one."""
    import subprocess
    src = os.path.join(ROOT, "tests", "c", "abi_host.c")
    exe = str(tmp_path / "abi_host")
    libdir = os.path.dirname(da.library_path())
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"), src,
                           "-L", libdir, "-l:" + os.path.basename(da.library_path()),
                           "-Wl,-rpath," + libdir, "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "all checks hold" in r.stdout

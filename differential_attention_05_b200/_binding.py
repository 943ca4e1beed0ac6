"""ctypes binding over libdiffattn.so (include/diffattn.h).

Argument marshalling only: tensors become pointers, shapes and element strides become
the parameter structs, and the current torch CUDA stream becomes the launch stream.
Every step of the operator runs in the library's kernels. There is no fallback: if the
library is missing or a call fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libdiffattn.so"

DIFFATTN_F32, DIFFATTN_BF16 = 0, 1
DIFFATTN_V1, DIFFATTN_V2 = 1, 2

STATUS = {
    0: "DIFFATTN_OK",
    -1: "DIFFATTN_ERR_INVALID_ARG",
    -2: "DIFFATTN_ERR_UNSUPPORTED",
    -3: "DIFFATTN_ERR_MISALIGNED",
    -4: "DIFFATTN_ERR_WORKSPACE",
    -5: "DIFFATTN_ERR_CUDA",
    -6: "DIFFATTN_ERR_TIMEOUT",
}

# every symbol include/diffattn.h declares
EXPORTS = (
    "diffattn_version",
    "diffattn_status_string",
    "diffattn_lambda",
    "diffattn_fwd_prefill",
    "diffattn_fwd_prefill_varlen",
    "diffattn_bwd_workspace_size",
    "diffattn_bwd_prefill",
    "diffattn_lambda_bwd",
    "diffattn_fwd_prefill_train",
    "diffattn_bwd_prefill_saved",
    "diffattn_decode_workspace_size",
    "diffattn_fwd_decode",
    "diffattn_fwd_decode_static",
    "diffattn_fwd_decode_v1",
    "diffattn_fwd_decode_paged",
    "diffattn_selftest_timeout",
    "diffattn_selftest_exp2",
    "diffattn_debug_bounds_violations",
)


class DiffattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, 'unknown')})")


class PrefillParams(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("seqlen", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("apply_norm", ctypes.c_int32),
        ("norm_eps", ctypes.c_float),
        ("q_strides", ctypes.c_int64 * 3),
        ("k_strides", ctypes.c_int64 * 3),
        ("v_strides", ctypes.c_int64 * 3),
        ("o_strides", ctypes.c_int64 * 3),
        ("kv_seqlen", ctypes.c_int32),
        ("window", ctypes.c_int32),
    ]


class DecodeParams(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("max_kv_len", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("num_splits", ctypes.c_int32),
        ("q_strides", ctypes.c_int64 * 2),
        ("kv_strides", ctypes.c_int64 * 3),
        ("o_strides", ctypes.c_int64 * 2),
    ]


_lib = None


def library_path() -> str:
    return os.environ.get("DIFFATTN_LIBRARY", os.path.join(_HERE, _LIB_NAME))


def load_library():
    """Load libdiffattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m differential_attention_05_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i32, f32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    lib.diffattn_version.restype = i32
    lib.diffattn_version.argtypes = []
    lib.diffattn_status_string.restype = ctypes.c_char_p
    lib.diffattn_status_string.argtypes = [i32]
    lib.diffattn_lambda.restype = i32
    lib.diffattn_lambda.argtypes = [f32p, f32p, f32p, f32p, i32, i32, i32, f32p, f32p, vp]
    lib.diffattn_fwd_prefill.restype = i32
    lib.diffattn_fwd_prefill.argtypes = [ctypes.POINTER(PrefillParams), vp, vp, vp, f32p, f32p,
                                         vp, vp, vp]
    lib.diffattn_fwd_prefill_varlen.restype = i32
    lib.diffattn_fwd_prefill_varlen.argtypes = [ctypes.POINTER(PrefillParams), vp, vp, i32, vp, vp,
                                                vp, f32p, f32p, vp, vp, vp]
    lib.diffattn_bwd_workspace_size.restype = i32
    lib.diffattn_bwd_workspace_size.argtypes = [ctypes.POINTER(PrefillParams),
                                                ctypes.POINTER(ctypes.c_size_t)]
    lib.diffattn_bwd_prefill.restype = i32
    lib.diffattn_bwd_prefill.argtypes = [ctypes.POINTER(PrefillParams), vp, vp, vp, f32p, f32p, vp,
                                         vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
    lib.diffattn_fwd_prefill_train.restype = i32
    lib.diffattn_fwd_prefill_train.argtypes = [ctypes.POINTER(PrefillParams), vp, vp, vp, f32p, vp, vp,
                                               f32p, vp, vp]
    lib.diffattn_bwd_prefill_saved.restype = i32
    lib.diffattn_bwd_prefill_saved.argtypes = [ctypes.POINTER(PrefillParams), vp, vp, vp, f32p, vp, vp,
                                               f32p, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
    lib.diffattn_lambda_bwd.restype = i32
    lib.diffattn_lambda_bwd.argtypes = [f32p, f32p, f32p, f32p, i32, i32, f32p, vp, vp, vp, vp, vp]
    lib.diffattn_decode_workspace_size.restype = i32
    lib.diffattn_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeParams),
                                                   ctypes.POINTER(ctypes.c_size_t)]
    lib.diffattn_fwd_decode.restype = i32
    lib.diffattn_fwd_decode.argtypes = [ctypes.POINTER(DecodeParams), vp, vp, vp, vp, f32p, vp,
                                        vp, ctypes.c_size_t, vp, vp]
    lib.diffattn_fwd_decode_static.restype = i32
    lib.diffattn_fwd_decode_static.argtypes = [ctypes.POINTER(DecodeParams), vp, vp, vp, vp, f32p,
                                               vp, vp, vp]
    lib.diffattn_fwd_decode_v1.restype = i32
    lib.diffattn_fwd_decode_v1.argtypes = [ctypes.POINTER(DecodeParams), vp, vp, vp, vp, f32p, f32p,
                                           i32, ctypes.c_float, vp, vp, ctypes.c_size_t, vp, vp]
    lib.diffattn_fwd_decode_paged.restype = i32
    lib.diffattn_fwd_decode_paged.argtypes = [ctypes.POINTER(DecodeParams), ctypes.POINTER(PagedKV),
                                              vp, vp, vp, vp, vp, f32p, f32p, i32, ctypes.c_float,
                                              vp, vp, ctypes.c_size_t, vp, vp]
    lib.diffattn_selftest_timeout.restype = i32
    lib.diffattn_selftest_timeout.argtypes = [vp, i32, vp]
    lib.diffattn_selftest_exp2.restype = i32
    lib.diffattn_selftest_exp2.argtypes = [vp, vp, vp, i32, vp]
    lib.diffattn_debug_bounds_violations.restype = i32
    lib.diffattn_debug_bounds_violations.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    _lib = lib
    return lib


def _check(fn: str, rc: int):
    if rc != 0:
        raise DiffattnError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DIFFATTN_BF16
    if t.dtype == torch.float32:
        return DIFFATTN_F32
    raise DiffattnError("dtype", -2)


def diffattn_status_string(status: int) -> str:
    return load_library().diffattn_status_string(int(status)).decode()


def diffattn_lambda(lq1, lk1, lq2, lk2, depth: int, lambda_out=None, lambda_init_out=None,
                    stream=None):
    """lambda[h] = exp(lq1[h].lk1[h]) - exp(lq2[h].lk2[h]) + lambda_init(depth), on device.
    lq*, lk*: float32 CUDA tensors [n_heads, dim]. Returns (lambda_out, lambda_init_out)."""
    import torch
    lib = load_library()
    H, dim = lq1.shape
    if lambda_out is None:
        lambda_out = torch.empty(H, dtype=torch.float32, device=lq1.device)
    if lambda_init_out is None:
        lambda_init_out = torch.empty(1, dtype=torch.float32, device=lq1.device)
    for t in (lq1, lk1, lq2, lk2):
        if not t.is_contiguous():
            raise DiffattnError("diffattn_lambda", -1)
    rc = lib.diffattn_lambda(_ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), H, dim, int(depth),
                             _ptr(lambda_out), _ptr(lambda_init_out), _stream(stream))
    _check("diffattn_lambda", rc)
    return lambda_out, lambda_init_out


def prefill_params(q, k, v, out, causal=True, apply_norm=None, norm_eps=1e-5,
                   window=0) -> PrefillParams:
    """Build the prefill parameter struct from tensor shapes and strides.
    V1: q [B,N,H,2,d], k [B,Nk,H,2,d], v [B,Nk,H,2d], out [B,N,H,2d].
    V2: q [B,N,Hq,d], k,v [B,Nk,Hkv,d], out [B,N,Hq/2,d]. Nk >= N: the queries are the last
    N positions (chunked prefill)."""
    p = PrefillParams()
    if q.dim() == 5:
        B, N, H, two, d = q.shape
        p.variant, p.n_q_heads, p.n_kv_heads = DIFFATTN_V1, H, H
        if two != 2:
            raise DiffattnError("diffattn_fwd_prefill", -1)
        p.apply_norm = 1 if apply_norm is None else int(bool(apply_norm))
        qs, ks = q.stride(), k.stride()
        p.q_strides[:] = (qs[0], qs[1], qs[2])
        p.k_strides[:] = (ks[0], ks[1], ks[2])
        if qs[3] != d or ks[3] != d or qs[4] != 1 or ks[4] != 1:
            raise DiffattnError("diffattn_fwd_prefill", -1)
    elif q.dim() == 4:
        B, N, Hq, d = q.shape
        p.variant, p.n_q_heads, p.n_kv_heads = DIFFATTN_V2, Hq, k.shape[2]
        p.apply_norm = 0 if apply_norm is None else int(bool(apply_norm))
        p.q_strides[:] = q.stride()[:3]
        p.k_strides[:] = k.stride()[:3]
        if q.stride(3) != 1 or k.stride(3) != 1:
            raise DiffattnError("diffattn_fwd_prefill", -1)
    else:
        raise DiffattnError("diffattn_fwd_prefill", -1)
    if v.stride(-1) != 1 or out.stride(-1) != 1:
        raise DiffattnError("diffattn_fwd_prefill", -1)
    p.dtype = _dtype_code(q)
    p.batch, p.seqlen, p.head_dim = B, N, d
    p.causal = int(bool(causal))
    p.norm_eps = float(norm_eps)
    if k.shape[1] != v.shape[1]:
        raise DiffattnError("diffattn_fwd_prefill", -1)
    p.kv_seqlen = int(k.shape[1])
    p.window = int(window)
    p.v_strides[:] = v.stride()[:3]
    p.o_strides[:] = out.stride()[:3]
    return p


def diffattn_fwd_prefill(q, k, v, lam, lambda_init=None, out=None, causal=True, apply_norm=None,
                         norm_eps=1e-5, dev_status=None, stream=None, window=0):
    """Fused differential attention prefill (see include/diffattn.h for layouts). k and v
    may hold more positions than q (chunked prefill); window > 0 is a causal sliding window."""
    import torch
    lib = load_library()
    if out is None:
        if q.dim() == 5:
            B, N, H, _, d = q.shape
            out = torch.empty((B, N, H, 2 * d), dtype=q.dtype, device=q.device)
        else:
            B, N, Hq, d = q.shape
            out = torch.empty((B, N, Hq // 2, d), dtype=q.dtype, device=q.device)
    p = prefill_params(q, k, v, out, causal, apply_norm, norm_eps, window)
    rc = lib.diffattn_fwd_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                  _ptr(lambda_init), _ptr(out), _ptr(dev_status), _stream(stream))
    _check("diffattn_fwd_prefill", rc)
    return out


def diffattn_fwd_prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, lam,
                                lambda_init=None, out=None, causal=True, apply_norm=None,
                                norm_eps=1e-5, window=0, dev_status=None, stream=None):
    """Prefill over packed sequences of different lengths (see include/diffattn.h).
    V1: q [Tq,H,2,d], k [Tk,H,2,d], v [Tk,H,2d] -> out [Tq,H,2d]. V2: q [Tq,Hq,d],
    k,v [Tk,Hkv,d] -> out [Tq,Hq/2,d]. cu_seqlens_q / _k: int32 [S+1] device offsets;
    max_seqlen_q: the longest sequence's query count (host int)."""
    import torch
    lib = load_library()
    if out is None:
        if q.dim() == 4:
            T, H, _, d = q.shape
            out = torch.empty((T, H, 2 * d), dtype=q.dtype, device=q.device)
        else:
            T, Hq, d = q.shape
            out = torch.empty((T, Hq // 2, d), dtype=q.dtype, device=q.device)
    # the packed tensors viewed with a batch axis of one: the fixed-length struct applies
    p = prefill_params(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), out.unsqueeze(0), causal,
                       apply_norm, norm_eps, window)
    p.batch = int(cu_seqlens_q.numel()) - 1
    if p.batch < 0 or cu_seqlens_k.numel() != cu_seqlens_q.numel():
        raise DiffattnError("diffattn_fwd_prefill_varlen", -1)
    p.seqlen, p.kv_seqlen = int(q.shape[0]), int(k.shape[0])
    for st in (p.q_strides, p.k_strides, p.v_strides, p.o_strides):
        st[0] = 0
    rc = lib.diffattn_fwd_prefill_varlen(ctypes.byref(p), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                         int(max_seqlen_q), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                         _ptr(lambda_init), _ptr(out), _ptr(dev_status),
                                         _stream(stream))
    _check("diffattn_fwd_prefill_varlen", rc)
    return out


def diffattn_bwd_workspace_size(p: PrefillParams) -> int:
    n = ctypes.c_size_t(0)
    _check("diffattn_bwd_workspace_size",
           load_library().diffattn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return int(n.value)


def diffattn_bwd_prefill(q, k, v, lam, dout, lambda_init=None, causal=True, apply_norm=None,
                         norm_eps=1e-5, window=0, workspace=None, dev_status=None, stream=None,
                         grads=None):
    """Gradients of diffattn_fwd_prefill (see include/diffattn.h): dout has the forward
    output's layout and dtype. Returns float32 (dq, dk, dv, dlambda) in the shapes of q, k,
    v and lambda (written into `grads` when given: four dense float32 tensors)."""
    import torch
    lib = load_library()
    p = prefill_params(q, k, v, dout, causal, apply_norm, norm_eps, window)
    if grads is None:
        dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
        dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
        dl = torch.empty(lam.shape, dtype=torch.float32, device=q.device)
    else:
        dq, dk, dv, dl = grads
    need = diffattn_bwd_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.diffattn_bwd_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                  _ptr(lambda_init), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                  _ptr(dl), _ptr(workspace), ws_bytes, _ptr(dev_status),
                                  _stream(stream))
    _check("diffattn_bwd_prefill", rc)
    return dq, dk, dv, dl


def diffattn_fwd_prefill_train(q, k, v, lam, out=None, o2=None, lse=None, causal=True, window=0,
                               dev_status=None, stream=None):
    """diffattn_fwd_prefill for training (V2 bf16, d = 128; see include/diffattn.h): returns
    (out, o2, lse) -- the output, the branch-2 output O_2 / l_2 in out's layout, and float32
    [B, Hq/2, N, 2] log2-domain log-sum-exps of both branches."""
    import torch
    lib = load_library()
    B, N, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, N, Hq // 2, d), dtype=q.dtype, device=q.device)
    if o2 is None:
        o2 = torch.empty_like(out)
    if lse is None:
        lse = torch.empty((B, Hq // 2, N, 2), dtype=torch.float32, device=q.device)
    if o2.stride() != out.stride():
        raise ValueError("o2 must have out's layout")
    p = prefill_params(q, k, v, out, causal, None, 1e-5, window)
    rc = lib.diffattn_fwd_prefill_train(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out),
                                        _ptr(o2), _ptr(lse), _ptr(dev_status), _stream(stream))
    _check("diffattn_fwd_prefill_train", rc)
    return out, o2, lse


def diffattn_bwd_prefill_saved(q, k, v, lam, out, o2, lse, dout, causal=True, window=0,
                               workspace=None, dev_status=None, stream=None, grads=None):
    """diffattn_bwd_prefill from diffattn_fwd_prefill_train's (out, o2, lse) (see
    include/diffattn.h): no recompute of the forward. Returns float32 (dq, dk, dv, dlambda)."""
    import torch
    lib = load_library()
    if out.stride() != dout.stride() or o2.stride() != dout.stride():
        raise ValueError("out, o2 and dout must share one layout")
    p = prefill_params(q, k, v, dout, causal, None, 1e-5, window)
    if grads is None:
        grads = (torch.empty(q.shape, dtype=torch.float32, device=q.device),
                 torch.empty(k.shape, dtype=torch.float32, device=q.device),
                 torch.empty(v.shape, dtype=torch.float32, device=q.device),
                 torch.empty(lam.shape, dtype=torch.float32, device=q.device))
    dq, dk, dv, dl = grads
    need = diffattn_bwd_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.diffattn_bwd_prefill_saved(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out),
                                        _ptr(o2), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                        _ptr(dl), _ptr(workspace), ws_bytes, _ptr(dev_status),
                                        _stream(stream))
    _check("diffattn_bwd_prefill_saved", rc)
    return dq, dk, dv, dl


def diffattn_lambda_bwd(lq1, lk1, lq2, lk2, dlambda, stream=None):
    """Gradients of the four [n_heads, dim] lambda vectors from dL/dlambda [n_heads]."""
    import torch
    lib = load_library()
    H, dim = lq1.shape
    outs = [torch.empty((H, dim), dtype=torch.float32, device=lq1.device) for _ in range(4)]
    rc = lib.diffattn_lambda_bwd(_ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), H, dim, _ptr(dlambda),
                                 *[_ptr(o) for o in outs], _stream(stream))
    _check("diffattn_lambda_bwd", rc)
    return tuple(outs)


def decode_params(q, k_cache, v_cache, out, num_splits=0) -> DecodeParams:
    p = DecodeParams()
    B, Hq, d = q.shape
    _, L, Hkv, _ = k_cache.shape
    if tuple(k_cache.stride()) != tuple(v_cache.stride()):
        raise DiffattnError("diffattn_fwd_decode", -1)
    p.variant, p.dtype = DIFFATTN_V2, _dtype_code(q)
    p.batch, p.max_kv_len, p.n_q_heads, p.n_kv_heads, p.head_dim = B, L, Hq, Hkv, d
    p.num_splits = int(num_splits)
    p.q_strides[:] = q.stride()[:2]
    p.kv_strides[:] = k_cache.stride()[:3]
    p.o_strides[:] = out.stride()[:2]
    return p


def decode_params_v1(q, k_cache, v_cache, out, num_splits=0) -> DecodeParams:
    """V1: q [B,H,2,d], k_cache [B,L,H,2,d], v_cache [B,L,H,2d], out [B,H,2d]."""
    p = DecodeParams()
    B, H, two, d = q.shape
    _, L = k_cache.shape[:2]
    if two != 2 or tuple(k_cache.stride()[:3]) != tuple(v_cache.stride()[:3]):
        raise DiffattnError("diffattn_fwd_decode_v1", -1)
    p.variant, p.dtype = DIFFATTN_V1, _dtype_code(q)
    p.batch, p.max_kv_len, p.n_q_heads, p.n_kv_heads, p.head_dim = B, L, H, H, d
    p.num_splits = int(num_splits)
    p.q_strides[:] = q.stride()[:2]
    p.kv_strides[:] = k_cache.stride()[:3]
    p.o_strides[:] = out.stride()[:2]
    return p


def diffattn_decode_workspace_size(p: DecodeParams) -> int:
    n = ctypes.c_size_t(0)
    _check("diffattn_decode_workspace_size",
           load_library().diffattn_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return int(n.value)


def diffattn_fwd_decode(q, k_cache, v_cache, lam, kv_len=None, out=None, workspace=None,
                        num_splits=0, dev_status=None, stream=None):
    """Split-KV differential decode (V2). q [B,Hq,d], caches [B,L,Hkv,d] -> out [B,Hq/2,d]."""
    import torch
    lib = load_library()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq // 2, d), dtype=q.dtype, device=q.device)
    p = decode_params(q, k_cache, v_cache, out, num_splits)
    need = diffattn_decode_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.diffattn_fwd_decode(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(kv_len), _ptr(lam), _ptr(out), _ptr(workspace), ws_bytes,
                                 _ptr(dev_status), _stream(stream))
    _check("diffattn_fwd_decode", rc)
    return out


def diffattn_fwd_decode_v1(q, k_cache, v_cache, lam, lambda_init=None, kv_len=None, out=None,
                           apply_norm=True, norm_eps=1e-5, workspace=None, num_splits=0,
                           dev_status=None, stream=None):
    """Split-KV differential decode (V1). q [B,H,2,d], k_cache [B,L,H,2,d],
    v_cache [B,L,H,2d] -> out [B,H,2d], per-head RMSNorm and (1 - lambda_init) scale when
    apply_norm."""
    import torch
    lib = load_library()
    B, H, _, d = q.shape
    if out is None:
        out = torch.empty((B, H, 2 * d), dtype=q.dtype, device=q.device)
    p = decode_params_v1(q, k_cache, v_cache, out, num_splits)
    need = diffattn_decode_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.diffattn_fwd_decode_v1(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(kv_len), _ptr(lam), _ptr(lambda_init), int(bool(apply_norm)),
                                    float(norm_eps), _ptr(out), _ptr(workspace), ws_bytes,
                                    _ptr(dev_status), _stream(stream))
    _check("diffattn_fwd_decode_v1", rc)
    return out


class PagedKV(ctypes.Structure):
    _fields_ = [
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("page_strides", ctypes.c_int64 * 3),
    ]


def paged_kv(k_pages, v_pages, block_table) -> PagedKV:
    """Pool geometry from the page tensors ([P, page_size, heads, ...]) and the block table
    ([B, max_pages_per_seq])."""
    if tuple(k_pages.stride()[:3]) != tuple(v_pages.stride()[:3]) or k_pages.shape[:2] != v_pages.shape[:2]:
        raise DiffattnError("diffattn_fwd_decode_paged", -1)
    pk = PagedKV()
    pk.num_pages, pk.page_size = int(k_pages.shape[0]), int(k_pages.shape[1])
    pk.max_pages_per_seq = int(block_table.shape[1])
    pk.page_strides[:] = k_pages.stride()[:3]
    return pk


def diffattn_fwd_decode_paged(q, k_pages, v_pages, block_table, lam, kv_len=None, lambda_init=None,
                              out=None, apply_norm=None, norm_eps=1e-5, workspace=None,
                              num_splits=0, max_kv_len=None, dev_status=None, stream=None):
    """Split-KV differential decode over a paged cache (block table [B, max_pages_per_seq],
    int32). V2: q [B,Hq,d], pages [P,page,Hkv,d] -> out [B,Hq/2,d]. V1: q [B,H,2,d],
    k_pages [P,page,H,2,d], v_pages [P,page,H,2d] -> out [B,H,2d] (norm and scale when
    apply_norm, default on). max_kv_len defaults to page_size * max_pages_per_seq."""
    import torch
    lib = load_library()
    pk = paged_kv(k_pages, v_pages, block_table)
    p = DecodeParams()
    v1 = q.dim() == 4
    B = q.shape[0]
    if v1:
        _, H, two, d = q.shape
        if two != 2:
            raise DiffattnError("diffattn_fwd_decode_paged", -1)
        p.variant, p.n_q_heads, p.n_kv_heads = DIFFATTN_V1, H, H
        oshape = (B, H, 2 * d)
        norm = True if apply_norm is None else bool(apply_norm)
    else:
        _, Hq, d = q.shape
        p.variant, p.n_q_heads, p.n_kv_heads = DIFFATTN_V2, Hq, int(k_pages.shape[2])
        oshape = (B, Hq // 2, d)
        norm = False if apply_norm is None else bool(apply_norm)
    if out is None:
        out = torch.empty(oshape, dtype=q.dtype, device=q.device)
    p.dtype = _dtype_code(q)
    p.batch, p.head_dim, p.num_splits = B, d, int(num_splits)
    p.max_kv_len = int(max_kv_len if max_kv_len is not None else pk.page_size * pk.max_pages_per_seq)
    p.q_strides[:] = q.stride()[:2]
    p.o_strides[:] = out.stride()[:2]
    need = diffattn_decode_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.diffattn_fwd_decode_paged(ctypes.byref(p), ctypes.byref(pk), _ptr(q), _ptr(k_pages),
                                       _ptr(v_pages), _ptr(block_table), _ptr(kv_len), _ptr(lam),
                                       _ptr(lambda_init), int(norm), float(norm_eps), _ptr(out),
                                       _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check("diffattn_fwd_decode_paged", rc)
    return out


def diffattn_fwd_decode_static(q, k_cache, v_cache, lam, kv_len=None, out=None, num_splits=0,
                               dev_status=None, stream=None):
    """diffattn_fwd_decode with the partial states in the library's own device array, for
    callers that cannot allocate a workspace (see include/diffattn.h). Calls that overlap
    on the GPU share that array and must be ordered."""
    import torch
    lib = load_library()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq // 2, d), dtype=q.dtype, device=q.device)
    p = decode_params(q, k_cache, v_cache, out, num_splits)
    rc = lib.diffattn_fwd_decode_static(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(kv_len), _ptr(lam), _ptr(out), _ptr(dev_status),
                                        _stream(stream))
    _check("diffattn_fwd_decode_static", rc)
    return out


def diffattn_selftest_timeout(dev_status, timeout_ms=200, stream=None):
    """Launch the bounded-wait self-test (see include/diffattn.h): a wait that nothing
    completes runs out after `timeout_ms` and DIFFATTN_ERR_TIMEOUT lands in `dev_status`
    (a device int32 tensor) when the block finishes."""
    lib = load_library()
    rc = lib.diffattn_selftest_timeout(_ptr(dev_status), int(timeout_ms), _stream(stream))
    _check("diffattn_selftest_timeout", rc)


def diffattn_selftest_exp2(x, stream=None):
    """Evaluate the V2 prefill's FMA-pipe 2^x and CUDA's exp2f over a device float32 tensor
    `x` (see include/diffattn.h); returns (y, y_ref), device float32 tensors like x."""
    import torch
    lib = load_library()
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    y, y_ref = torch.empty_like(x), torch.empty_like(x)
    rc = lib.diffattn_selftest_exp2(_ptr(x), _ptr(y), _ptr(y_ref), int(x.numel()), _stream(stream))
    _check("diffattn_selftest_exp2", rc)
    return y, y_ref


def diffattn_debug_bounds_violations():
    """The bounds-checked build's count of skipped out-of-range accesses since the last call
    (see include/diffattn.h), or None when the loaded library is the normal build."""
    lib = load_library()
    n = ctypes.c_int32(0)
    rc = lib.diffattn_debug_bounds_violations(ctypes.byref(n))
    if rc == -2:  # DIFFATTN_ERR_UNSUPPORTED: the normal build
        return None
    _check("diffattn_debug_bounds_violations", rc)
    return int(n.value)

"""Gated MLA hot path for NVIDIA B200 (sm_100a): thin Python binding of libgmla.so.

Every function below marshals arguments for the C ABI of the same name
(include/gmla.h) and nothing else: all arithmetic runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing this module raises ImportError -- there is no fallback.

Layer (the "Gated MLA" problem page): C = X W_c^T, Q = X W_q^T, K = C W_k^T,
V = C W_v^T, per-head causal softmax attention, heads joined, gate
sigmoid(X W_g^T), output projection W_o^T.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "GmlaError", "lib", "library_path",
    "gmla_latent_project", "gmla_latent_project_heads",
    "gmla_expand_kv", "gmla_attend_prefill", "gmla_attend_prefill_varlen", "gmla_attend_prefill_varlen_workspace_size",
    "gmla_attend_decode", "gmla_attend_decode_workspace_size", "gmla_attend_decode_varlen",
    "gmla_attend_decode_varlen_workspace_size", "gmla_attend_decode_partial", "gmla_attend_decode_partial_workspace_size",
    "gmla_decode_combine", "gmla_attend_decode_noalloc", "gmla_attend_decode_noalloc_max_bytes",
    "gmla_gate_out", "gmla_gate_out_heads", "gmla_gate_out_workspace_size", "gmla_get_device_status",
    "gmla_selftest_wait_timeout", "gmla_status_string",
    "gmla_version", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libgmla.so")

STATUS = {0: "GMLA_OK", 1: "GMLA_ERR_ARG", 2: "GMLA_ERR_UNSUPPORTED", 3: "GMLA_ERR_CUDA",
          4: "GMLA_ERR_TIMEOUT", 5: "GMLA_ERR_WORKSPACE"}

if not os.path.exists(library_path):
    raise ImportError(f"libgmla.so not built ({library_path}); run `python causal_head_latent_b200/build.py`")

lib = ctypes.CDLL(library_path)

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_st = ctypes.c_int
_i64x3 = ctypes.c_int64 * 3

lib.gmla_latent_project.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _i64, _i64,
                                    _p, _p, _p]
lib.gmla_latent_project.restype = _st
lib.gmla_latent_project_heads.argtypes = [_p, _i64, _i64, _i64, _i64, _i64, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _i64,
                                          _i64, _p, _p, _p]
lib.gmla_latent_project_heads.restype = _st
lib.gmla_expand_kv.argtypes = [_p, _i64, _i64, _i64, _i64, _i64, _p, _p, _i64, _p, _p, _p]
lib.gmla_expand_kv.restype = _st
lib.gmla_attend_prefill.argtypes = [_p, _i64x3, _p, _i64x3, _p, _i64x3, _i64, _i64, _i64, _i64, _i64,
                                    ctypes.c_int, ctypes.c_float, _p, _p, _i64x3, _p, _p, _p]
lib.gmla_attend_prefill.restype = _st
lib.gmla_attend_prefill_varlen.argtypes = [_p, _i64x3, _p, _i64x3, _p, _i64x3, _i64, _i64, _i64, _i64, _i64, _p, _p,
                                           ctypes.c_int, ctypes.c_float, _p, _p, _i64x3, _p, _p, _sz, _p]
lib.gmla_attend_prefill_varlen.restype = _st
lib.gmla_attend_prefill_varlen_workspace_size.argtypes = [_i64]
lib.gmla_attend_prefill_varlen_workspace_size.restype = _sz
lib.gmla_attend_decode.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _p, ctypes.c_float, _p, _p, _p,
                                   _p, _sz, _p]
lib.gmla_attend_decode.restype = _st
lib.gmla_attend_decode_workspace_size.argtypes = [_i64, _i64, _i64, _i64]
lib.gmla_attend_decode_workspace_size.restype = _sz
lib.gmla_attend_decode_varlen.argtypes = [_p, _p, _i64, _i64, _p, _i64, _i64, _i64, _p, _p, ctypes.c_float, _p, _p,
                                          _p, _p, _sz, _p]
lib.gmla_attend_decode_varlen.restype = _st
lib.gmla_attend_decode_varlen_workspace_size.argtypes = [_i64, _i64, _i64, _i64]
lib.gmla_attend_decode_varlen_workspace_size.restype = _sz
lib.gmla_attend_decode_partial.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _p, ctypes.c_float, _p,
                                           _p, _p, _sz, _p]
lib.gmla_attend_decode_partial.restype = _st
lib.gmla_attend_decode_partial_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64]
lib.gmla_attend_decode_partial_workspace_size.restype = _sz
lib.gmla_decode_combine.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _p, _p, _p, _p]
lib.gmla_decode_combine.restype = _st
lib.gmla_attend_decode_noalloc.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _p, ctypes.c_float, _p,
                                           _p, _p, _p]
lib.gmla_attend_decode_noalloc.restype = _st
lib.gmla_attend_decode_noalloc_max_bytes.argtypes = []
lib.gmla_attend_decode_noalloc_max_bytes.restype = _sz
lib.gmla_gate_out.argtypes = [_p, _p, _p, _i64, _i64, _p, _p, _sz, _p]
lib.gmla_gate_out.restype = _st
lib.gmla_gate_out_heads.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _sz, _p]
lib.gmla_gate_out_heads.restype = _st
lib.gmla_gate_out_workspace_size.argtypes = [_i64, _i64]
lib.gmla_gate_out_workspace_size.restype = _sz
lib.gmla_get_device_status.argtypes = [_p]
lib.gmla_get_device_status.restype = _st
lib.gmla_selftest_wait_timeout.argtypes = [ctypes.c_uint, _p]
lib.gmla_selftest_wait_timeout.restype = _st
lib.gmla_status_string.argtypes = [_st]
lib.gmla_status_string.restype = ctypes.c_char_p
lib.gmla_version.argtypes = []
lib.gmla_version.restype = ctypes.c_int


class GmlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({gmla_status_string(code)})")


def _check(code: int, where: str) -> int:
    if code != 0:
        raise GmlaError(code, where)
    return code


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    return t.data_ptr()


def _bf16(t, name):
    if t is not None and t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    return t


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(workspace):
    if workspace is None:
        return None, 0
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def gmla_status_string(code: int) -> str:
    return lib.gmla_status_string(code).decode()


def gmla_version() -> int:
    return lib.gmla_version()


def gmla_get_device_status(stream=None, raise_on_error: bool = True) -> int:
    code = lib.gmla_get_device_status(_stream(stream))
    return _check(code, "gmla_get_device_status") if raise_on_error else code


def gmla_selftest_wait_timeout(milliseconds: int = 20, stream=None) -> int:
    """Launch a kernel whose bounded wait runs out (see include/gmla.h); returns the launch status."""
    return _check(lib.gmla_selftest_wait_timeout(int(milliseconds), _stream(stream)), "gmla_selftest_wait_timeout")


def gmla_latent_project(X, W_q, W_g, W_c, W_k, W_v, Q=None, G=None, C=None, cache_len_max=None, cache_pos=0,
                        K=None, V=None, stream=None, check=True):
    """X [B, T, d_model]; C [B, cache_len_max, d_c] (rows cache_pos..cache_pos+T-1 written)."""
    for n, t in (("X", X), ("W_q", W_q), ("W_g", W_g), ("W_c", W_c), ("W_k", W_k), ("W_v", W_v),
                 ("Q", Q), ("G", G), ("C", C), ("K", K), ("V", V)):
        _bf16(t, n)
    B, T, d = X.shape
    d_c = W_c.shape[0] if W_c is not None else (C.shape[-1] if C is not None else 0)
    if cache_len_max is None:
        cache_len_max = C.shape[1] if C is not None else T
    code = lib.gmla_latent_project(_ptr(X), B, T, d, _ptr(W_q), _ptr(W_g), _ptr(W_c), d_c, _ptr(W_k), _ptr(W_v),
                                   _ptr(Q), _ptr(G), _ptr(C), cache_len_max, cache_pos, _ptr(K), _ptr(V),
                                   _stream(stream))
    return _check(code, "gmla_latent_project") if check else code


def gmla_latent_project_heads(X, head_begin, head_end, W_q, W_g, W_c, W_k, W_v, Q=None, G=None, C=None,
                              cache_len_max=None, cache_pos=0, K=None, V=None, stream=None, check=True):
    """Projections of heads [head_begin, head_end) only: full weights in, Q, G, K, V
    [B, T, 128*(head_end-head_begin)] out; C (full latent) as gmla_latent_project."""
    for n, t in (("X", X), ("W_q", W_q), ("W_g", W_g), ("W_c", W_c), ("W_k", W_k), ("W_v", W_v),
                 ("Q", Q), ("G", G), ("C", C), ("K", K), ("V", V)):
        _bf16(t, n)
    B, T, d = X.shape
    d_c = W_c.shape[0] if W_c is not None else (C.shape[-1] if C is not None else 0)
    if cache_len_max is None:
        cache_len_max = C.shape[1] if C is not None else T
    code = lib.gmla_latent_project_heads(_ptr(X), B, T, d, int(head_begin), int(head_end), _ptr(W_q), _ptr(W_g),
                                         _ptr(W_c), d_c, _ptr(W_k), _ptr(W_v), _ptr(Q), _ptr(G), _ptr(C),
                                         cache_len_max, cache_pos, _ptr(K), _ptr(V), _stream(stream))
    return _check(code, "gmla_latent_project_heads") if check else code


def gmla_expand_kv(C, row0, rows, W_k=None, W_v=None, K=None, V=None, stream=None, check=True):
    """K, V [B, rows, d_model] = C[:, row0:row0+rows] [W_k; W_v]^T; C [B, cache_len_max, d_c]."""
    for n, t in (("C", C), ("W_k", W_k), ("W_v", W_v), ("K", K), ("V", V)):
        _bf16(t, n)
    B, Lmax, d_c = C.shape
    d_model = (W_k if W_k is not None else W_v).shape[0]
    code = lib.gmla_expand_kv(_ptr(C), B, Lmax, int(row0), int(rows), d_c, _ptr(W_k), _ptr(W_v), d_model, _ptr(K),
                              _ptr(V), _stream(stream))
    return _check(code, "gmla_expand_kv") if check else code


def _bthd_strides(t, layout):
    """(batch, token, head) element strides of a 4-D tensor in layout 'bthd' or 'bhtd'."""
    if t.stride(-1) != 1:
        raise ValueError("head dimension must be contiguous")
    s = t.stride()
    return _i64x3(s[0], s[1], s[2]) if layout == "bthd" else _i64x3(s[0], s[2], s[1])


def gmla_attend_prefill(Q, K, V, O, causal=True, scale=0.0, G=None, lse=None, weights=None, layout="bthd",
                        stream=None, check=True):
    """Q, O [B,Tq,H,D] (or [B,H,Tq,D] with layout='bhtd'); K, V [B,Tk,H,D]; G [B,Tq,H*D] or None."""
    for n, t in (("Q", Q), ("K", K), ("V", V), ("O", O), ("G", G)):
        _bf16(t, n)
    if layout == "bthd":
        B, Tq, H, D = Q.shape
        Tk = K.shape[1]
    else:
        B, H, Tq, D = Q.shape
        Tk = K.shape[2]
    if lse is not None and lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    if weights is not None and weights.dtype != torch.float32:
        raise TypeError("weights must be float32")
    code = lib.gmla_attend_prefill(_ptr(Q), _bthd_strides(Q, layout), _ptr(K), _bthd_strides(K, layout), _ptr(V),
                                   _bthd_strides(V, layout), B, H, Tq, Tk, D, int(bool(causal)), float(scale),
                                   _ptr(G), _ptr(O), _bthd_strides(O, layout), _ptr(lse), _ptr(weights),
                                   _stream(stream))
    return _check(code, "gmla_attend_prefill") if check else code


def gmla_attend_prefill_varlen_workspace_size(B) -> int:
    return lib.gmla_attend_prefill_varlen_workspace_size(B)


def gmla_attend_prefill_varlen(Q, K, V, O, q_lens, kv_lens, causal=True, scale=0.0, G=None, lse=None, workspace=None,
                               layout="bthd", stream=None, check=True):
    """Padded batch: Q, O [B,Tq_max,H,D] (or [B,H,Tq_max,D] with layout='bhtd'); K, V [B,Tk_max,H,D];
    q_lens, kv_lens: B host integers each (see include/gmla.h)."""
    for n, t in (("Q", Q), ("K", K), ("V", V), ("O", O), ("G", G)):
        _bf16(t, n)
    if layout == "bthd":
        B, Tq, H, D = Q.shape
        Tk = K.shape[1]
    else:
        B, H, Tq, D = Q.shape
        Tk = K.shape[2]
    if len(q_lens) != B or len(kv_lens) != B:
        raise ValueError("q_lens and kv_lens need one length per sequence")
    if lse is not None and lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    ql = (ctypes.c_int64 * B)(*[int(x) for x in q_lens])
    kl = (ctypes.c_int64 * B)(*[int(x) for x in kv_lens])
    wp, wb = _ws(workspace)
    code = lib.gmla_attend_prefill_varlen(_ptr(Q), _bthd_strides(Q, layout), _ptr(K), _bthd_strides(K, layout),
                                          _ptr(V), _bthd_strides(V, layout), B, H, Tq, Tk, D, ctypes.cast(ql, _p),
                                          ctypes.cast(kl, _p), int(bool(causal)), float(scale), _ptr(G), _ptr(O),
                                          _bthd_strides(O, layout), _ptr(lse), wp, wb, _stream(stream))
    return _check(code, "gmla_attend_prefill_varlen") if check else code


def gmla_attend_decode_workspace_size(B, L, H, d_c) -> int:
    return lib.gmla_attend_decode_workspace_size(B, L, H, d_c)


def gmla_attend_decode(Q, C, L, W_k, W_v, O, num_heads, scale=0.0, G=None, weights=None, workspace=None,
                       stream=None, check=True):
    """Q, O, G [B, H*D]; C [B, cache_len_max, d_c]; rows 0..L-1 visible."""
    for n, t in (("Q", Q), ("C", C), ("W_k", W_k), ("W_v", W_v), ("O", O), ("G", G)):
        _bf16(t, n)
    B, d = Q.shape
    H = int(num_heads)
    D = d // H
    _, Lmax, d_c = C.shape
    wp, wb = _ws(workspace)
    code = lib.gmla_attend_decode(_ptr(Q), _ptr(C), B, Lmax, L, H, D, d_c, _ptr(W_k), _ptr(W_v), float(scale),
                                  _ptr(G), _ptr(O), _ptr(weights), wp, wb, _stream(stream))
    return _check(code, "gmla_attend_decode") if check else code


def gmla_attend_decode_varlen_workspace_size(B, cache_len_max, H, d_c) -> int:
    return lib.gmla_attend_decode_varlen_workspace_size(B, cache_len_max, H, d_c)


def gmla_attend_decode_varlen(Q, C, lens, W_k, W_v, O, num_heads, scale=0.0, G=None, weights=None, workspace=None,
                              stream=None, check=True):
    """Q, O, G [B, H*D]; C [B, cache_len_max, d_c]; lens: B host integers, sequence b
    sees cache rows 0..lens[b]-1 (see include/gmla.h)."""
    for n, t in (("Q", Q), ("C", C), ("W_k", W_k), ("W_v", W_v), ("O", O), ("G", G)):
        _bf16(t, n)
    B, d = Q.shape
    H = int(num_heads)
    D = d // H
    _, Lmax, d_c = C.shape
    if len(lens) != B:
        raise ValueError("lens needs one length per sequence")
    lens_arr = (ctypes.c_int64 * B)(*[int(x) for x in lens])
    wp, wb = _ws(workspace)
    code = lib.gmla_attend_decode_varlen(_ptr(Q), _ptr(C), B, Lmax, ctypes.cast(lens_arr, _p), H, D, d_c, _ptr(W_k),
                                         _ptr(W_v), float(scale), _ptr(G), _ptr(O), _ptr(weights), wp, wb,
                                         _stream(stream))
    return _check(code, "gmla_attend_decode_varlen") if check else code


def gmla_attend_decode_noalloc_max_bytes() -> int:
    return lib.gmla_attend_decode_noalloc_max_bytes()


def gmla_attend_decode_noalloc(Q, C, L, W_k, W_v, O, num_heads, scale=0.0, G=None, weights=None, stream=None,
                               check=True):
    """gmla_attend_decode without a workspace, for callers that cannot allocate device
    memory at decode time; the scratch is a fixed array inside the library (see
    include/gmla.h).  Calls that overlap on the GPU share that array and race."""
    for n, t in (("Q", Q), ("C", C), ("W_k", W_k), ("W_v", W_v), ("O", O), ("G", G)):
        _bf16(t, n)
    B, d = Q.shape
    H = int(num_heads)
    D = d // H
    _, Lmax, d_c = C.shape
    code = lib.gmla_attend_decode_noalloc(_ptr(Q), _ptr(C), B, Lmax, L, H, D, d_c, _ptr(W_k), _ptr(W_v),
                                          float(scale), _ptr(G), _ptr(O), _ptr(weights), _stream(stream))
    return _check(code, "gmla_attend_decode_noalloc") if check else code


def gmla_attend_decode_partial_workspace_size(B, k0, k1, H, d_c) -> int:
    return lib.gmla_attend_decode_partial_workspace_size(B, k0, k1, H, d_c)


def gmla_attend_decode_partial(Q, C, k0, k1, W_k, lse, ctx, num_heads, scale=0.0, workspace=None, stream=None,
                               check=True):
    """Softmax state over cached rows [k0, k1): Q [B, H*D]; C [B, cache_len_max, d_c];
    lse float32 [B, H] and ctx float32 [B, H, d_c] outputs (see include/gmla.h)."""
    for n, t in (("Q", Q), ("C", C), ("W_k", W_k)):
        _bf16(t, n)
    for n, t in (("lse", lse), ("ctx", ctx)):
        if t.dtype != torch.float32:
            raise TypeError(f"{n} must be float32")
    B, d = Q.shape
    H = int(num_heads)
    D = d // H
    _, Lmax, d_c = C.shape
    wp, wb = _ws(workspace)
    code = lib.gmla_attend_decode_partial(_ptr(Q), _ptr(C), B, Lmax, int(k0), int(k1), H, D, d_c, _ptr(W_k),
                                          float(scale), _ptr(lse), _ptr(ctx), wp, wb, _stream(stream))
    return _check(code, "gmla_attend_decode_partial") if check else code


def gmla_decode_combine(lse, ctx, W_v, O, G=None, stream=None, check=True):
    """Merge stacked decode states lse [n, B, H], ctx [n, B, H, d_c] (float32) into
    O [B, H*D] = gate(W_v^(h) c^) (see include/gmla.h)."""
    for n, t in (("W_v", W_v), ("O", O), ("G", G)):
        _bf16(t, n)
    for n, t in (("lse", lse), ("ctx", ctx)):
        if t.dtype != torch.float32:
            raise TypeError(f"{n} must be float32")
    n_parts, B, H, d_c = ctx.shape
    D = O.shape[-1] // H
    code = lib.gmla_decode_combine(_ptr(lse), _ptr(ctx), n_parts, B, H, D, d_c, _ptr(W_v), _ptr(G), _ptr(O),
                                   _stream(stream))
    return _check(code, "gmla_decode_combine") if check else code


def gmla_gate_out_workspace_size(M, d_model) -> int:
    return lib.gmla_gate_out_workspace_size(M, d_model)


def gmla_gate_out(O, W_o, Y, G=None, workspace=None, stream=None, check=True):
    """Y = (sigmoid(G) (.) O) W_o^T; O, G, Y [M, d_model] (any leading shape flattened);
    W_o [d_model, d_model]; a workspace is needed only with G."""
    for n, t in (("O", O), ("W_o", W_o), ("Y", Y), ("G", G)):
        _bf16(t, n)
    d = O.shape[-1]
    M = O.numel() // d
    wp, wb = _ws(workspace)
    code = lib.gmla_gate_out(_ptr(O), _ptr(G), _ptr(W_o), M, d, _ptr(Y), wp, wb, _stream(stream))
    return _check(code, "gmla_gate_out") if check else code


def gmla_gate_out_heads(O, W_o, Y, head_begin, head_end, G=None, workspace=None, stream=None, check=True):
    """Share of heads [head_begin, head_end) in Y: O, G [M, 128*(head_end-head_begin)];
    W_o the full [d_model, d_model]; Y [M, d_model]."""
    for n, t in (("O", O), ("W_o", W_o), ("Y", Y), ("G", G)):
        _bf16(t, n)
    w = O.shape[-1]
    M = O.numel() // w
    d = W_o.shape[0]
    wp, wb = _ws(workspace)
    code = lib.gmla_gate_out_heads(_ptr(O), _ptr(G), _ptr(W_o), M, d, int(head_begin), int(head_end), _ptr(Y), wp,
                                   wb, _stream(stream))
    return _check(code, "gmla_gate_out_heads") if check else code

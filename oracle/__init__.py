"""Gated MLA oracle: a plain, slow float64 CPU implementation.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and
bench.py's CPU-baseline leg import this package.  It shares no code with the
CUDA path (``causal_head_latent_b200``) and never imports it; the two meet only
through the seeded inputs of ``synth_inputs``.

The arithmetic lives in ``gmla_oracle.c`` (one function per step of the
method, plain loops, float64).  This module marshals numpy arrays and composes
the steps in the order of the "Gated MLA" problem page, section
"Implementation order":

1. project the hidden states into queries and latents: Q = X W_q^T, C = X W_c^T;
2. expand the latents: K = C W_k^T, V = C W_v^T;
3. split Q, K, V into H heads of width D_h = d_model / H (head h owns
   channels [h*D_h, (h+1)*D_h));
4. per head, scaled scores, the causal mask when requested, softmax over keys;
5. combine the values and join the heads back to model width (concatenation);
6. gate with sigmoid(X W_g^T) channel by channel, then apply W_o^T;
7. return the output and the latent cache C.

Decode (one new query over a latent cache) uses the same definition, not the
absorbed form: it rebuilds K and V of the requested heads from the cache.

Every function here is pinned by tests/test_oracle_pins.py against facts the
pages and the mathematics fix (worked examples, closed forms, invariants,
an independent dense numpy formulation on tiny shapes).
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None
LAYER_MUTATION = None  # test-only: "gate_after_wo", "wo_untransposed", "heads_summed"


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_long)
        L.orc_linear.argtypes = [dp, ctypes.c_long, ctypes.c_long, ctypes.c_long, dp, ctypes.c_long,
                                 dp, ctypes.c_long, lp, ctypes.c_long]
        L.orc_attention.argtypes = [dp, lp, dp, lp, dp, lp, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                    ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_double,
                                    dp, lp, dp, dp, lp, ctypes.c_long]
        L.orc_gate.argtypes = [dp, dp, ctypes.c_long, dp]
        L.orc_round_bf16.argtypes = [dp, ctypes.c_long, dp]
        L.orc_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().orc_num_threads())


@contextlib.contextmanager
def mutation(code):
    """Test-only: switch in a deliberate mistake (see gmla_oracle.c / LAYER_MUTATION)."""
    global LAYER_MUTATION
    mut = ctypes.c_int.in_dll(lib(), "orc_mutation")
    old_c, old_py = mut.value, LAYER_MUTATION
    if isinstance(code, int):
        mut.value = code
    else:
        LAYER_MUTATION = code
    try:
        yield
    finally:
        mut.value = old_c
        LAYER_MUTATION = old_py


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _lp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_long))


def widen(x) -> np.ndarray:
    """float64 view of an input: bfloat16 bit patterns (uint16) are widened exactly;
    float arrays are converted."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float64)


def round_bf16(x) -> np.ndarray:
    """bfloat16 round-to-nearest-even of float64 values, returned as float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().orc_round_bf16(_dp(x), x.size, _dp(out))
    return out


def linear(X, W, rows=None) -> np.ndarray:
    """Y = X W^T over the last axis of X (nn.Linear orientation, W: [N, K]).
    rows: optional flat row indices of X (as [M, K]) to compute; other rows are NaN."""
    X = widen(X)
    W = widen(W)
    K = X.shape[-1]
    N = W.shape[0]
    assert W.shape[1] == K
    X2 = np.ascontiguousarray(X.reshape(-1, K))
    M = X2.shape[0]
    Y = np.full((M, N), np.nan) if rows is not None else np.empty((M, N))
    if rows is None:
        lib().orc_linear(_dp(X2), K, M, K, _dp(W), N, _dp(Y), N, None, 0)
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        lib().orc_linear(_dp(X2), K, M, K, _dp(W), N, _dp(Y), N, _lp(r), r.size)
    return Y.reshape(X.shape[:-1] + (N,))


def attention(Q, K, V, causal=True, scale=None, layout="bthd", want_weights=False, want_lse=False, rows=None):
    """Per-head softmax attention.

    layout "bthd": Q [B,Tq,H,D], K/V [B,Tk,H,D] (heads split from model width);
    layout "bhtd": Q [B,H,Tq,D], K/V [B,H,Tk,D] (the softmax page's layout).
    Query t sits at absolute position Tk - Tq + t.  scale defaults to 1/sqrt(D).
    rows: optional list of (b, h, t) triples to compute (others stay NaN).
    Returns O in the layout of Q, and optionally weights [B,H,Tq,Tk] and lse [B,H,Tq].
    """
    Q, K, V = widen(Q), widen(K), widen(V)
    if layout == "bthd":
        B, Tq, H, D = Q.shape
        Tk = K.shape[1]
        st = lambda a: np.array([a.strides[0], a.strides[1], a.strides[2]], dtype=np.int64) // 8
    elif layout == "bhtd":
        B, H, Tq, D = Q.shape
        Tk = K.shape[2]
        st = lambda a: np.array([a.strides[0], a.strides[2], a.strides[1]], dtype=np.int64) // 8
    else:
        raise ValueError(layout)
    assert K.shape == V.shape and Tq <= Tk and Tk >= 1
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    O = np.full(Q.shape, np.nan) if rows is not None else np.empty(Q.shape)
    Wt = np.zeros((B, H, Tq, Tk)) if want_weights else None
    lse = np.full((B, H, Tq), np.nan) if want_lse else None
    qs, ks, vs, os_ = st(Q), st(K), st(V), st(O)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    lib().orc_attention(_dp(Q), _lp(qs), _dp(K), _lp(ks), _dp(V), _lp(vs), B, H, Tq, Tk, D,
                        int(bool(causal)), float(scale), _dp(O), _lp(os_),
                        _dp(Wt) if want_weights else None, _dp(lse) if want_lse else None,
                        None if r is None else _lp(r), 0 if r is None else r.size // 3)
    out = [O]
    if want_weights:
        out.append(Wt)
    if want_lse:
        out.append(lse)
    return out[0] if len(out) == 1 else tuple(out)


def gate(O, G) -> np.ndarray:
    """sigmoid(G) (.) O, element by element ("Gated MLA", the channel-wise output gate)."""
    O = widen(O)
    G = widen(G)
    assert O.shape == G.shape
    out = np.empty_like(O)
    lib().orc_gate(_dp(np.ascontiguousarray(O)), _dp(np.ascontiguousarray(G)), O.size, _dp(out))
    return out


def gated_mla(X, W_q, W_c, W_k, W_v, W_g, W_o, num_heads, causal=True, round_boundaries=False,
              intermediates=False):
    """The page's ``gated_mla`` (starter signature of the "Gated MLA" problem page):
    returns {"output": Y, "latent_cache": C} with Y shaped like X and C [B, T, d_c].

    round_boundaries=True rounds Q, G, C, K, V and the gated context to
    bfloat16 where the library stores them as bfloat16 (for chained checks)."""
    X = widen(X)
    B, T, d = X.shape
    H = int(num_heads)
    if H <= 0 or d % H != 0:
        raise ValueError("model width must be divisible by the positive head count")
    D = d // H
    rb = round_bf16 if round_boundaries else (lambda a: a)
    Q = rb(linear(X, W_q))                      # step 1
    C = rb(linear(X, W_c))
    K = rb(linear(C, W_k))                      # step 2
    V = rb(linear(C, W_v))
    Qh = Q.reshape(B, T, H, D)                  # step 3
    Kh = K.reshape(B, T, H, D)
    Vh = V.reshape(B, T, H, D)
    Oh = attention(Qh, Kh, Vh, causal=causal)   # step 4
    if LAYER_MUTATION == "heads_summed":        # test-only mistake: sum heads instead of joining
        Ot = np.repeat(Oh.sum(axis=2, keepdims=True), H, axis=2).reshape(B, T, d)
    else:
        Ot = Oh.reshape(B, T, d)                # step 5: concatenate heads
    G = rb(linear(X, W_g))                      # step 6
    if LAYER_MUTATION == "gate_after_wo":
        Og = Ot
        Y = gate(linear(Og, W_o), G)
    elif LAYER_MUTATION == "wo_untransposed":
        Og = rb(gate(Ot, G))
        Y = Og @ widen(W_o)
    else:
        Og = rb(gate(Ot, G))
        Y = linear(Og, W_o)
    res = {"output": Y, "latent_cache": C}      # step 7
    if intermediates:
        res.update(Q=Q, C=C, K=K, V=V, G=G, O=Ot, O_gated=Og)
    return res


def decode_latent(q, cache, L, W_k, W_v, num_heads, G=None, scale=None, heads=None, want_weights=False):
    """One new query per sequence over a latent cache, by the plain definition.

    q: [B, d_model] queries; cache: [B, L_max, d_c] latents of which rows
    0..L-1 are visible (the new token's own latent included, at row L-1);
    heads: optional list of (b, h) pairs to compute (default: all).
    For each requested (b, h), K_h = C_b[:L] W_k^(h)T and V_h = C_b[:L] W_v^(h)T
    are rebuilt from the cache (W^(h) = rows h*D..h*D+D-1), then the query at
    position L-1 attends to all L keys.  Returns the per-head context [B, d]
    (NaN where not computed), gated by sigmoid(G) when G is given, and
    optionally the weights [B, H, L] (zeros where not computed)."""
    qd = widen(q)
    B, d = qd.shape
    H = int(num_heads)
    D = d // H
    Wk = widen(W_k)
    Wv = widen(W_v)
    out = np.full((B, d), np.nan)
    wts = np.zeros((B, H, L)) if want_weights else None
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    wide = {}  # sequences widened to float64 on first use (the cache can be many GB)
    for b, h in pairs:
        if b not in wide:
            wide[b] = widen(np.ascontiguousarray(cache[b, :L]))
        Cb = wide[b]
        Kh = linear(Cb, Wk[h * D:(h + 1) * D])          # [L, D]
        Vh = linear(Cb, Wv[h * D:(h + 1) * D])
        qh = qd[b, h * D:(h + 1) * D].reshape(1, 1, 1, D)
        res = attention(qh, Kh.reshape(1, L, 1, D), Vh.reshape(1, L, 1, D), causal=True, scale=scale,
                        want_weights=want_weights)
        if want_weights:
            o, w = res
            wts[b, h] = w[0, 0, 0]
        else:
            o = res
        out[b, h * D:(h + 1) * D] = o.reshape(D)
    if G is not None:
        Gw = widen(G)
        m = ~np.isnan(out)
        gated = np.full_like(out, np.nan)
        gated[m] = gate(out[m], Gw[m])
        out = gated
    return (out, wts) if want_weights else out

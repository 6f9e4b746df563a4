"""Decode without a caller workspace (gmla_attend_decode_noalloc).

This entry point serves callers that cannot allocate device memory when they
decode -- for instance a runtime that reserved all device memory for its own
pool -- by keeping the decode scratch in a fixed array inside the library.
Its result must match gmla_attend_decode (which takes a caller workspace)
within the parity tolerance, on consecutive calls that reuse the shared array,
and oversized problems must be refused before anything is launched.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import Draw
from tests.gpu_util import ROW_SUM, assert_parity, f64, to_dev

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Lmax, H, d_c):
    d = 128 * H
    dr = Draw(seed)
    return {"q": dr.normal((B, d)), "cache": dr.normal((B, Lmax, d_c)),
            "Wk": dr.normal((d, d_c), 1 / np.sqrt(d_c)), "Wv": dr.normal((d, d_c), 1 / np.sqrt(d_c)),
            "G": dr.normal((B, d))}


def test_noalloc_decode_matches_workspace_decode_on_consecutive_calls():
    import causal_head_latent_b200 as g
    assert g.gmla_attend_decode_noalloc_max_bytes() == 32 << 20
    cases = [(700, 4, 2049, 3000, 96, 512), (701, 32, 40000, 40000, 96, 512)]
    for seed, B, L, Lmax, H, d_c in cases:   # two calls in a row share the library's scratch array
        x = _inputs(seed, B, Lmax, H, d_c)
        Q, C, Wk, Wv, G = (to_dev(x[k]) for k in ("q", "cache", "Wk", "Wv", "G"))
        d = 128 * H
        ref = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(g.gmla_attend_decode_workspace_size(B, L, H, d_c), dtype=torch.uint8, device="cuda")
        g.gmla_attend_decode(Q, C, L, Wk, Wv, ref, H, G=G, workspace=ws)
        out = torch.full((B, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        g.gmla_attend_decode_noalloc(Q, C, L, Wk, Wv, out, H, G=G)
        g.gmla_get_device_status()
        assert_parity(f64(out), f64(ref), f"no-alloc vs workspace decode, B={B} L={L}")
        # the no-alloc call may split the keys differently, so it is also held to the
        # oracle's plain decode (K and V rebuilt from the cache) on sampled heads
        pairs = [(0, 0), (B - 1, H - 1), (B // 2, 17)]
        oref = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"], heads=pairs)
        sel = np.concatenate([np.arange(h * 128, (h + 1) * 128) + b * d for b, h in pairs])
        assert_parity(f64(out).reshape(-1)[sel], oref.reshape(-1)[sel], f"no-alloc vs oracle, B={B} L={L}")


def test_noalloc_decode_debug_weights():
    """The debug softmax weights of the no-alloc call (normalised through the
    log-sum-exp kept in the shared scratch): rows sum to one and match the
    oracle's weights."""
    import causal_head_latent_b200 as g
    B, L, Lmax, H, d_c = 2, 777, 800, 4, 512
    x = _inputs(702, B, Lmax, H, d_c)
    Q, C, Wk, Wv, G = (to_dev(x[k]) for k in ("q", "cache", "Wk", "Wv", "G"))
    out = torch.empty(B, 128 * H, dtype=torch.bfloat16, device="cuda")
    W = torch.full((B, H, L), float("nan"), device="cuda")
    g.gmla_attend_decode_noalloc(Q, C, L, Wk, Wv, out, H, G=G, weights=W)
    g.gmla_get_device_status()
    w = f64(W)
    assert np.abs(w.sum(-1) - 1.0).max() <= ROW_SUM
    ref, wref = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"], want_weights=True)
    assert_parity(f64(out), ref, "no-alloc decode with weights")
    assert np.all(np.abs(w - wref) <= 2e-5 + 1e-2 * wref)


def test_noalloc_decode_refuses_problems_beyond_its_scratch():
    import causal_head_latent_b200 as g
    B, L, H, d_c = 128, 64, 96, 512   # one split needs about 37 MiB of scratch
    d = 128 * H
    Q = torch.zeros(B, d, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(B, L, d_c, dtype=torch.bfloat16, device="cuda")
    Wk = torch.zeros(d, d_c, dtype=torch.bfloat16, device="cuda")
    Wv = torch.zeros_like(Wk)
    O = torch.zeros(B, d, dtype=torch.bfloat16, device="cuda")
    code = g.gmla_attend_decode_noalloc(Q, C, L, Wk, Wv, O, H, check=False)
    assert g.STATUS[code] == "GMLA_ERR_WORKSPACE"
    g.gmla_get_device_status()

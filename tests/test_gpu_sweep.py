"""GPU parity at the long-context sizes of the context-length table on the
"Foundations" page (section "The quadratic cost", 8K -> 128K -> 1M tokens):
causal prefill attention on sampled rows and latent-cache decode on sampled
heads, against the float64 oracle through the C ABI.  These are the sizes the
long-context sweep of bench.py times."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import Draw, prefill_qkv
from tests.gpu_util import assert_parity, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import causal_head_latent_b200 as gm
    return gm


@pytest.mark.parametrize("T", [131072, 1048576])
def test_prefill_long_context_sampled(g, T):
    """Causal prefill B=1, H=2 at T = 128K and 1M: rows at tile edges, the middle,
    the end and random positions, per head."""
    H = 2
    inp = prefill_qkv(700 + T % 997, 1, T, H)
    Q, K, V = (to_dev(inp[k]) for k in ("Q", "K", "V"))
    O = torch.empty_like(Q)
    g.gmla_attend_prefill(Q, K, V, O)
    g.gmla_get_device_status()
    got = f64(O)
    del Q, K, V
    rng = np.random.default_rng(T)
    ts = sorted(set([0, 1, 127, 128, 255, 256, T // 2, T - 129, T - 2, T - 1] + list(rng.integers(0, T, 6))))
    for h in range(H):
        sl = lambda k: inp[k][:, :, h:h + 1]
        ref = orc.attention(sl("Q"), sl("K"), sl("V"), rows=[(0, 0, t) for t in ts])
        assert_parity(np.stack([got[0, t, h] for t in ts]), np.stack([ref[0, t, 0] for t in ts]),
                      f"prefill T={T} head {h} sampled rows")
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("L", [131072, 1048576])
def test_decode_long_context_sampled(g, L):
    """Latent-cache decode B=2, H=96, d_c=512 at L = 128K and 1M, checked on
    sampled (b, h) pairs (the oracle rebuilds K_h, V_h from the cache)."""
    B, H, d_c = 2, 96, 512
    d = 128 * H
    dr = Draw(800 + L % 991)
    q = dr.normal((B, d))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    cache = dr.normal((B, L, d_c))
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    work = torch.empty(g.gmla_attend_decode_workspace_size(B, L, H, d_c), dtype=torch.uint8, device="cuda")
    g.gmla_attend_decode(to_dev(q), to_dev(cache), L, to_dev(Wk), to_dev(Wv), O, H, workspace=work)
    g.gmla_get_device_status()
    pairs = [(0, 0), (1, 95)] if L > 200000 else [(0, 0), (1, 95), (0, 48)]
    ref = orc.decode_latent(q, cache, L, Wk, Wv, H, heads=pairs)
    got = f64(O)
    sel = np.concatenate([np.arange(h * 128, (h + 1) * 128) + b * d for b, h in pairs])
    assert_parity(got.reshape(-1)[sel], ref.reshape(-1)[sel], f"decode L={L} sampled heads")
    assert np.all(np.isfinite(got))

"""GPU parity of the calls that split one decode or one prefill layer over
several GPUs, emulated here on one GPU (every share runs in turn on cuda:0):

* context-parallel decode -- gmla_attend_decode_partial over disjoint ranges of
  cached rows, the states stacked as an all-gather would stack them, then
  gmla_decode_combine -- against the oracle's plain decode over all rows
  (softmax over keys, "Kimi K3 - Softmax over keys"; K and V rebuilt from the
  cache, "Gated MLA" page);
* head-parallel prefill -- gmla_latent_project_heads, gmla_attend_prefill on the
  range's heads and gmla_gate_out_heads per head range, the shares summed as a
  reduction over GPUs would sum them -- against the oracle's layer.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import Draw, layer_weights
from tests.gpu_util import assert_parity, bits, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import causal_head_latent_b200 as gm
    return gm


def ws(nbytes):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device="cuda")


def _decode_inputs(seed, B, Lmax, H, d_c):
    d = 128 * H
    dr = Draw(seed)
    return {"q": dr.normal((B, d)), "cache": dr.normal((B, Lmax, d_c)),
            "Wk": dr.normal((d, d_c), 1 / np.sqrt(d_c)), "Wv": dr.normal((d, d_c), 1 / np.sqrt(d_c)),
            "G": dr.normal((B, d))}


def _oracle_state(x, b, h, k0, k1):
    """Oracle state of head h of sequence b over cached rows [k0, k1): the natural
    log-sum-exp of the scaled scores and c^ = sum_s a_s c_s with the weights
    normalised over the range (K_h rebuilt from the cache)."""
    D = 128
    cb = orc.widen(np.ascontiguousarray(x["cache"][b, k0:k1]))
    Kh = orc.linear(cb, x["Wk"][h * D:(h + 1) * D])
    qh = orc.widen(x["q"][b, h * D:(h + 1) * D]).reshape(1, 1, 1, D)
    n = k1 - k0
    _, wts, lse = orc.attention(qh, Kh.reshape(1, n, 1, D), Kh.reshape(1, n, 1, D), causal=True, want_weights=True,
                                want_lse=True)
    return lse[0, 0, 0], wts[0, 0, 0] @ cb


def _run_slices(g, x, B, L, H, d_c, slices, G=True):
    Q, C, Wk, Wv = (to_dev(x[k]) for k in ("q", "cache", "Wk", "Wv"))
    n = len(slices)
    lse = torch.empty(n, B, H, dtype=torch.float32, device="cuda")
    ctx = torch.empty(n, B, H, d_c, dtype=torch.float32, device="cuda")
    for i, (k0, k1) in enumerate(slices):
        work = ws(g.gmla_attend_decode_partial_workspace_size(B, k0, k1, H, d_c))
        g.gmla_attend_decode_partial(Q, C, k0, k1, Wk, lse[i], ctx[i], H, workspace=work)
    O = torch.full((B, 128 * H), float("nan"), dtype=torch.bfloat16, device="cuda")
    g.gmla_decode_combine(lse, ctx, Wv, O, G=to_dev(x["G"]) if G else None)
    g.gmla_get_device_status()
    return lse, ctx, O


@pytest.mark.parametrize("B,L,Lmax,H,d_c,cuts", [(3, 2049, 2100, 8, 512, (1000,)),
                                                 (2, 700, 700, 96, 512, (1, 350, 699)),
                                                 (4, 5000, 5000, 4, 256, (48, 2500, 4952))])
def test_partial_states_and_combine_match_oracle(g, B, L, Lmax, H, d_c, cuts):
    """Disjoint key ranges (a one-row range, ranges that end inside a tile)
    merged by gmla_decode_combine equal the decode over all L rows; each
    range's log-sum-exp and normalised latent context match the oracle's."""
    x = _decode_inputs(800 + L, B, Lmax, H, d_c)
    edges = (0,) + tuple(cuts) + (L,)
    slices = list(zip(edges[:-1], edges[1:]))
    lse, ctx, O = _run_slices(g, x, B, L, H, d_c, slices)
    ref = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"])
    assert_parity(f64(O), ref, f"combined decode over {len(slices)} ranges")
    lse_h, ctx_h = lse.cpu().double().numpy(), ctx.cpu().double().numpy()
    for i, (k0, k1) in enumerate(slices):
        for b, h in ((0, 0), (B - 1, H - 1), (B // 2, H // 2)):
            l_ref, c_ref = _oracle_state(x, b, h, k0, k1)
            # scores carry the bfloat16 rounding of q~ (relative 2^-9 per element): ~1e-3 in the log-sum-exp
            assert abs(lse_h[i, b, h] - l_ref) <= 5e-3, (i, b, h, lse_h[i, b, h], l_ref)
            assert_parity(ctx_h[i, b, h], c_ref, f"range {k0}..{k1} context (b={b}, h={h})")


def test_single_range_equals_workspace_decode(g):
    """One range over all rows, merged alone, gives gmla_attend_decode's result: both
    against the oracle, and against each other to within a few bfloat16 roundings
    (the combine applies W_v on CUDA cores in float32, the decode on tensor cores
    with the latent context split into two bfloat16 halves)."""
    B, L, H, d_c = 2, 3000, 96, 512
    x = _decode_inputs(870, B, L, H, d_c)
    _, _, O = _run_slices(g, x, B, L, H, d_c, [(0, L)])
    ref = torch.empty(B, 128 * H, dtype=torch.bfloat16, device="cuda")
    g.gmla_attend_decode(to_dev(x["q"]), to_dev(x["cache"]), L, to_dev(x["Wk"]), to_dev(x["Wv"]), ref, H,
                         G=to_dev(x["G"]), workspace=ws(g.gmla_attend_decode_workspace_size(B, L, H, d_c)))
    g.gmla_get_device_status()
    want = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"])
    assert_parity(f64(O), want, "one range through the combine")
    assert_parity(f64(ref), want, "gmla_attend_decode")
    a, b = f64(O), f64(ref)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.abs(b) + 1e-3 * np.abs(b).max())


def test_empty_range_is_skipped(g):
    """An empty range (a GPU whose slice holds no row) yields lse = -inf and a zero
    context, and merging it changes nothing."""
    B, L, H, d_c = 2, 900, 4, 128
    x = _decode_inputs(880, B, L, H, d_c)
    lse, ctx, O = _run_slices(g, x, B, L, H, d_c, [(0, 400), (400, 400), (400, L)])
    assert torch.all(torch.isneginf(lse[1])) and torch.all(ctx[1] == 0)
    ref = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"])
    assert_parity(f64(O), ref, "combine with an empty range")


def _layer(seed, B, T, H, d_c):
    d = 128 * H
    w = layer_weights(Draw(seed), d, d_c, x_shape=(B, T, d))
    return w, {k: to_dev(v) for k, v in w.items()}


@pytest.mark.parametrize("B,T,H,d_c,cuts", [(2, 300, 4, 128, (2,)), (1, 257, 6, 64, (1, 3))])
def test_head_ranges_sum_to_the_layer(g, B, T, H, d_c, cuts):
    """Per head range: projections of the range's heads (the latent in full),
    attention over those heads with the gate, and the range's share of W_o.
    The shares sum to the oracle's layer output; each range's Q equals the
    matching columns of the full projection bit for bit."""
    d = 128 * H
    w, t = _layer(900 + T, B, T, H, d_c)
    edges = (0,) + tuple(cuts) + (H,)
    Qfull = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], None, None, None, None, Q=Qfull)
    Ysum = np.zeros((B, T, d))
    for h0, h1 in zip(edges[:-1], edges[1:]):
        wr = 128 * (h1 - h0)
        Q, G, K, V, O = (torch.empty(B, T, wr, dtype=torch.bfloat16, device="cuda") for _ in range(5))
        C = torch.empty(B, T, d_c, dtype=torch.bfloat16, device="cuda")
        g.gmla_latent_project_heads(t["X"], h0, h1, t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C,
                                    K=K, V=V)
        v4 = lambda z: z.view(B, T, h1 - h0, 128)
        g.gmla_attend_prefill(v4(Q), v4(K), v4(V), v4(O), G=G)
        Y = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
        g.gmla_gate_out_heads(O, t["W_o"], Y, h0, h1)
        g.gmla_get_device_status()
        assert np.array_equal(bits(Q), bits(Qfull[:, :, 128 * h0:128 * h1]))
        Ysum += f64(Y)
    ref = orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H,
                        round_boundaries=True)
    assert_parity(Ysum, ref["output"], "sum of head-range shares")


def test_gate_out_heads_with_gate(g):
    """The ungated context of a head range with its gate logits: the share
    (sigmoid(G) (.) O) W_o[:, range]^T equals the oracle's."""
    rng = np.random.default_rng(9)
    from synth_inputs import bf16_bits_from_f64
    M, H, h0, h1 = 200, 4, 1, 3
    d, wr = 128 * H, 128 * (h1 - h0)
    O = bf16_bits_from_f64(rng.standard_normal((M, wr)))
    Gl = bf16_bits_from_f64(rng.standard_normal((M, wr)))
    W = bf16_bits_from_f64(rng.standard_normal((d, d)) / np.sqrt(d))
    Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_gate_out_heads(to_dev(O), to_dev(W), Y, h0, h1, G=to_dev(Gl),
                          workspace=ws(g.gmla_gate_out_workspace_size(M, wr)))
    g.gmla_get_device_status()
    ref = orc.linear(orc.gate(O, Gl), W[:, 128 * h0:128 * h1])
    assert_parity(f64(Y), ref, "gated head-range share")

"""Pins for the float64 oracle (CPU only).

Each test ties the oracle to something other than itself: a worked example
printed on the pages (fixtures in tests/golden/, each with its citation), a
closed form, an invariant, or an independent dense numpy formulation on tiny
shapes.  The mutation tests at the end switch in plausible mistakes and check
that at least one pin fails for each.
"""
import math

import numpy as np
import pytest

import oracle as orc
from synth_inputs import Draw, bf16_bits_from_f64, f64_from_bf16_bits, layer_weights
from tests.conftest import golden

# ---------------------------------------------------------------- helpers


def dense_layer(X, Wq, Wc, Wk, Wv, Wg, Wo, H, causal=True):
    """Independent dense formulation: per head softmax(QK^T/sqrt(D) + M) V with an
    explicit additive mask matrix, numpy matmuls, heads joined by reshape."""
    B, T, d = X.shape
    D = d // H
    C = X @ Wc.T
    Q = (X @ Wq.T).reshape(B, T, H, D).transpose(0, 2, 1, 3)
    K = (C @ Wk.T).reshape(B, T, H, D).transpose(0, 2, 1, 3)
    V = (C @ Wv.T).reshape(B, T, H, D).transpose(0, 2, 1, 3)
    M = np.where(np.tril(np.ones((T, T))) > 0, 0.0, -np.inf) if causal else np.zeros((T, T))
    S = Q @ K.transpose(0, 1, 3, 2) / math.sqrt(D) + M
    E = np.exp(S - S.max(axis=-1, keepdims=True))
    A = E / E.sum(axis=-1, keepdims=True)
    O = (A @ V).transpose(0, 2, 1, 3).reshape(B, T, d)
    gate = 1.0 / (1.0 + np.exp(-(X @ Wg.T)))
    return (gate * O) @ Wo.T, C, A, O


def tiny_layer(seed, B, T, d, H, d_c, bf16=False):
    dr = Draw(seed)
    w = layer_weights(dr, d, d_c, x_shape=(B, T, d), bf16=bf16)
    return {k: orc.widen(v) for k, v in w.items()}


def run_layer(w, H, causal=True, **kw):
    return orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H,
                         causal=causal, intermediates=True, **kw)


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- worked examples on the pages


def test_three_token_causal_pattern():
    g = golden("three_token_causal.json")
    Q, K, V = rand((1, 3, 2, 16), 1), rand((1, 3, 2, 16), 2), rand((1, 3, 2, 16), 3)
    for causal, key in ((True, "causal_visible"), (False, "noncausal_visible")):
        _, W = orc.attention(Q, K, V, causal=causal, want_weights=True)
        vis = np.array(g[key])
        for h in range(2):
            w = W[0, h]
            assert np.all(w[vis == 0] == 0.0)      # blocked keys weigh exactly zero
            assert np.all(w[vis == 1] > 0.0)       # every permitted key gets weight
            np.testing.assert_allclose(w.sum(-1), 1.0, atol=1e-14)


def test_gate_worked_example():
    g = golden("gate_example.json")
    out = orc.gate(np.array([g["context"]]), np.array([g["gate_logit"]]))
    assert out[0] == g["gated"]
    assert orc.gate(np.array([1.0]), np.array([0.0]))[0] == g["sigmoid"]


def test_latent_cache_identical_causal_and_noncausal():
    w = tiny_layer(11, 2, 3, 16, 2, 8)
    a = run_layer(w, 2, causal=True)
    b = run_layer(w, 2, causal=False)
    assert np.array_equal(a["latent_cache"], b["latent_cache"])
    assert a["latent_cache"].shape == (2, 3, 8)
    assert not np.array_equal(a["output"][:, :2], b["output"][:, :2])  # the mask matters before t = T-1


def test_decode_shape_of_softmax_page():
    g = golden("decode_softmax_shape.json")
    Tk, H = g["keys"], 4
    rng = np.random.default_rng(5)
    Q, K, V = rng.standard_normal((1, H, 1, 8)), rng.standard_normal((1, H, Tk, 8)), rng.standard_normal((1, H, Tk, 8))
    _, W = orc.attention(Q, K, V, causal=True, layout="bhtd", want_weights=True)
    assert W.shape == (1, H, g["queries"], g["keys"])
    # the single query sits at position p = 1000 and sees keys 0..p, all of them
    assert np.all(W > 0.0)
    np.testing.assert_allclose(W.sum(-1), 1.0, atol=1e-13)


def test_dot_product_orders_match_causal_pair_count():
    g = golden("dot_product_orders.json")
    for row in g["rows"]:
        T = row["T"]
        pairs = T * (T + 1) / 2
        assert abs(pairs / row["dot_products"] - 1.0) < g["relative_tolerance"]


def test_k3_dims_fixture():
    g = golden("k3_dims.json")
    assert g["num_attention_heads"] * g["head_dim"] == 12288
    assert g["num_attention_heads"] * 256 == g["uncompressed_dims"]


# ---------------------------------------------------------------- softmax facts


@pytest.mark.parametrize("Tq,Tk", [(1, 1), (5, 5), (7, 7), (3, 10), (1, 33)])
def test_rows_sum_to_one_and_blocked_zero(Tq, Tk):
    Q, K, V = rand((2, Tq, 3, 8), 10 + Tq), rand((2, Tk, 3, 8), 20 + Tk), rand((2, Tk, 3, 8), 30)
    _, W = orc.attention(Q, K, V, causal=True, want_weights=True)
    np.testing.assert_allclose(W.sum(-1), 1.0, atol=1e-12)
    for t in range(Tq):
        pos = Tk - Tq + t
        assert np.all(W[:, :, t, pos + 1:] == 0.0)
        assert np.all(W[:, :, t, :pos + 1] > 0.0)


def test_first_query_returns_first_value_exactly():
    Q, K, V = rand((2, 9, 4, 16), 40), rand((2, 9, 4, 16), 41), rand((2, 9, 4, 16), 42)
    O = orc.attention(Q, K, V, causal=True)
    assert np.array_equal(O[:, 0], V[:, 0])


def test_uniform_scores_give_mean_of_visible_values():
    T = 12
    Q = np.zeros((1, T, 2, 8))
    K, V = rand((1, T, 2, 8), 43), rand((1, T, 2, 8), 44)
    O = orc.attention(Q, K, V, causal=True)
    for t in range(T):
        np.testing.assert_allclose(O[0, t], V[0, :t + 1].mean(axis=0), rtol=0, atol=1e-14)
    On = orc.attention(Q, K, V, causal=False)
    np.testing.assert_allclose(On[0], np.broadcast_to(V[0].mean(axis=0), On[0].shape), atol=1e-14)


def test_softmax_shift_invariance():
    # a key feature equal to 1 for every key adds q[t, -1]/sqrt(D) to every score of row t
    T, D = 10, 8
    Q, K, V = rand((1, T, 1, D), 45), rand((1, T, 1, D), 46), rand((1, T, 1, D), 47)
    K[..., -1] = 1.0
    _, W1 = orc.attention(Q, K, V, want_weights=True)
    Q2 = Q.copy()
    Q2[..., -1] += 37.0
    _, W2 = orc.attention(Q2, K, V, want_weights=True)
    np.testing.assert_allclose(W1, W2, atol=1e-13)


def test_scale_gives_unit_variance_scores():
    D, n = 128, 20000
    rng = np.random.default_rng(48)
    q, k = rng.standard_normal((n, D)), rng.standard_normal((n, D))
    # scores through the oracle: one query per row against one key, with weights = 1 -> read lse
    Q = q.reshape(1, n, 1, D)
    K = k.reshape(1, n, 1, D)
    s = np.empty(n)
    # lse of a single-key row equals its scaled score
    for j in range(0, n, 2000):
        _, lse = orc.attention(Q[:, j:j + 2000].transpose(1, 0, 2, 3), K[:, j:j + 2000].transpose(1, 0, 2, 3),
                               K[:, j:j + 2000].transpose(1, 0, 2, 3), want_lse=True)
        s[j:j + 2000] = lse[:, 0, 0]
    assert abs(s.var() - 1.0) < 0.05
    np.testing.assert_allclose(s, (q * k).sum(1) / math.sqrt(D), atol=1e-12)


# ---------------------------------------------------------------- brute force against a dense formulation


@pytest.mark.parametrize("B,T,d,H,d_c", [(1, 1, 8, 1, 4), (1, 2, 8, 2, 4), (1, 3, 16, 2, 8),
                                         (2, 5, 16, 4, 8), (1, 8, 64, 4, 32)])
@pytest.mark.parametrize("causal", [True, False])
def test_layer_matches_dense_formulation(B, T, d, H, d_c, causal):
    w = tiny_layer(100 + T * 7 + H, B, T, d, H, d_c)
    r = run_layer(w, H, causal=causal)
    Y, C, A, O = dense_layer(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H, causal)
    np.testing.assert_allclose(r["latent_cache"], C, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["O"], O, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r["output"], Y, rtol=1e-11, atol=1e-12)
    assert r["output"].shape == w["X"].shape


def test_tiny_fp32_forward_config():
    """Tiny Gated MLA forward: B=1, T=8, d_model=64, H=4 x D_h=16, d_c=32, fp32 inputs, seed 0."""
    dr = Draw(0)
    w = layer_weights(dr, 64, 32, x_shape=(1, 8, 64), bf16=False)
    assert all(v.dtype == np.float32 for v in w.values())
    w = {k: orc.widen(v) for k, v in w.items()}
    r = run_layer(w, 4)
    Y, C, _, _ = dense_layer(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], 4)
    assert r["output"].shape == (1, 8, 64) and r["latent_cache"].shape == (1, 8, 32)
    np.testing.assert_allclose(r["output"], Y, rtol=1e-11, atol=1e-12)
    assert np.all(np.isfinite(r["output"]))


# ---------------------------------------------------------------- structure of the layer


def test_gate_zero_logits_halve_the_output():
    w = tiny_layer(12, 1, 4, 16, 2, 8)
    w["W_g"] = np.zeros_like(w["W_g"])
    r = run_layer(w, 2)
    np.testing.assert_allclose(r["output"], 0.5 * (r["O"] @ w["W_o"].T), rtol=1e-13, atol=1e-14)


def test_closed_gate_gives_zero_output():
    w = tiny_layer(13, 1, 4, 16, 2, 8)
    w["W_g"] = np.zeros_like(w["W_g"])
    w["W_g"][:, 0] = -1e6          # logits -1e6 * x_0: sigmoid underflows to exactly 0 where x_0 > 0
    w["X"][..., 0] = 1.0
    r = run_layer(w, 2)
    assert np.all(r["output"] == 0.0)
    assert np.all(orc.gate(np.ones(3), np.full(3, -np.inf)) == 0.0)


def test_gate_is_channelwise_and_before_output_projection():
    w = tiny_layer(14, 1, 3, 16, 2, 8)
    r = run_layer(w, 2)
    g = 1.0 / (1.0 + np.exp(-(w["X"] @ w["W_g"].T)))
    np.testing.assert_allclose(r["O_gated"], g * r["O"], rtol=1e-14)
    np.testing.assert_allclose(r["output"], (g * r["O"]) @ w["W_o"].T, rtol=1e-12, atol=1e-14)
    # a per-token gate (one number per token) would not reproduce per-channel control
    assert np.ptp(g, axis=-1).min() > 0


def test_heads_are_concatenated_not_summed():
    H, D, d_c = 3, 4, 8
    w = tiny_layer(15, 1, 5, H * D, H, d_c)
    r = run_layer(w, H)
    perm = [2, 0, 1]
    idx = np.concatenate([np.arange(p * D, (p + 1) * D) for p in perm])
    w2 = dict(w)
    for k in ("W_q", "W_k", "W_v"):
        w2[k] = w[k][idx]
    r2 = run_layer(w2, H)
    np.testing.assert_allclose(r2["O"], r["O"][..., idx], rtol=1e-12, atol=1e-14)


def test_causal_prefix_property():
    w = tiny_layer(16, 1, 6, 16, 2, 8)
    r = run_layer(w, 2)
    w2 = dict(w)
    w2["X"] = w["X"].copy()
    w2["X"][:, 4:] += 3.0
    r2 = run_layer(w2, 2)
    assert np.array_equal(r["output"][:, :4], r2["output"][:, :4])
    assert not np.array_equal(r["output"][:, 4:], r2["output"][:, 4:])


def test_noncausal_permutation_equivariance():
    # no positional encoding: permuting tokens permutes the non-causal output
    w = tiny_layer(17, 1, 6, 16, 2, 8)
    r = run_layer(w, 2, causal=False)
    perm = np.array([3, 0, 5, 1, 4, 2])
    w2 = dict(w)
    w2["X"] = w["X"][:, perm]
    r2 = run_layer(w2, 2, causal=False)
    np.testing.assert_allclose(r2["output"], r["output"][:, perm], rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- decode


def _absorbed_decode(q, Cc, L, Wk, Wv, H):
    """Absorbed form written independently: q~_h = W_k^(h)T q_h, weights over
    latents, context mixed in latent space, then W_v^(h)."""
    B, d = q.shape
    D = d // H
    out = np.empty((B, d))
    for b in range(B):
        for h in range(H):
            qt = Wk[h * D:(h + 1) * D].T @ q[b, h * D:(h + 1) * D]      # [d_c]
            s = Cc[b, :L] @ qt / math.sqrt(D)
            a = np.exp(s - s.max())
            a /= a.sum()
            chat = a @ Cc[b, :L]                                        # [d_c]
            out[b, h * D:(h + 1) * D] = Wv[h * D:(h + 1) * D] @ chat
    return out


def test_decode_absorption_identity():
    B, H, D, d_c, L = 2, 3, 8, 16, 37
    rng = np.random.default_rng(50)
    q = rng.standard_normal((B, H * D))
    Cc = rng.standard_normal((B, L + 5, d_c))
    Wk = rng.standard_normal((H * D, d_c)) / 4
    Wv = rng.standard_normal((H * D, d_c)) / 4
    o = orc.decode_latent(q, Cc, L, Wk, Wv, H)
    np.testing.assert_allclose(o, _absorbed_decode(q, Cc, L, Wk, Wv, H), rtol=1e-11, atol=1e-12)


def test_decode_equals_prefill_row():
    B, T, d, H, d_c = 1, 7, 16, 2, 8
    w = tiny_layer(18, B, T, d, H, d_c)
    r = run_layer(w, H)
    for t in range(T):
        o = orc.decode_latent(r["Q"][:, t], r["latent_cache"], t + 1, w["W_k"], w["W_v"], H, G=r["G"][:, t])
        np.testing.assert_allclose(o, r["O_gated"][:, t], rtol=1e-12, atol=1e-13)


def test_decode_weights_and_subset():
    B, H, D, d_c, L = 2, 4, 8, 16, 20
    rng = np.random.default_rng(51)
    q = rng.standard_normal((B, H * D))
    Cc = rng.standard_normal((B, L, d_c))
    Wk = rng.standard_normal((H * D, d_c))
    Wv = rng.standard_normal((H * D, d_c))
    full, W = orc.decode_latent(q, Cc, L, Wk, Wv, H, want_weights=True)
    np.testing.assert_allclose(W.sum(-1), 1.0, atol=1e-12)
    sub = orc.decode_latent(q, Cc, L, Wk, Wv, H, heads=[(1, 2)])
    np.testing.assert_array_equal(sub[1, 16:24], full[1, 16:24])
    assert np.isnan(sub[0]).all()


# ---------------------------------------------------------------- bfloat16 rounding helpers


def test_bf16_rounding_known_values():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -30, 3.0e-3])
    exp = np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7, 197 * 2 ** -16])
    np.testing.assert_array_equal(orc.round_bf16(vals), exp)
    np.testing.assert_array_equal(f64_from_bf16_bits(bf16_bits_from_f64(vals)), exp)


def test_bf16_rounding_agrees_between_oracle_and_inputs():
    x = np.random.default_rng(52).standard_normal(100000) * np.exp(np.random.default_rng(53).uniform(-20, 20, 100000))
    a = orc.round_bf16(x)
    b = f64_from_bf16_bits(bf16_bits_from_f64(x))
    np.testing.assert_array_equal(a, b)
    import torch
    c = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    # float32 -> bf16 is a second rounding; compare only where x is exact in float32
    exact = x.astype(np.float32).astype(np.float64) == x
    np.testing.assert_array_equal(a[exact], c[exact])
    xf = x.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(orc.round_bf16(xf), torch.from_numpy(xf.astype(np.float32)).to(torch.bfloat16).double().numpy())


# ---------------------------------------------------------------- planted mistakes are caught


def _pins_pass():
    """A compact battery of the pins above; returns False if any fails."""
    try:
        test_three_token_causal_pattern()
        test_rows_sum_to_one_and_blocked_zero(3, 10)
        test_first_query_returns_first_value_exactly()
        test_uniform_scores_give_mean_of_visible_values()
        test_scale_gives_unit_variance_scores()
        test_layer_matches_dense_formulation(2, 5, 16, 4, 8, True)
        test_gate_is_channelwise_and_before_output_projection()
        test_heads_are_concatenated_not_summed()
        test_decode_absorption_identity()
    except AssertionError:
        return False
    return True


def test_pins_pass_on_the_unmutated_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("code", [1, 2, 3, 4, "gate_after_wo", "wo_untransposed", "heads_summed"])
def test_each_planted_mistake_fails_a_pin(code):
    with orc.mutation(code):
        assert not _pins_pass()

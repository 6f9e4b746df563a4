"""GPU parity: attention over explicit Q, K, V (gmla_attend_prefill) against the
float64 oracle, through the C ABI, on seeded synthetic inputs."""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import SEEDS, decode_plain_qkv, prefill_qkv
from tests.gpu_util import ROW_SUM, assert_parity, bits, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import causal_head_latent_b200 as gm
    return gm


def run_prefill(g, inp, causal=True, gate=False, lse=False, weights=False, layout="bthd"):
    Q, K, V = to_dev(inp["Q"]), to_dev(inp["K"]), to_dev(inp["V"])
    O = torch.empty_like(Q)
    if layout == "bthd":
        B, Tq, H, D = Q.shape
        Tk = K.shape[1]
    else:
        B, H, Tq, D = Q.shape
        Tk = K.shape[2]
    G = to_dev(inp["G"]) if gate else None
    L = torch.full((B, H, Tq), float("nan"), device="cuda") if lse else None
    W = torch.full((B, H, Tq, Tk), float("nan"), device="cuda") if weights else None
    before = [bits(t).copy() for t in (Q, K, V)]
    g.gmla_attend_prefill(Q, K, V, O, causal=causal, G=G, lse=L, weights=W, layout=layout)
    g.gmla_get_device_status()
    for b0, t in zip(before, (Q, K, V)):
        assert np.array_equal(b0, bits(t)), "an input was modified"
    return O, L, W


@pytest.mark.parametrize("B,H,Tq,Tk", [(2, 3, 300, 300), (1, 2, 128, 128), (1, 2, 5, 5), (1, 1, 129, 129),
                                       (2, 2, 200, 333), (1, 2, 256, 1000), (1, 3, 7, 130)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_matches_oracle(g, B, H, Tq, Tk, causal):
    inp = prefill_qkv(101 + Tq + Tk, B, Tq, H, Tk=Tk)
    O, L, W = run_prefill(g, inp, causal=causal, lse=True, weights=True)
    ref, wref, lref = orc.attention(inp["Q"], inp["K"], inp["V"], causal=causal, want_weights=True, want_lse=True)
    assert_parity(f64(O), ref, "O")
    np.testing.assert_allclose(f64(L), lref, rtol=0, atol=2e-4)
    w = f64(W)
    assert np.abs(w.sum(-1) - 1.0).max() <= ROW_SUM
    assert np.all(w[wref == 0.0] == 0.0)     # blocked keys weigh exactly zero
    assert np.abs(w - wref).max() < 1e-4


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_many_items_per_cta(g, causal):
    """More query pairs than SMs (B=2, H=40, T=1100: 400 items), so running CTAs
    take over the items of CTAs that have not started and carry their
    pipelines from one item to the next; the last pair of every head has rows
    for its first query tile only.  Every output and log-sum-exp is compared."""
    B, H, T = 2, 40, 1100
    inp = prefill_qkv(171 + causal, B, T, H, gate=True)
    Q, K, V, G = (to_dev(inp[k]) for k in ("Q", "K", "V", "G"))
    O = torch.empty_like(Q)
    L = torch.empty(B, H, T, device="cuda")
    g.gmla_attend_prefill(Q, K, V, O, causal=causal, G=G, lse=L)
    g.gmla_get_device_status()
    ref, lref = orc.attention(inp["Q"], inp["K"], inp["V"], causal=causal, want_lse=True)
    ref = orc.gate(ref.reshape(B, T, -1), inp["G"]).reshape(ref.shape)
    assert_parity(f64(O), ref, "O over 400 items")
    np.testing.assert_allclose(f64(L), lref, rtol=0, atol=2e-4)


def test_prefill_gate_and_layout(g):
    inp = prefill_qkv(7, 2, 260, 3, gate=True)
    O, _, _ = run_prefill(g, inp, gate=True)
    ref = orc.attention(inp["Q"], inp["K"], inp["V"])
    B, T, H, D = ref.shape
    gated = orc.gate(ref.reshape(B, T, H * D), inp["G"]).reshape(ref.shape)
    assert_parity(f64(O), gated, "gated O")
    # [B, H, T, D] layout through the strides
    inp2 = {k: np.ascontiguousarray(v.transpose(0, 2, 1, 3)) for k, v in inp.items() if k != "G"}
    O2, _, _ = run_prefill(g, inp2, layout="bhtd")
    ref2 = orc.attention(inp2["Q"], inp2["K"], inp2["V"], layout="bhtd")
    assert_parity(f64(O2), ref2, "bhtd O")


def test_first_query_returns_first_value_exactly(g):
    inp = prefill_qkv(8, 2, 300, 2)
    O, _, _ = run_prefill(g, inp)
    assert np.array_equal(bits(O)[:, 0], inp["V"][:, 0])


def test_uniform_scores_give_mean(g):
    inp = prefill_qkv(9, 1, 300, 2)
    inp["Q"] = np.zeros_like(inp["Q"])
    O, _, _ = run_prefill(g, inp)
    V = orc.widen(inp["V"])
    mean = np.cumsum(V, axis=1) / np.arange(1, 301).reshape(1, -1, 1, 1)
    assert_parity(f64(O), mean, "uniform-score mean")


def test_gate_extremes(g):
    inp = prefill_qkv(10, 1, 200, 2, gate=True)
    ninf = np.uint16(0xFF80)   # bfloat16 -inf
    inp["G"] = np.full_like(inp["G"], ninf)
    O, _, _ = run_prefill(g, inp, gate=True)
    assert np.all(f64(O) == 0.0)
    inp["G"] = np.zeros_like(inp["G"])
    O, _, _ = run_prefill(g, inp, gate=True)
    ref = orc.attention(inp["Q"], inp["K"], inp["V"])
    assert_parity(f64(O), 0.5 * ref, "gate 0 halves")


def test_decode_softmax_page_shape_full(g):
    """Decode exactly as the softmax page: B=8, 96 heads, 1 query at p=1000, 1001 keys, [B,H,T,D]."""
    inp = decode_plain_qkv(SEEDS["decode_plain"], 8, 96, 1001)
    O, L, W = run_prefill(g, inp, lse=True, weights=True, layout="bhtd")
    ref, wref = orc.attention(inp["Q"], inp["K"], inp["V"], layout="bhtd", want_weights=True)
    assert_parity(f64(O), ref, "decode O")
    w = f64(W)
    assert np.abs(w.sum(-1) - 1.0).max() <= ROW_SUM
    assert np.abs(w - wref).max() < 1e-5


@pytest.mark.parametrize("Tq,Tk", [(1, 1), (1, 2), (1, 5), (2, 16), (1, 17), (1, 129), (1, 131), (4, 193), (3, 200),
                                   (4, 517), (1, 768), (3, 769), (2, 1024), (1, 1015)])
@pytest.mark.parametrize("causal", [True, False])
def test_few_query_rows_matches_oracle(g, Tq, Tk, causal):
    """Tq <= 4 runs on the CUDA-core rows kernel.  The key counts cover tiny inputs
    and last-visible-key positions whose residue mod 64 falls on every half-warp
    pairing (the loop must keep both half-warps of a warp together), and key
    counts of 8 to 16 whole or ragged tiles (517, 768, 769, 1015, 1024)."""
    inp = prefill_qkv(61 + Tk + Tq, 2, Tq, 3, Tk=Tk, gate=True)
    O, L, W = run_prefill(g, inp, causal=causal, gate=True, lse=True, weights=True)
    ref, wref, lref = orc.attention(inp["Q"], inp["K"], inp["V"], causal=causal, want_weights=True, want_lse=True)
    assert_parity(f64(O), orc.gate(ref.reshape(2, Tq, -1), inp["G"]).reshape(ref.shape), "few-query rows")
    np.testing.assert_allclose(f64(L), lref, atol=5e-4)
    w = f64(W)
    assert np.abs(w.sum(-1) - 1.0).max() <= ROW_SUM
    assert np.all(w[wref == 0.0] == 0.0)
    assert np.abs(w - wref).max() < 1e-4


@pytest.mark.parametrize("B,H,T", [(1, 20, 2048), (3, 7, 1100)])
def test_prefill_launch_groups_every_row(g, B, H, T):
    """CTAs launch in groups of (b, h) pairs, the query pairs longest first
    across a group.  Here B*H = 20 pairs in groups of 16 (one full group and a
    partial one of 4), and 21 pairs of a ragged length (a group of 16 that spans
    three sequences and a partial one of 5): every output row of every head
    against the oracle."""
    inp = prefill_qkv(77 + H + T, B, T, H)
    O, L, _ = run_prefill(g, inp, lse=True)
    ref, lref = orc.attention(inp["Q"], inp["K"], inp["V"], want_lse=True)
    assert_parity(f64(O), ref, "grouped launch, all rows")
    np.testing.assert_allclose(f64(L), lref, atol=5e-4)


def test_prefill_8k_full_size_sampled(g):
    """Causal prefill B=1, H=96, T=8192 (the timed launch), checked on sampled rows."""
    T, H = 8192, 96
    inp = prefill_qkv(SEEDS["prefill_attn"], 1, T, H)
    O, L, _ = run_prefill(g, inp, lse=True)
    rng = np.random.default_rng(0)
    ts = [0, 1, 127, 128, 129, 4095, 4096, 8190, 8191] + list(rng.integers(0, T, 23))
    hs = [0, 47, 95] + list(rng.integers(0, H, 5))
    rows = np.array([(0, h, t) for h in hs for t in ts], dtype=np.int64)
    ref, lref = orc.attention(inp["Q"], inp["K"], inp["V"], rows=rows, want_lse=True)
    got = f64(O)
    sel_g = np.stack([got[0, t, h] for _, h, t in rows])
    sel_r = np.stack([ref[0, t, h] for _, h, t in rows])
    assert_parity(sel_g, sel_r, "8K prefill sampled rows")
    lg = f64(L)
    np.testing.assert_allclose([lg[0, h, t] for _, h, t in rows], [lref[0, h, t] for _, h, t in rows], atol=5e-4)
    # the whole output is finite and the first row is exactly v_0
    assert np.all(np.isfinite(got))
    assert np.array_equal(bits(O)[0, 0], inp["V"][0, 0])

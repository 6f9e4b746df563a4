"""GPU parity: projections (gmla_latent_project), output projection
(gmla_gate_out), latent-cache decode (gmla_attend_decode) and the chained
layer, against the float64 oracle through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import SEEDS, Draw, layer_weights
from tests.gpu_util import ROW_SUM, assert_parity, bits, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import causal_head_latent_b200 as gm
    return gm


def make_layer(seed, B, T, d, d_c):
    dr = Draw(seed)
    w = layer_weights(dr, d, d_c, x_shape=(B, T, d))
    return w, {k: to_dev(v) for k, v in w.items()}


def ws(nbytes):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("B,T,d,d_c,cache_len_max,cache_pos", [(2, 200, 256, 64, 200, 0), (1, 130, 384, 128, 300, 17),
                                                               (3, 1, 256, 64, 9, 8)])
def test_latent_project_matches_oracle(g, B, T, d, d_c, cache_len_max, cache_pos):
    w, t = make_layer(200 + T, B, T, d, d_c)
    Q = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    G = torch.empty_like(Q)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    C = torch.zeros(B, cache_len_max, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C,
                          cache_pos=cache_pos, K=K, V=V)
    g.gmla_get_device_status()
    assert_parity(f64(Q), orc.linear(w["X"], w["W_q"]), "Q")
    assert_parity(f64(G), orc.linear(w["X"], w["W_g"]), "G")
    Cg = f64(C)
    assert_parity(Cg[:, cache_pos:cache_pos + T], orc.linear(w["X"], w["W_c"]), "C")
    # rows outside [cache_pos, cache_pos + T) untouched
    assert np.all(Cg[:, :cache_pos] == 0) and np.all(Cg[:, cache_pos + T:] == 0)
    # K, V are expanded from the latents as stored in bfloat16; the oracle rounds its
    # own latents at the same boundary (no GPU value feeds the oracle)
    Cr = orc.round_bf16(orc.linear(w["X"], w["W_c"]))
    assert_parity(f64(K), orc.linear(Cr, w["W_k"]), "K")
    assert_parity(f64(V), orc.linear(Cr, w["W_v"]), "V")


@pytest.mark.parametrize("B,d,d_c,cache_len_max,cache_pos", [(32, 1024, 128, 9, 5), (7, 1536, 64, 3, 2)])
def test_decode_step_projections_split_k(g, B, d, d_c, cache_len_max, cache_pos):
    """One new token per sequence (M = B <= 32 rows, K = d >= 768): fewer output
    tiles than SMs, so the products run split over the K chunks by clusters of
    CTAs whose partial rows are added in the first CTA.  Q, G, the appended
    latent and the output projection against the oracle; cache rows other than
    cache_pos untouched."""
    w, t = make_layer(500 + B, B, 1, d, d_c)
    Q = torch.empty(B, 1, d, dtype=torch.bfloat16, device="cuda")
    G = torch.empty_like(Q)
    C = torch.zeros(B, cache_len_max, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], None, None, Q=Q, G=G, C=C, cache_pos=cache_pos)
    Y = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_gate_out(t["X"].view(B, d), t["W_o"], Y)
    g.gmla_get_device_status()
    assert_parity(f64(Q), orc.linear(w["X"], w["W_q"]), "Q")
    assert_parity(f64(G), orc.linear(w["X"], w["W_g"]), "G")
    Cg = f64(C)
    assert_parity(Cg[:, cache_pos:cache_pos + 1], orc.linear(w["X"], w["W_c"]), "C")
    assert np.all(Cg[:, :cache_pos] == 0) and np.all(Cg[:, cache_pos + 1:] == 0)
    assert_parity(f64(Y), orc.linear(w["X"].reshape(B, d), w["W_o"]), "Y")


def test_decode_step_projections_full_size(g):
    """The decode step's products at their full size: 32 new tokens, d_model=12288,
    d_c=512.  [Q | G | C] has 131 tiles of 192 columns (the last of the latent's
    512 columns a partial tile) run unsplit, W_o 64 tiles of 192 split over
    two-CTA clusters (128 CTAs).  Every row against the oracle; the appended
    latent lands in its cache row only."""
    B, d, d_c, cache_len_max, cache_pos = 32, 12288, 512, 6, 4
    w, t = make_layer(SEEDS["layer_prefill"] + 1, B, 1, d, d_c)
    Q = torch.empty(B, 1, d, dtype=torch.bfloat16, device="cuda")
    G = torch.empty_like(Q)
    C = torch.zeros(B, cache_len_max, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], None, None, Q=Q, G=G, C=C, cache_pos=cache_pos)
    Y = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_gate_out(t["X"].view(B, d), t["W_o"], Y)
    g.gmla_get_device_status()
    del t
    torch.cuda.empty_cache()
    X2 = w["X"].reshape(B, d)
    assert_parity(f64(Q).reshape(B, d), orc.linear(X2, w["W_q"]), "Q (131 tiles of 192)")
    assert_parity(f64(G).reshape(B, d), orc.linear(X2, w["W_g"]), "G")
    Cg = f64(C)
    assert_parity(Cg[:, cache_pos], orc.linear(X2, w["W_c"]), "C (partial last tile)")
    assert np.all(Cg[:, :cache_pos] == 0) and np.all(Cg[:, cache_pos + 1:] == 0)
    assert_parity(f64(Y), orc.linear(X2, w["W_o"]), "Y (64 tiles of 192, split in two)")


@pytest.mark.parametrize("with_v", [False, True])
def test_expand_kv_few_rows_wide(g, with_v):
    """A few rows of one sequence expanded to a wide d_model (16384): K alone runs
    64 tiles of 256 columns split over two-CTA clusters, K and V together 128
    tiles of 256 unsplit (192-column tiles would need more CTAs than SMs)."""
    B, Lmax, d_c, d = 1, 64, 512, 16384
    dr = Draw(37)
    cache = dr.normal((B, Lmax, d_c))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    row0, rows = 7, 20
    K = torch.empty(B, rows, d, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K) if with_v else None
    g.gmla_expand_kv(to_dev(cache), row0, rows, W_k=to_dev(Wk), W_v=to_dev(Wv) if with_v else None, K=K, V=V)
    g.gmla_get_device_status()
    assert_parity(f64(K), orc.linear(cache[:, row0:row0 + rows], Wk), "expanded K")
    if with_v:
        assert_parity(f64(V), orc.linear(cache[:, row0:row0 + rows], Wv), "expanded V")


def test_gate_out_matches_oracle(g):
    rng = np.random.default_rng(3)
    from synth_inputs import bf16_bits_from_f64
    M, d = 300, 384
    O = bf16_bits_from_f64(rng.standard_normal((M, d)))
    W = bf16_bits_from_f64(rng.standard_normal((d, d)) / np.sqrt(d))
    Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_gate_out(to_dev(O), to_dev(W), Y)
    g.gmla_get_device_status()
    assert_parity(f64(Y), orc.linear(O, W), "Y")


def test_gate_out_with_gate_matches_oracle(g):
    """gmla_gate_out given the gate logits: Y = (sigmoid(G) (.) O) W_o^T, the gate
    before W_o ("Gated MLA" page, "The channel-wise output gate"); logits of -inf
    close every channel, so Y is exactly 0 there."""
    rng = np.random.default_rng(5)
    from synth_inputs import bf16_bits_from_f64
    M, d = 300, 384
    O = bf16_bits_from_f64(rng.standard_normal((M, d)))
    Gl = bf16_bits_from_f64(rng.standard_normal((M, d)))
    Gl[17] = 0xFF80  # bfloat16 -inf: row 17 fully gated off
    W = bf16_bits_from_f64(rng.standard_normal((d, d)) / np.sqrt(d))
    Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    work = ws(g.gmla_gate_out_workspace_size(M, d))
    g.gmla_gate_out(to_dev(O), to_dev(W), Y, G=to_dev(Gl), workspace=work)
    g.gmla_get_device_status()
    ref = orc.linear(orc.gate(O, Gl), W)
    assert np.all(ref[17] == 0)
    got = f64(Y)
    assert np.all(got[17] == 0)
    assert_parity(got, ref, "gated Y")
    # without its workspace the gated form is refused before any launch
    assert g.STATUS[g.gmla_gate_out(to_dev(O), to_dev(W), Y, G=to_dev(Gl), check=False)] == "GMLA_ERR_WORKSPACE"


def test_gemm_persistent_multi_tile_full_output(g):
    """More than 2 x 148 output tiles per launch, so every CTA of the persistent
    GEMM runs three or four tiles: both TMEM accumulators, the phase flips of
    their barriers across tiles and several groups of the grouped raster are
    exercised, and every output element is compared with the oracle."""
    B, T, H, d_c = 2, 2048, 12, 512
    d = 128 * H
    w, t = make_layer(41, B, T, d, d_c)
    Q = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    G, K, V = (torch.empty_like(Q) for _ in range(3))
    C = torch.empty(B, T, d_c, dtype=torch.bfloat16, device="cuda")
    # [Q | G | C]: 32 m-tiles x (6 + 6 + 2) n-tiles = 448 tiles; [K | V]: 32 x 12 = 384 tiles
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C, K=K, V=V)
    # W_o with the gate: 64 m-tiles x 6 n-tiles = 384 tiles
    dr = Draw(43)
    O2, G2 = dr.normal((8192, d)), dr.normal((8192, d))
    Y2 = torch.empty(8192, d, dtype=torch.bfloat16, device="cuda")
    g.gmla_gate_out(to_dev(O2), t["W_o"], Y2, G=to_dev(G2), workspace=ws(g.gmla_gate_out_workspace_size(8192, d)))
    g.gmla_get_device_status()
    assert_parity(f64(Q), orc.linear(w["X"], w["W_q"]), "Q (448 tiles)")
    assert_parity(f64(G), orc.linear(w["X"], w["W_g"]), "G (448 tiles)")
    Cref = orc.linear(w["X"], w["W_c"])
    assert_parity(f64(C), Cref, "C (448 tiles)")
    Cr = orc.round_bf16(Cref)
    assert_parity(f64(K), orc.linear(Cr, w["W_k"]), "K (384 tiles)")
    assert_parity(f64(V), orc.linear(Cr, w["W_v"]), "V (384 tiles)")
    assert_parity(f64(Y2), orc.linear(orc.gate(O2, G2), w["W_o"]), "gated W_o (384 tiles)")


def test_layer_full_size_sampled_rows(g):
    """The full layer at its prefill size -- B=2, T=4096, d_model=12288 (96 heads of
    128), d_c=512 -- through the C ABI: gmla_latent_project (Q, G, C, K, V),
    gmla_attend_prefill with the gate, gmla_gate_out.  The GEMMs run 12416, 12288
    and 6144 tiles on 148 CTAs.  Checked at 32 token rows spread over both
    sequences and all four 16-m-tile raster groups, against the oracle, which
    rounds to bfloat16 where the library stores bfloat16 ("Gated MLA" page,
    "Implementation order")."""
    B, T, H, d_c = 2, 4096, 96, 512
    d = 128 * H
    w, t = make_layer(SEEDS["layer_prefill"], B, T, d, d_c)
    Q = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    G, K, V, O, Y = (torch.empty_like(Q) for _ in range(5))
    C = torch.empty(B, T, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C, K=K, V=V)
    v4 = lambda x: x.view(B, T, H, 128)
    g.gmla_attend_prefill(v4(Q), v4(K), v4(V), v4(O), G=G)
    g.gmla_gate_out(O, t["W_o"], Y)
    g.gmla_get_device_status()
    del t
    torch.cuda.empty_cache()

    rng = np.random.default_rng(4)
    m_tiles = np.concatenate([rng.choice(np.arange(q * 16, q * 16 + 16), 8, replace=False) for q in range(4)])
    rows = np.sort(m_tiles * 128 + rng.integers(0, 128, m_tiles.size))  # flat token rows in [0, B*T)
    rb = orc.round_bf16
    X2 = w["X"].reshape(B * T, d)
    flat = lambda x: f64(x).reshape(B * T, -1)[rows]
    # per-step checks on the sampled rows
    Qref = orc.linear(X2, w["W_q"], rows=rows)[rows]
    assert_parity(flat(Q), Qref, "Q rows")
    Gref = orc.linear(X2, w["W_g"], rows=rows)[rows]
    assert_parity(flat(G), Gref, "G rows")
    Call = orc.linear(X2, w["W_c"])                                  # every row: keys and values need them
    assert_parity(flat(C), Call[rows], "C rows")
    Kall = orc.linear(rb(Call), w["W_k"])
    Vall = orc.linear(rb(Call), w["W_v"])
    assert_parity(flat(K), Kall[rows], "K rows")
    assert_parity(flat(V), Vall[rows], "V rows")
    # chained: attention of the sampled rows over the oracle's own bf16-rounded K, V
    Qfull = np.zeros((B * T, d))
    Qfull[rows] = rb(Qref)
    trip = np.array([(r // T, h, r % T) for r in rows for h in range(H)], dtype=np.int64)
    Oh = orc.attention(Qfull.reshape(B, T, H, 128), rb(Kall).reshape(B, T, H, 128), rb(Vall).reshape(B, T, H, 128),
                       rows=trip)
    Og = rb(orc.gate(Oh.reshape(B * T, d)[rows], rb(Gref)))
    assert_parity(flat(O), Og, "gated context rows")
    Ofull = np.zeros((B * T, d))
    Ofull[rows] = Og
    assert_parity(flat(Y), orc.linear(Ofull, w["W_o"], rows=rows)[rows], "Y rows")


def test_layer_chained_matches_oracle(g):
    """X -> projections -> attention (+ gate) -> W_o, against the oracle that rounds
    to bfloat16 at the same library boundaries."""
    B, T, H, d_c = 2, 300, 3, 128
    d = 128 * H
    w, t = make_layer(17, B, T, d, d_c)
    Q = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    G, K, V, O, Y = (torch.empty_like(Q) for _ in range(5))
    C = torch.empty(B, T, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C, K=K, V=V)
    g.gmla_attend_prefill(Q.view(B, T, H, 128), K.view(B, T, H, 128), V.view(B, T, H, 128), O.view(B, T, H, 128),
                          G=G)
    g.gmla_gate_out(O, t["W_o"], Y)
    g.gmla_get_device_status()
    ref = orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H,
                        round_boundaries=True, intermediates=True)
    assert_parity(f64(C), ref["latent_cache"], "latent cache")
    assert_parity(f64(O), ref["O_gated"], "gated context")
    assert_parity(f64(Y), ref["output"], "Y")
    assert Y.shape == t["X"].shape and Y.dtype == t["X"].dtype


@pytest.mark.parametrize("T1,T2", [(300, 200), (128, 1), (1, 257)])
def test_chunked_prefill_matches_full_layer(g, T1, T2):
    """Two prefill chunks of the same sequences through the latent cache: the
    second chunk appends its latents at cache_pos = T1, re-expands K and V for
    rows 0..T1+T2-1 (gmla_expand_kv) and attends with Tq = T2 < Tk = T1 + T2.
    Its layer output equals rows T1.. of the oracle's full-sequence layer; the
    cache and the expanded K, V equal a single-pass run bit for bit."""
    B, H, d_c = 2, 2, 128
    T = T1 + T2
    d = 128 * H
    w, t = make_layer(29, B, T, d, d_c)
    C = torch.zeros(B, T, d_c, dtype=torch.bfloat16, device="cuda")
    Y2 = None
    for P, Tc in ((0, T1), (T1, T2)):
        Xc = t["X"][:, P:P + Tc].contiguous()
        Q = torch.empty(B, Tc, d, dtype=torch.bfloat16, device="cuda")
        G, O, Y = (torch.empty_like(Q) for _ in range(3))
        g.gmla_latent_project(Xc, t["W_q"], t["W_g"], t["W_c"], None, None, Q=Q, G=G, C=C, cache_pos=P)
        K = torch.empty(B, P + Tc, d, dtype=torch.bfloat16, device="cuda")
        V = torch.empty_like(K)
        g.gmla_expand_kv(C, 0, P + Tc, W_k=t["W_k"], W_v=t["W_v"], K=K, V=V)
        g.gmla_attend_prefill(Q.view(B, Tc, H, 128), K.view(B, P + Tc, H, 128), V.view(B, P + Tc, H, 128),
                              O.view(B, Tc, H, 128), G=G)
        g.gmla_gate_out(O, t["W_o"], Y)
        Y2 = Y
    g.gmla_get_device_status()
    ref = orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H,
                        round_boundaries=True)
    assert_parity(f64(Y2), ref["output"][:, T1:], "second chunk vs full-sequence layer")
    # single pass: same latents, and expansion of all rows equals the chunked run's last expansion
    C1 = torch.empty_like(C)
    K1 = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    V1 = torch.empty_like(K1)
    g.gmla_latent_project(t["X"], None, None, t["W_c"], t["W_k"], t["W_v"], C=C1, K=K1, V=V1)
    g.gmla_get_device_status()
    assert np.array_equal(bits(C), bits(C1))
    assert np.array_equal(bits(K), bits(K1)) and np.array_equal(bits(V), bits(V1))


def test_expand_kv_row_range(g):
    """gmla_expand_kv over an interior row range of a longer cache equals those rows
    of the full expansion."""
    B, Lmax, H, d_c = 3, 700, 2, 192
    d = 128 * H
    dr = Draw(31)
    cache = dr.normal((B, Lmax, d_c))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Cd, Wkd, Wvd = to_dev(cache), to_dev(Wk), to_dev(Wv)
    row0, rows = 133, 400
    K = torch.empty(B, rows, d, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    g.gmla_expand_kv(Cd, row0, rows, W_k=Wkd, W_v=Wvd, K=K, V=V)
    g.gmla_get_device_status()
    ref_k = orc.linear(cache[:, row0:row0 + rows], Wk)
    ref_v = orc.linear(cache[:, row0:row0 + rows], Wv)
    assert_parity(f64(K), ref_k, "expanded K")
    assert_parity(f64(V), ref_v, "expanded V")


@pytest.mark.parametrize("B,L,Lmax,H,d_c", [(3, 700, 700, 4, 128), (2, 1, 5, 2, 64), (1, 2049, 3000, 3, 512),
                                             (2, 4163, 4200, 96, 512), (1, 63, 64, 1, 512), (33, 500, 520, 5, 512),
                                             (70, 97, 100, 3, 192)])
def test_attend_decode_matches_oracle(g, B, L, Lmax, H, d_c):
    d = 128 * H
    dr = Draw(300 + L)
    q = dr.normal((B, d))
    cache = dr.normal((B, Lmax, d_c))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Gl = dr.normal((B, d))
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    W = torch.full((B, H, L), float("nan"), device="cuda")
    work = ws(g.gmla_attend_decode_workspace_size(B, L, H, d_c))
    g.gmla_attend_decode(to_dev(q), to_dev(cache), L, to_dev(Wk), to_dev(Wv), O, H, G=to_dev(Gl), weights=W,
                         workspace=work)
    g.gmla_get_device_status()
    ref, wref = orc.decode_latent(q, cache, L, Wk, Wv, H, G=Gl, want_weights=True)
    assert_parity(f64(O), ref, "decode O")
    w = f64(W)
    assert np.abs(w.sum(-1) - 1.0).max() <= ROW_SUM
    # q~ = W_k^T q is rounded to bfloat16 (relative 2^-9 per element), which moves a
    # unit-variance log2-domain score by ~1.6e-3 (1 sigma, d_c = 512); a weight moves
    # by ln2 * (ds_k - sum_j w_j ds_j), i.e. relatively, so the bound is relative:
    # ln2 * 2 * 7 sigma ~ 1e-2, plus an absolute floor for the float32 exp2.
    assert np.all(np.abs(w - wref) <= 2e-5 + 1e-2 * wref)


def test_attend_decode_ignores_unwritten_cache_rows(g):
    """Cache rows at or past L are never read as data: filled with NaN they
    leave the output equal to the oracle's on the L visible rows (a ragged
    last tile reads zeros there)."""
    B, L, Lmax, H, d_c = 2, 1000, 1100, 8, 512
    d = 128 * H
    dr = Draw(411)
    q = dr.normal((B, d))
    cache = dr.normal((B, Lmax, d_c))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    dirty = cache.copy()
    dirty[:, L:, :] = 0x7FC0  # bfloat16 quiet NaN
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    work = ws(g.gmla_attend_decode_workspace_size(B, L, H, d_c))
    g.gmla_attend_decode(to_dev(q), to_dev(dirty), L, to_dev(Wk), to_dev(Wv), O, H, workspace=work)
    g.gmla_get_device_status()
    ref = orc.decode_latent(q, np.ascontiguousarray(cache[:, :L]), L, Wk, Wv, H)
    got = f64(O)
    assert np.all(np.isfinite(got))
    assert_parity(got, ref, "decode with NaN past L")


def test_attend_decode_full_size_sampled(g):
    """Latent-cache decode at the timed size: B=32, L=131072, d_c=512, 96 heads;
    checked on sampled (b, h) pairs (the oracle rebuilds K_h, V_h from the cache)."""
    B, L, H, d_c = 32, 131072, 96, 512
    d = 128 * H
    dr = Draw(SEEDS["latent_decode"] + 100)
    q = dr.normal((B, d))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Gl = dr.normal((B, d))
    cache = dr.normal((B, L, d_c))
    Cd = to_dev(cache)
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    work = ws(g.gmla_attend_decode_workspace_size(B, L, H, d_c))
    g.gmla_attend_decode(to_dev(q), Cd, L, to_dev(Wk), to_dev(Wv), O, H, G=to_dev(Gl), workspace=work)
    g.gmla_get_device_status()
    pairs = [(0, 0), (31, 95), (7, 48), (19, 3)]
    ref = orc.decode_latent(q, cache, L, Wk, Wv, H, G=Gl, heads=pairs)
    got = f64(O)
    sel = np.concatenate([np.arange(h * 128, (h + 1) * 128) + b * d for b, h in pairs])
    assert_parity(got.reshape(-1)[sel], ref.reshape(-1)[sel], "decode full-size sampled heads")
    assert np.all(np.isfinite(got))


def test_decode_equals_prefill_last_row(g):
    """Decode of token t over latents 0..t equals row t of causal prefill (same GPU inputs)."""
    B, T, H, d_c = 1, 257, 2, 128
    d = 128 * H
    w, t = make_layer(23, B, T, d, d_c)
    Q = torch.empty(B, T, d, dtype=torch.bfloat16, device="cuda")
    G, K, V, O = (torch.empty_like(Q) for _ in range(4))
    C = torch.empty(B, T, d_c, dtype=torch.bfloat16, device="cuda")
    g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=Q, G=G, C=C, K=K, V=V)
    g.gmla_attend_prefill(Q.view(B, T, H, 128), K.view(B, T, H, 128), V.view(B, T, H, 128), O.view(B, T, H, 128),
                          G=G)
    Od = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    work = ws(g.gmla_attend_decode_workspace_size(B, T, H, d_c))
    g.gmla_attend_decode(Q[:, -1].contiguous(), C, T, t["W_k"], t["W_v"], Od, H, G=G[:, -1].contiguous(),
                         workspace=work)
    g.gmla_get_device_status()
    assert_parity(f64(Od), f64(O[:, -1]), "decode vs prefill row", rel_l2=1e-2)

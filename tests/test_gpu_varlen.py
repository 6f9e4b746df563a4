"""GPU parity of the per-sequence-length decode (gmla_attend_decode_varlen): the
two-dimensional padding mask of the "Kimi K2 - Construct causal mask" page in
length form, each sequence checked against the oracle on its own visible rows."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import Draw
from tests.gpu_util import ROW_SUM, assert_parity, bits, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import causal_head_latent_b200 as gm
    return gm


def _inputs(seed, B, Lmax, H, d_c):
    d = 128 * H
    dr = Draw(seed)
    q = dr.normal((B, d))
    cache = dr.normal((B, Lmax, d_c))
    Wk = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Wv = dr.normal((d, d_c), 1 / np.sqrt(d_c))
    Gl = dr.normal((B, d))
    return q, cache, Wk, Wv, Gl


def test_decode_varlen_matches_oracle_per_sequence(g):
    """Lengths 1, a partial tile, one tile, a multi-split length and the full cache;
    rows past each length hold NaN."""
    B, Lmax, H, d_c = 5, 4200, 8, 512
    lens = [1, 47, 48, 1000, 4200]
    d = 128 * H
    q, cache, Wk, Wv, Gl = _inputs(1201, B, Lmax, H, d_c)
    dirty = cache.copy()
    for b, n in enumerate(lens):
        dirty[b, n:, :] = 0x7FC0  # bfloat16 quiet NaN past the sequence's length
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    W = torch.full((B, H, Lmax), float("nan"), device="cuda")
    work = torch.empty(g.gmla_attend_decode_varlen_workspace_size(B, Lmax, H, d_c), dtype=torch.uint8, device="cuda")
    g.gmla_attend_decode_varlen(to_dev(q), to_dev(dirty), lens, to_dev(Wk), to_dev(Wv), O, H, G=to_dev(Gl),
                                weights=W, workspace=work)
    g.gmla_get_device_status()
    got, w = f64(O), f64(W)
    assert np.all(np.isfinite(got))
    for b, n in enumerate(lens):
        ref, wref = orc.decode_latent(q[b:b + 1], np.ascontiguousarray(cache[b:b + 1, :n]), n, Wk, Wv, H,
                                      G=Gl[b:b + 1], want_weights=True)
        assert_parity(got[b:b + 1], ref, f"varlen decode sequence {b} (length {n})")
        assert np.abs(w[b, :, :n].sum(-1) - 1.0).max() <= ROW_SUM
        assert np.all(w[b, :, n:] == 0.0)
        # relative bound: see test_attend_decode_matches_oracle (bfloat16 absorbed query)
        assert np.all(np.abs(w[b, :, :n] - wref[0]) <= 2e-5 + 1e-2 * wref[0])


def test_decode_varlen_equal_lengths_matches_oracle(g):
    """All lengths equal to cache_len_max: the work-item plan cuts the rows
    differently from gmla_attend_decode's split plan, and both match the oracle."""
    B, L, H, d_c = 3, 2049, 16, 512
    d = 128 * H
    q, cache, Wk, Wv, Gl = _inputs(1202, B, L, H, d_c)
    t = {k: to_dev(v) for k, v in (("q", q), ("C", cache), ("Wk", Wk), ("Wv", Wv), ("G", Gl))}
    O1 = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    O2 = torch.empty_like(O1)
    w1 = torch.empty(g.gmla_attend_decode_workspace_size(B, L, H, d_c), dtype=torch.uint8, device="cuda")
    w2 = torch.empty(g.gmla_attend_decode_varlen_workspace_size(B, L, H, d_c), dtype=torch.uint8, device="cuda")
    g.gmla_attend_decode(t["q"], t["C"], L, t["Wk"], t["Wv"], O1, H, G=t["G"], workspace=w1)
    g.gmla_attend_decode_varlen(t["q"], t["C"], [L] * B, t["Wk"], t["Wv"], O2, H, G=t["G"], workspace=w2)
    g.gmla_get_device_status()
    ref = orc.decode_latent(q, cache, L, Wk, Wv, H, G=Gl)
    assert_parity(f64(O1), ref, "uniform decode, equal lengths")
    assert_parity(f64(O2), ref, "varlen decode, equal lengths")


def test_decode_varlen_skewed_lengths_many_items(g):
    """One long sequence next to short ones: the long one is cut into dozens of
    work items whose states sit in records past B and are merged through the
    per-sequence record offsets; a 1-row and a sub-tile sequence keep one item."""
    B, Lmax, H, d_c = 4, 6000, 4, 512
    lens = [6000, 1, 130, 2500]
    d = 128 * H
    q, cache, Wk, Wv, Gl = _inputs(1204, B, Lmax, H, d_c)
    dirty = cache.copy()
    for b, n in enumerate(lens):
        dirty[b, n:, :] = 0x7FC0
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    W = torch.full((B, H, Lmax), float("nan"), device="cuda")
    work = torch.empty(g.gmla_attend_decode_varlen_workspace_size(B, Lmax, H, d_c), dtype=torch.uint8, device="cuda")
    g.gmla_attend_decode_varlen(to_dev(q), to_dev(dirty), lens, to_dev(Wk), to_dev(Wv), O, H, G=to_dev(Gl),
                                weights=W, workspace=work)
    g.gmla_get_device_status()
    got, w = f64(O), f64(W)
    for b, n in enumerate(lens):
        ref = orc.decode_latent(q[b:b + 1], np.ascontiguousarray(cache[b:b + 1, :n]), n, Wk, Wv, H, G=Gl[b:b + 1])
        assert_parity(got[b:b + 1], ref, f"skewed varlen decode sequence {b} (length {n})")
        assert np.abs(w[b, :, :n].sum(-1) - 1.0).max() <= ROW_SUM
        assert np.all(w[b, :, n:] == 0.0)


def test_decode_varlen_full_size_sampled(g):
    """B=32 sequences of mixed lengths up to 131072 cached latents, 96 heads, d_c=512,
    checked on sampled (b, h) pairs."""
    B, Lmax, H, d_c = 32, 131072, 96, 512
    d = 128 * H
    rng = np.random.default_rng(1203)
    lens = [int(x) for x in rng.integers(1, Lmax + 1, B)]
    lens[3], lens[17] = 1, Lmax
    q, cache, Wk, Wv, Gl = _inputs(1203, B, Lmax, H, d_c)
    O = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    work = torch.empty(g.gmla_attend_decode_varlen_workspace_size(B, Lmax, H, d_c), dtype=torch.uint8, device="cuda")
    g.gmla_attend_decode_varlen(to_dev(q), to_dev(cache), lens, to_dev(Wk), to_dev(Wv), O, H, G=to_dev(Gl),
                                workspace=work)
    g.gmla_get_device_status()
    got = f64(O)
    assert np.all(np.isfinite(got))
    for b, h in [(3, 0), (17, 95), (8, 40)]:
        n = lens[b]
        ref = orc.decode_latent(q[b:b + 1], np.ascontiguousarray(cache[b:b + 1, :n]), n, Wk, Wv, H, G=Gl[b:b + 1],
                                heads=[(0, h)])
        sl = slice(h * 128, (h + 1) * 128)
        assert_parity(got[b, sl], ref[0, sl], f"varlen full-size b={b} h={h} length {n}")


def _prefill_varlen_inputs(seed, B, Tq, Tk, H, q_lens, kv_lens):
    from synth_inputs import prefill_qkv
    inp = prefill_qkv(seed, B, Tq, H, Tk=Tk, gate=True)
    dirty = {k: v.copy() for k, v in inp.items()}
    for b in range(B):
        dirty["Q"][b, q_lens[b]:] = 0x7FC0  # bfloat16 quiet NaN in the padding
        dirty["K"][b, kv_lens[b]:] = 0x7FC0
        dirty["V"][b, kv_lens[b]:] = 0x7FC0
    return inp, dirty


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_varlen_matches_oracle_per_sequence(g, causal):
    """Padded prefill batch: a full square sequence, an empty one, a 37-row chunk
    continuing 483 cached keys, a single tile, and a 1-row chunk over 257 keys.
    NaN padding; output and lse rows past each q_len stay untouched."""
    B, H, Tq, Tk = 5, 2, 300, 520
    q_lens = [300, 0, 37, 129, 1]
    kv_lens = [300, 5, 520, 129, 257]
    inp, dirty = _prefill_varlen_inputs(1301, B, Tq, Tk, H, q_lens, kv_lens)
    Q, K, V, G = (to_dev(dirty[k]) for k in ("Q", "K", "V", "G"))
    sentinel = 0x1234
    O = torch.from_numpy(np.full((B, Tq, H, 128), sentinel, dtype=np.int16)).view(torch.bfloat16).cuda()
    lse = torch.full((B, H, Tq), float("nan"), device="cuda")
    work = torch.empty(g.gmla_attend_prefill_varlen_workspace_size(B), dtype=torch.uint8, device="cuda")
    g.gmla_attend_prefill_varlen(Q, K, V, O, q_lens, kv_lens, causal=causal, G=G, lse=lse, workspace=work)
    g.gmla_get_device_status()
    got, ob, lg = f64(O), bits(O), f64(lse)
    for b in range(B):
        q, kv = q_lens[b], kv_lens[b]
        assert np.all(ob[b, q:] == sentinel), f"sequence {b}: padded output rows were written"
        assert np.all(np.isnan(lg[b, :, q:]))
        if q == 0:
            continue
        ref, lref = orc.attention(inp["Q"][b:b + 1, :q], inp["K"][b:b + 1, :kv], inp["V"][b:b + 1, :kv],
                                  causal=causal, want_lse=True)
        ref = orc.gate(ref.reshape(1, q, -1), inp["G"][b:b + 1, :q]).reshape(ref.shape)
        assert_parity(got[b:b + 1, :q], ref, f"varlen prefill sequence {b} (q={q}, kv={kv})")
        np.testing.assert_allclose(lg[b:b + 1, :, :q], lref, atol=5e-4)


def test_prefill_varlen_equal_lengths_equals_uniform(g):
    """All lengths at their maxima: the same kernel as gmla_attend_prefill reading the
    same data through per-sequence maps, so the outputs match bit for bit."""
    B, H, Tq, Tk = 2, 3, 300, 333
    from synth_inputs import prefill_qkv
    inp = prefill_qkv(1302, B, Tq, H, Tk=Tk, gate=True)
    Q, K, V, G = (to_dev(inp[k]) for k in ("Q", "K", "V", "G"))
    O1, O2 = torch.empty_like(Q), torch.empty_like(Q)
    g.gmla_attend_prefill(Q, K, V, O1, G=G)
    work = torch.empty(g.gmla_attend_prefill_varlen_workspace_size(B), dtype=torch.uint8, device="cuda")
    g.gmla_attend_prefill_varlen(Q, K, V, O2, [Tq] * B, [Tk] * B, G=G, workspace=work)
    g.gmla_get_device_status()
    assert np.array_equal(bits(O1), bits(O2))


def test_prefill_varlen_large_sampled(g):
    """Mixed lengths up to 8192 (a full square sequence, a 1000-row chunk over 8192
    keys, a 4096-row chunk over 6000 keys), sampled rows per sequence and head."""
    B, H, Tq, Tk = 3, 4, 8192, 8192
    q_lens, kv_lens = [8192, 1000, 4096], [8192, 8192, 6000]
    inp, dirty = _prefill_varlen_inputs(1303, B, Tq, Tk, H, q_lens, kv_lens)
    Q, K, V = (to_dev(dirty[k]) for k in ("Q", "K", "V"))
    O = torch.zeros_like(Q)
    work = torch.empty(g.gmla_attend_prefill_varlen_workspace_size(B), dtype=torch.uint8, device="cuda")
    g.gmla_attend_prefill_varlen(Q, K, V, O, q_lens, kv_lens, workspace=work)
    g.gmla_get_device_status()
    got = f64(O)
    rng = np.random.default_rng(1303)
    for b in range(B):
        q, kv = q_lens[b], kv_lens[b]
        ts = sorted(set([0, 1, 127, 128, q // 2, q - 1] + list(rng.integers(0, q, 4))))
        for h in (0, H - 1):
            sl = lambda k, n: inp[k][b:b + 1, :n, h:h + 1]
            ref = orc.attention(sl("Q", q), sl("K", kv), sl("V", kv), rows=[(0, 0, t) for t in ts])
            assert_parity(np.stack([got[b, t, h] for t in ts]), np.stack([ref[0, t, 0] for t in ts]),
                          f"varlen prefill b={b} h={h}")
    assert np.all(np.isfinite(got))

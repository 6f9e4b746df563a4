"""Multi-GPU host logic on the CPU, as two or three gloo ranks.

* Context-parallel decode (causal_head_latent_b200.cp): the key slices cover the
  cache once on tile edges; each rank's state reaches the merge at its rank's
  position of the all-gather; merged, the states give the oracle's decode over
  all rows.
* Head-parallel prefill (causal_head_latent_b200.tp): the head ranges cover the
  heads once; the ranks' shares of the output projection, summed by the
  all-reduce (or reduce-scattered over token rows), give the oracle's layer.

The per-rank arithmetic here is a float64 reference with the contract of the
library call it stands in for (the GPU calls themselves are checked on one GPU
in tests/test_gpu_parallel.py); what these tests exercise is the plan and the
exchange.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as orc
from causal_head_latent_b200.cp import key_slices, owner_of_row
from causal_head_latent_b200.tp import head_slices
from synth_inputs import Draw, layer_weights

D = 128


def test_key_slices_cover_the_cache_once_on_tile_edges():
    for L in (0, 1, 47, 48, 49, 1000, 131072, 131073):
        for world in (1, 2, 3, 8):
            sl = key_slices(L, world)
            assert len(sl) == world
            rows = [i for k0, k1 in sl for i in range(k0, k1)]
            assert rows == list(range(L))
            for k0, k1 in sl:
                assert (k0 % 48 == 0 or k0 == k1 == L) and (k1 % 48 == 0 or k1 == L)
            tiles = [math.ceil((k1 - k0) / 48) for k0, k1 in sl]
            assert max(tiles) - min(tiles) <= 1
            if L:
                k0, k1 = sl[owner_of_row(L, world, L - 1)]
                assert k0 <= L - 1 < k1


def test_head_slices_cover_the_heads_once():
    for H in (1, 2, 5, 96):
        for world in range(1, min(H, 8) + 1):
            sl = head_slices(H, world)
            assert [h for a, b in sl for h in range(a, b)] == list(range(H))
            assert max(b - a for a, b in sl) - min(b - a for a, b in sl) <= 1
    with pytest.raises(ValueError):
        head_slices(2, 3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _decode_problem():
    B, L, H, d_c = 2, 300, 3, 64
    dr = Draw(61)
    x = {"q": dr.normal((B, H * D)), "cache": dr.normal((B, L, d_c)), "Wk": dr.normal((H * D, d_c), 1 / np.sqrt(d_c)),
         "Wv": dr.normal((H * D, d_c), 1 / np.sqrt(d_c)), "G": dr.normal((B, H * D))}
    return B, L, H, d_c, x


def _state_ref(x, H, k0, k1):
    """float64 state over cached rows [k0, k1): the contract of gmla_attend_decode_partial."""
    B = x["q"].shape[0]
    d_c = x["cache"].shape[-1]
    lse = np.full((B, H), -np.inf)
    ctx = np.zeros((B, H, d_c))
    if k1 == k0:
        return lse, ctx
    for b in range(B):
        cb = orc.widen(np.ascontiguousarray(x["cache"][b, k0:k1]))
        for h in range(H):
            Kh = orc.linear(cb, x["Wk"][h * D:(h + 1) * D])
            qh = orc.widen(x["q"][b, h * D:(h + 1) * D]).reshape(1, 1, 1, D)
            n = k1 - k0
            _, w, l = orc.attention(qh, Kh.reshape(1, n, 1, D), Kh.reshape(1, n, 1, D), want_weights=True,
                                    want_lse=True)
            lse[b, h] = l[0, 0, 0]
            ctx[b, h] = w[0, 0, 0] @ cb
    return lse, ctx


def _combine_ref(lse_all, ctx_all, Wv, G, H):
    """float64 merge: the contract of gmla_decode_combine."""
    m = lse_all.max(0)
    w = np.exp(lse_all - m)
    w /= w.sum(0)
    chat = (w[..., None] * ctx_all).sum(0)                       # [B, H, d_c]
    Wv = orc.widen(Wv)
    o = np.stack([np.stack([orc.linear(chat[b, h][None], Wv[h * D:(h + 1) * D])[0] for h in range(H)])
                  for b in range(chat.shape[0])]).reshape(chat.shape[0], H * D)
    return orc.gate(o, G)


def _cp_worker(rank, world, port, out):
    import torch.distributed as dist

    from causal_head_latent_b200.cp import ContextParallelDecode
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, L, H, d_c, x = _decode_problem()
        k0, k1 = key_slices(L, world)[rank]
        C_local = x["cache"][:, k0:k1]          # this rank's rows only

        def partial(Q, C_loc, n_rows, W_k, lse, ctx):
            assert n_rows == C_loc.shape[1] == k1 - k0
            lo, c = _state_ref({"q": Q, "cache": C_loc, "Wk": W_k}, H, 0, n_rows)
            lse.copy_(torch.from_numpy(lo))
            ctx.copy_(torch.from_numpy(c))

        seen = {}

        def combine(lse_all, ctx_all, W_v, G, O):
            seen["lse"] = lse_all.numpy().copy()
            O[...] = torch.from_numpy(_combine_ref(lse_all.numpy(), ctx_all.numpy(), W_v, G, H))

        cp = ContextParallelDecode(B, H, d_c, device="cpu", partial=partial, combine=combine)
        assert cp.slice(L) == (k0, k1)
        O = torch.empty(B, H * D, dtype=torch.float64)
        cp.step(x["q"], C_local, L, x["Wk"], x["Wv"], O, G=x["G"])
        out.put((rank, O.numpy(), seen["lse"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, L, H, d_c, x = _decode_problem()
    ref = orc.decode_latent(x["q"], x["cache"], L, x["Wk"], x["Wv"], H, G=x["G"])
    slices = key_slices(L, world)
    for rank, O, lse_all in res:
        np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)
        for r, (k0, k1) in enumerate(slices):   # state r of the gather is rank r's slice
            np.testing.assert_allclose(lse_all[r], _state_ref(x, H, k0, k1)[0], rtol=1e-12, atol=1e-12)


def _layer_problem():
    B, T, H, d_c = 2, 6, 3, 16
    w = layer_weights(Draw(62), H * D, d_c, x_shape=(B, T, H * D))
    return B, T, H, d_c, w


def _share_ref(X, W, h0, h1):
    """float64 share of heads [h0, h1): the contract of the GPU share (project the
    range's heads, attend with the gate, the range's columns of W_o)."""
    B, T, d = X.shape
    r = slice(128 * h0, 128 * h1)
    C = orc.linear(X, W["W_c"])
    Q = orc.linear(X, orc.widen(W["W_q"])[r])
    G = orc.linear(X, orc.widen(W["W_g"])[r])
    K = orc.linear(C, orc.widen(W["W_k"])[r])
    V = orc.linear(C, orc.widen(W["W_v"])[r])
    n = h1 - h0
    O = orc.attention(Q.reshape(B, T, n, D), K.reshape(B, T, n, D), V.reshape(B, T, n, D)).reshape(B, T, n * D)
    Y = orc.linear(orc.gate(O, G), orc.widen(W["W_o"])[:, r])
    return torch.from_numpy(C), torch.from_numpy(np.ascontiguousarray(Y))


def _tp_worker(rank, world, port, mode, out):
    import torch.distributed as dist

    from causal_head_latent_b200.tp import HeadParallelPrefill
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, T, H, d_c, w = _layer_problem()
        tp = HeadParallelPrefill(H, share=_share_ref)
        assert (tp.h0, tp.h1) == head_slices(H, world)[rank]
        C, Y = tp.forward(w["X"], w, mode=mode)
        out.put((rank, C.numpy(), Y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mode", [(2, "all"), (3, "all"), (2, "rows")])
def test_head_parallel_prefill_over_gloo_ranks(world, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, T, H, d_c, w = _layer_problem()
    ref = orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], H)
    Yref = ref["output"].reshape(B * T, H * D)
    rows = B * T // world
    for rank, C, Y in res:
        np.testing.assert_allclose(C, ref["latent_cache"], rtol=0, atol=0)
        if mode == "all":
            np.testing.assert_allclose(Y.reshape(B * T, -1), Yref, rtol=1e-10, atol=1e-12)
        else:
            np.testing.assert_allclose(Y, Yref[rank * rows:(rank + 1) * rows], rtol=1e-10, atol=1e-12)

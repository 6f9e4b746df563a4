"""Data-parallel host logic on CPU: sequence sharding and the slowest-rank timing
reduction, run as two gloo ranks.  The sharded oracle results must equal the
unsharded ones exactly (sequences are independent)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from causal_head_latent_b200.dp import max_over_ranks, shard_range, sum_over_ranks


def test_shard_range_covers_everything_once():
    for n in (0, 1, 5, 32, 33):
        for world in (1, 2, 3, 8):
            got = [shard_range(n, r, world) for r in range(world)]
            items = [i for b, e in got for i in range(b, e)]
            assert items == list(range(n))
            sizes = [e - b for b, e in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import oracle as orc
    from synth_inputs import Draw, layer_weights
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = layer_weights(Draw(42), 16, 8, x_shape=(5, 4, 16), bf16=False)
        b0, b1 = shard_range(5, rank, world)
        r = orc.gated_mla(w["X"][b0:b1], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], 2)
        slowest = max_over_ranks(float(rank + 1) * 10.0)
        total = sum_over_ranks(float(b1 - b0))
        out.put((rank, b0, b1, r["output"], slowest, total))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle as orc
    from synth_inputs import Draw, layer_weights
    w = layer_weights(Draw(42), 16, 8, x_shape=(5, 4, 16), bf16=False)
    full = orc.gated_mla(w["X"], w["W_q"], w["W_c"], w["W_k"], w["W_v"], w["W_g"], w["W_o"], 2)["output"]
    for rank, b0, b1, y, slowest, total in res:
        assert slowest == 20.0 and total == 5.0
        np.testing.assert_array_equal(y, full[b0:b1])

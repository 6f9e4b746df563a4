"""Head-parallel (tensor-parallel) prefill of one Gated MLA layer.

The heads are independent until the output projection ("Gated MLA" page,
"Split attention into heads": heads are joined by concatenation, then gated
channel by channel and projected by W_o).  Rank r of N takes a contiguous
range of heads: it projects only those heads' queries, gate logits, keys and
values (rows of W_q, W_g, W_k, W_v; the latent C is shared by every head and
computed in full on every rank), attends over them, and multiplies its gated
context by the matching columns of W_o (gmla_gate_out_heads).  W_o mixes all
channels, so the layer output is the SUM of the ranks' shares: one reduction
(all-reduce, or reduce-scatter over token rows) of Y [B*T, d_model] is the only
exchange.

Host plumbing only: the arithmetic runs in the library's kernels, the
reduction in torch.distributed (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations


def head_slices(H: int, world: int) -> list[tuple[int, int]]:
    """Contiguous head ranges [h0, h1), one per rank in rank order, covering every
    head once; sizes differ by at most one head.  world must not exceed H."""
    if world <= 0 or H < world:
        raise ValueError("need at least one head per rank")
    base, extra = divmod(H, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def reduce_shares(Y_share, mode="all", out=None, group=None):
    """Sum the ranks' shares of the layer output.  mode "all": all-reduce in
    place, every rank gets Y.  mode "rows": reduce-scatter over token rows
    (dim 0 of the [M, d_model] share, M a multiple of the world size) into
    `out` [M / world, d_model]: rank r gets rows r*M/world ...."""
    import torch.distributed as dist
    if mode == "all":
        dist.all_reduce(Y_share, group=group)
        return Y_share
    if mode == "rows":
        dist.reduce_scatter_tensor(out, Y_share.contiguous(), group=group)
        return out
    raise ValueError(mode)


class HeadParallelPrefill:
    """Prefill of one layer with the heads split over the ranks of `group` by
    head_slices(H, world).

    forward(X, W) with X [B, T, d_model] (the same on every rank) and the FULL
    weights W = {W_q, W_g, W_c, W_k, W_v, W_o} returns this rank's latent cache
    C [B, T, d_c] (identical on every rank) and the layer output Y [B, T,
    d_model] after the reduction.

    `share` defaults to the library calls (gmla_latent_project_heads,
    gmla_attend_prefill with the gate, gmla_gate_out_heads); the CPU tests pass
    a float64 reference with the same contract to check the head plan and the
    reduction without a GPU.
    """

    def __init__(self, H, group=None, share=None):
        import torch.distributed as dist
        self.H, self.group = int(H), group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.h0, self.h1 = head_slices(self.H, self.world)[self.rank]
        self.share = share or self._share_gpu

    def _share_gpu(self, X, W, h0, h1):
        import torch

        from . import gmla_attend_prefill, gmla_gate_out_heads, gmla_latent_project_heads
        B, T, d = X.shape
        d_c = W["W_c"].shape[0]
        wr = 128 * (h1 - h0)
        Q, G, K, V, O = (torch.empty(B, T, wr, dtype=X.dtype, device=X.device) for _ in range(5))
        C = torch.empty(B, T, d_c, dtype=X.dtype, device=X.device)
        gmla_latent_project_heads(X, h0, h1, W["W_q"], W["W_g"], W["W_c"], W["W_k"], W["W_v"], Q=Q, G=G, C=C, K=K,
                                  V=V)
        v4 = lambda z: z.view(B, T, h1 - h0, 128)
        gmla_attend_prefill(v4(Q), v4(K), v4(V), v4(O), G=G)
        Y = torch.empty(B, T, d, dtype=X.dtype, device=X.device)
        gmla_gate_out_heads(O, W["W_o"], Y, h0, h1)
        return C, Y

    def forward(self, X, W, mode="all"):
        C, Y = self.share(X, W, self.h0, self.h1)
        B, T, d = Y.shape
        if mode == "all":
            reduce_shares(Y.view(B * T, d), "all", group=self.group)
            return C, Y
        out = Y.new_empty(B * T // self.world, d)
        return C, reduce_shares(Y.view(B * T, d), "rows", out=out, group=self.group)

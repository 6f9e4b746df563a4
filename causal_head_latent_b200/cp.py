"""Context-parallel decode: the latent cache of every sequence split along its
length over several GPUs.

Why: the decode reads every cached latent once per new token, and at long
context the cache dominates ("Le Transformer et l'attention" page, the cost
table: the cache of a 1M-token context is 128 times that of 8K).  Splitting the
rows of the cache over N GPUs divides both the memory and the per-token read
by N.  The softmax over keys ("Kimi K3 - Softmax over keys") does not split
naively, but its log-sum-exp form does: each GPU computes, for its rows only,
the normalised latent context and its log-sum-exp
(gmla_attend_decode_partial); one all-gather brings every GPU the N states;
gmla_decode_combine merges them exactly and applies W_v and the gate.

The exchange per token is one all-gather of B*H*(d_c + 1) float32 values per
GPU (6.3 MB at B=32, 96 heads, d_c=512) against a cache slice of B*L/N*d_c*2
bytes read locally.  Decode is not split by heads: every head reads the same
latents, so a head split would read the whole cache on every GPU.

Host plumbing only: the arithmetic runs in the library's kernels, the
exchange in torch.distributed (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

TILE_KEYS = 48  # keys per tile of the decode kernel: slice edges on tile edges keep every tile whole


def key_slices(L: int, world: int, tile: int = TILE_KEYS) -> list[tuple[int, int]]:
    """Contiguous slices [k0, k1) of the L cached rows, one per rank in rank order:
    they cover every row exactly once, their edges fall on multiples of `tile`
    (except the end, L), and their sizes differ by at most one tile.  Ranks past
    the last tile get an empty slice."""
    if world <= 0 or L < 0 or tile <= 0:
        raise ValueError("bad slice request")
    tiles = (L + tile - 1) // tile
    base, extra = divmod(tiles, world)
    out, t = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        k0, k1 = min(t * tile, L), min((t + n) * tile, L)
        out.append((k0, k1))
        t += n
    return out


def owner_of_row(L: int, world: int, row: int, tile: int = TILE_KEYS) -> int:
    """Rank whose slice holds cached row `row` (where a new token's latent goes)."""
    for r, (k0, k1) in enumerate(key_slices(L, world, tile)):
        if k0 <= row < k1:
            return r
    raise ValueError("row outside the cache")


def gather_states(lse, ctx, lse_all, ctx_all, group=None):
    """All-gather this rank's decode state (lse [B, H], ctx [B, H, d_c]) into
    lse_all [world, B, H] and ctx_all [world, B, H, d_c], stacked in rank order
    (the layout gmla_decode_combine reads).  The buffers are written through
    flat views, so the gather needs no copy afterwards."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(lse_all.view(-1, *lse.shape[1:]), lse.contiguous(), group=group)
    dist.all_gather_into_tensor(ctx_all.view(-1, *ctx.shape[1:]), ctx.contiguous(), group=group)
    return lse_all, ctx_all


class ContextParallelDecode:
    """One decode step of a Gated MLA layer whose latent cache is split over the
    ranks of `group` by key_slices(L, world).

    This rank holds rows [k0, k1) of every sequence in its own cache buffer
    C_local [B, rows_max, d_c] (local row i = global row k0 + i).  step() takes
    the new tokens' queries Q [B, H*128] (identical on every rank; the rank that
    owns row L-1 has already appended the new latent there), computes this
    rank's state, exchanges the states and returns O [B, H*128] = the gated
    head contexts, the same on every rank.

    `partial` and `combine` default to the library calls; the CPU tests pass
    float64 reference functions with the same contract to check the slicing and
    the exchange without a GPU.
    """

    def __init__(self, B, H, d_c, group=None, device=None, partial=None, combine=None):
        import torch
        import torch.distributed as dist
        self.B, self.H, self.d_c, self.group = int(B), int(H), int(d_c), group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.device = device
        self.partial = partial or self._partial_gpu
        self.combine = combine or self._combine_gpu
        f = torch.float32 if device is None or str(device).startswith("cuda") else torch.float64
        self.dtype = f
        self.lse = torch.empty(self.B, self.H, dtype=f, device=device)
        self.ctx = torch.empty(self.B, self.H, self.d_c, dtype=f, device=device)
        self.lse_all = torch.empty(self.world, self.B, self.H, dtype=f, device=device)
        self.ctx_all = torch.empty(self.world, self.B, self.H, self.d_c, dtype=f, device=device)
        self._ws = None

    def slice(self, L):
        return key_slices(L, self.world)[self.rank]

    def _partial_gpu(self, Q, C_local, n_rows, W_k, lse, ctx):
        import torch

        from . import gmla_attend_decode_partial, gmla_attend_decode_partial_workspace_size
        need = gmla_attend_decode_partial_workspace_size(self.B, 0, n_rows, self.H, self.d_c)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
        gmla_attend_decode_partial(Q, C_local, 0, n_rows, W_k, lse, ctx, self.H, workspace=self._ws)

    def _combine_gpu(self, lse_all, ctx_all, W_v, G, O):
        from . import gmla_decode_combine
        gmla_decode_combine(lse_all, ctx_all, W_v, O, G=G)

    def step(self, Q, C_local, L, W_k, W_v, O, G=None):
        k0, k1 = self.slice(L)
        self.partial(Q, C_local, k1 - k0, W_k, self.lse, self.ctx)
        gather_states(self.lse, self.ctx, self.lse_all, self.ctx_all, self.group)
        self.combine(self.lse_all, self.ctx_all, W_v, G, O)
        return O

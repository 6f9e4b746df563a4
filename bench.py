"""Benchmark of the Gated MLA hot path on B200.

One step = one pass of the whole hot path, every step of the method, over one
synthetic batch of each workload shape:
  prefill  causal attention, B=1, 96 heads, T=8192, D_h=128 (gmla_attend_prefill)
  decode   one new token for B=32 sequences over L=131072 cached latents of width
           512: projections of the new token with the latent appended at row
           L-1 (gmla_latent_project), absorbed attention over the latent cache
           with log-sum-exp combine and gate (gmla_attend_decode), W_o
           (gmla_gate_out); d_model = 12288.
  plain    decode attention over explicit K, V in the "Softmax over keys" page's
           shape: B=8, 96 heads, one query, 1001 keys (gmla_attend_prefill, Tq=1)
  layer    the full layer prefill, B=2, T=4096, d_model=12288, d_c=512:
           projections with K/V expansion, gated causal attention, W_o.
Headline value: prefill attention TFLOP/s (causal pairs only:
4*D_h*H*B*T(T+1)/2 flop).  The decode half of the metric -- latent-cache GB/s
of gmla_attend_decode -- is reported in the "decode" object, the other two
workloads in "decode_plain" and "layer".  Every input but the plain decode's
is larger than L2 (Q/K/V 604 MB, cache 4.3 GB, layer weights 0.9 GB); the
plain decode (394 MB) runs after the others, which evict it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--parts all|prefill|decode|plain|layer] [--workload step|layer|sweep|varlen]

With --gpus N > 1 (launched by torch.distributed.run) every rank runs the same
per-GPU workload (data-parallel replicas, no collective on the data path);
value is the total over ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attention TFLOP/s & decode latent-cache GB/s, % of B200 roofline"

# workload sizes
P_B, P_H, P_T, D = 1, 96, 8192, 128
DEC_B, DEC_L, DC, DM = 32, 131072, 512, 12288
L_B, L_T = 2, 4096   # --workload layer: full layer prefill
# --workload sweep: context lengths of the "Foundations" page's cost table (8K, 128K, 1M);
# prefill at B=1 with SWEEP_H heads (the per-head cost is what scales), decode at B=SWEEP_B
SWEEP_T = (8192, 131072, 1048576)
SWEEP_H = 8
SWEEP_B = 4
SWEEP_PAGE = {"dot_products_per_head": (3.2e7, 8.2e9, 5.2e11), "kv_cache": (1, 16, 128)}
# --workload varlen: a padded prefill batch of chunks continuing differently cached sequences
# (per-sequence query / key lengths) and a decode batch with per-sequence cache lengths
VL_H = 32
VL_Q = (8192, 4096, 2048, 1024, 8192, 512, 3000, 100)
VL_KV = (8192, 8192, 6000, 1024, 8192, 4096, 3000, 5000)
VL_DEC_B, VL_DEC_LMAX = 32, 131072


PL_B, PL_TK = 8, 1001  # plain decode over explicit K, V (the "Softmax over keys" page, p = 1000)


def plain_decode_bytes(B=PL_B, H=96, Tk=PL_TK):
    # Q, K, V and O of gmla_attend_prefill with one query
    return 2.0 * B * H * D * (2 * Tk + 2)


def prefill_flops(B=P_B, H=P_H, T=P_T):
    return 4.0 * D * H * B * T * (T + 1) / 2


def decode_bytes(B=None, L=None, H=96, dc=DC):
    # algorithmic bytes of gmla_attend_decode: the visible latents, W_k, W_v, q, G and O
    B = DEC_B if B is None else B
    L = DEC_L if L is None else L
    d = H * D
    return 2.0 * (B * L * dc + 2 * d * dc + 3 * B * d)


def decode_step_bytes(B=None, L=None, dc=DC, dm=DM):
    # whole decode step: attend_decode plus W_q, W_g, W_c, W_o and the new-token activations
    B = DEC_B if B is None else B
    return decode_bytes(B, L, dm // D, dc) + 2.0 * (3 * dm * dm + dc * dm + 4 * B * dm + B * dc)


def layer_flops(B=L_B, T=L_T, d=DM, dc=DC):
    M = B * T
    return 2.0 * M * d * (2 * d + dc) + 2.0 * M * dc * 2 * d + prefill_flops(B, d // D, T) + 2.0 * M * d * d


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the dominant kernels,
# from one ncu capture each (profiles/).  Reported only while the kernel sources are the ones that
# were captured (sha1 over the code of the listed files, in order, comments and whitespace left
# out); any change of the code makes it null until the next capture.
PROFILED_TRAFFIC = {
    "attn_prefill_kernel": {"sources": ["attn_prefill.cu", "launch_plan.h"], "sha1": "a98378f246e60ba619fae741d7af6d76b1f88f43",
                            "bytes": 620.145152e6 + 188.867072e6,
                            "how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch at the timed size "
                                   "(B=1 H=96 T=8192)"},
    "gmla_attend_decode": {"sources": ["attn_latent.cu", "attn_latent_tc.cu", "attn_latent_side.cu"],
                           "sha1": "9f2cf61be9e22857aafd74a04684d4d91b9d9c41",
                           "bytes": (540.408320e6 - 536.870912e6 + 8 * 536.870912e6) + 29.337088e6 + 13.393664e6
                                    + 56.872192e6 + 19.722240e6,
                           "how": "ncu dram bytes of the four kernels of one call at L=16384 (absorb, stream, merge, "
                                  "W_v); the stream kernel's cache reads (B*L*1 KB) scaled x8 to L=131072, the rest "
                                  "(q~, partial states, W_k, W_v) unscaled"},
    # decode over explicit K/V (B=8, H=96, Tk=1001): one launch at the timed size
    "attn_rows_kernel": {"sources": ["attn_rows.cu"], "sha1": "7914ef626f5b25e912d0e76e039b93074b41d327",
                         "bytes": 393.975296e6 + 3.392e6,
                         "how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch at the timed size"},
    # layer prefill: the [Q | G | C] projection, the layer's longest launch
    "gemm_kernel": {"sources": ["gemm.cu", "launch_plan.h"], "sha1": "517f893587a228afcaa3734593b18f69703d6164",
                    "bytes": 4931.942144e6 + 406.335488e6,
                    "how": "ncu dram bytes of the [Q|G|C] projection launch of the B=2 T=4096 layer"},
}


def code_only(text):
    """C++/CUDA source with its comments removed and whitespace collapsed, so that
    an edit of a comment does not count as a change of the kernel (string and
    character literals, inline PTX included, are kept verbatim)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif text[i] in "\"'":
            q, j = text[i], i + 1
            while j < n and text[j] != q:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return " ".join("".join(out).split())


def sources_sha1(files):
    """sha1 of the code of the listed csrc files (comments and whitespace left out)."""
    import hashlib
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "causal_head_latent_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode("utf-8"))
    return h.hexdigest()


def profiled_traffic(kernel):
    ent = PROFILED_TRAFFIC.get(kernel)
    if not ent or ent["bytes"] is None or ent["sha1"] is None:
        return None, "no ncu capture of the current source"
    if sources_sha1(ent["sources"]) != ent["sha1"]:
        return None, "kernel changed since the ncu capture"
    return ent["bytes"], ent["how"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples every 50 ms, each with the host
    time it was taken, so that a summary can be cut for any timed region."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.samples = []  # (host time, sm MHz, max MHz, set of active reasons)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        import datetime
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                t = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(f[2]), float(f[3])
            except ValueError:
                continue
            self.samples.append((t, sm, mx, {n for n, v in zip(self.NAMES, f[6:10]) if v.lower().startswith("active")}))

    def summary(self, t0=None, t1=None):
        """Median SM clock, max clock and active reasons of the samples in [t0, t1]
        (host time); a region shorter than the sampling period takes the samples
        nearest to it."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sel = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not sel and self.samples and t0 is not None:
            mid = 0.5 * (t0 + t1)
            near = sorted(self.samples, key=lambda x: abs(x[0] - mid))[:2]
            sel = [x for x in near if abs(x[0] - mid) < 0.2]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(x[1] for x in sel), "sm_max_mhz": max(x[2] for x in sel),
                "reasons": sorted(set().union(*(x[3] for x in sel))), "samples": len(sel)}


# ------------------------------------------------------------------ distributed plumbing


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n_gpus > 1 and world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} needs torch.distributed.run with {n_gpus} processes (WORLD_SIZE={world})")
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device="cuda", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ workloads


def dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class PrefillPart:
    """Causal prefill attention B=1, H=96, T=8192."""

    def __init__(self, seed):
        import torch
        from synth_inputs import prefill_qkv
        inp = prefill_qkv(seed, P_B, P_T, P_H)
        self.host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory() for k, v in inp.items()}
        self.Q, self.K, self.V = (self.host[k].cuda() for k in ("Q", "K", "V"))
        self.O = torch.empty_like(self.Q)
        self.O_host = torch.empty(self.O.shape, dtype=torch.bfloat16).pin_memory()
        self.flops = prefill_flops()
        self.launches = 1

    def run(self):
        import causal_head_latent_b200 as g
        g.gmla_attend_prefill(self.Q, self.K, self.V, self.O, causal=True)

    def run_e2e(self):
        """Through the public API with host buffers: H2D of Q, K, V, the call, D2H of O."""
        import causal_head_latent_b200 as g
        for k, t in (("Q", self.Q), ("K", self.K), ("V", self.V)):
            t.copy_(self.host[k], non_blocking=True)
        g.gmla_attend_prefill(self.Q, self.K, self.V, self.O, causal=True)
        self.O_host.copy_(self.O, non_blocking=True)

    def run_e2e_chunked(self, n_chunks=8):
        """The same through the public API as a chunked prefill: the rows of Q, K, V are copied
        in n_chunks pieces on one stream while gmla_attend_prefill runs each piece of query rows
        over the keys copied so far (queries at the end of the key range, causal) on the current
        stream, and each piece of O is copied back on a third stream, so that the copies in both
        directions overlap the attention."""
        import torch

        import causal_head_latent_b200 as g
        cs = torch.cuda.current_stream()
        if not hasattr(self, "_h2d"):
            self._h2d, self._d2h = torch.cuda.Stream(), torch.cuda.Stream()
        assert P_B == 1 and P_T % n_chunks == 0  # row pieces of a [1, T, H, D] buffer are contiguous
        start = torch.cuda.Event()
        start.record(cs)
        self._h2d.wait_event(start)
        self._d2h.wait_event(start)
        step = P_T // n_chunks
        for i in range(n_chunks):
            r0, r1 = i * step, (i + 1) * step
            with torch.cuda.stream(self._h2d):
                for k, t in (("Q", self.Q), ("K", self.K), ("V", self.V)):
                    t[:, r0:r1].copy_(self.host[k][:, r0:r1], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(self._h2d)
            cs.wait_event(landed)
            g.gmla_attend_prefill(self.Q[:, r0:r1], self.K[:, :r1], self.V[:, :r1], self.O[:, r0:r1], causal=True)
            computed = torch.cuda.Event()
            computed.record(cs)
            self._d2h.wait_event(computed)
            with torch.cuda.stream(self._d2h):
                self.O_host[:, r0:r1].copy_(self.O[:, r0:r1], non_blocking=True)
        done = torch.cuda.Event()
        done.record(self._d2h)
        cs.wait_event(done)

    def e2e_bytes(self):
        h2d = sum(self.host[k].numel() * 2 for k in ("Q", "K", "V"))
        return h2d, self.O.numel() * 2


class DecodePart:
    """One decode step: B=32 new tokens over L=131072 cached latents (d_c=512), d_model=12288."""

    def __init__(self, seed):
        import torch

        import causal_head_latent_b200 as g
        from synth_inputs import Draw, layer_weights
        dr = Draw(seed)
        w = layer_weights(dr, DM, DC, x_shape=(DEC_B, 1, DM))
        cache = dr.normal((DEC_B, DEC_L, DC))
        self.W = {k: dev(v) for k, v in w.items() if k != "X"}
        self.X_host = torch.from_numpy(w["X"].view(np.int16)).view(torch.bfloat16).pin_memory()
        self.X = self.X_host.cuda()
        self.C = dev(cache)
        del cache
        self.Q = torch.empty(DEC_B, 1, DM, dtype=torch.bfloat16, device="cuda")
        self.G = torch.empty_like(self.Q)
        self.O = torch.empty(DEC_B, DM, dtype=torch.bfloat16, device="cuda")
        self.Y = torch.empty_like(self.O)
        self.Y_host = torch.empty(self.Y.shape, dtype=torch.bfloat16).pin_memory()
        self.ws_d = torch.empty(g.gmla_attend_decode_workspace_size(DEC_B, DEC_L, DM // D, DC), dtype=torch.uint8,
                                device="cuda")
        self.bytes = decode_bytes()
        self.launches = 5  # projection GEMM, absorb, latent stream, combine, W_o GEMM

    def project(self):
        import causal_head_latent_b200 as g
        W = self.W
        g.gmla_latent_project(self.X, W["W_q"], W["W_g"], W["W_c"], None, None, Q=self.Q, G=self.G, C=self.C,
                              cache_pos=DEC_L - 1)

    def attend(self):
        import causal_head_latent_b200 as g
        g.gmla_attend_decode(self.Q.view(DEC_B, DM), self.C, DEC_L, self.W["W_k"], self.W["W_v"], self.O, DM // D,
                             G=self.G.view(DEC_B, DM), workspace=self.ws_d)

    def out(self):
        import causal_head_latent_b200 as g
        g.gmla_gate_out(self.O, self.W["W_o"], self.Y)

    def run_e2e(self):
        self.X.copy_(self.X_host, non_blocking=True)
        self.project()
        self.attend()
        self.out()
        self.Y_host.copy_(self.Y, non_blocking=True)


class PlainDecodePart:
    """Decode attention over explicit K, V: B=8, 96 heads, one query at position
    1000 over 1001 keys, [B, H, T, D] layout (the "Softmax over keys" page)."""

    def __init__(self, seed):
        import torch
        from synth_inputs import decode_plain_qkv
        inp = decode_plain_qkv(seed, PL_B, 96, PL_TK)
        self.Q, self.K, self.V = (dev(inp[k]) for k in ("Q", "K", "V"))
        self.O = torch.empty_like(self.Q)
        self.bytes = plain_decode_bytes()
        self.launches = 1

    def run(self):
        import causal_head_latent_b200 as g
        g.gmla_attend_prefill(self.Q, self.K, self.V, self.O, causal=True, layout="bhtd")


class LayerPart:
    """Full Gated MLA layer prefill: B=2, T=4096, d_model=12288, d_c=512."""

    def __init__(self, seed):
        import torch
        from synth_inputs import Draw, layer_weights
        w = layer_weights(Draw(seed), DM, DC, x_shape=(L_B, L_T, DM))
        self.t = {k: dev(v) for k, v in w.items()}
        self.Q = torch.empty(L_B, L_T, DM, dtype=torch.bfloat16, device="cuda")
        self.G, self.K, self.V, self.O, self.Y = (torch.empty_like(self.Q) for _ in range(5))
        self.C = torch.empty(L_B, L_T, DC, dtype=torch.bfloat16, device="cuda")
        self.flops = layer_flops()
        self.launches = 4  # [Q|G|C] GEMM, [K|V] GEMM, attention, W_o GEMM

    def project(self):
        import causal_head_latent_b200 as g
        t = self.t
        g.gmla_latent_project(t["X"], t["W_q"], t["W_g"], t["W_c"], t["W_k"], t["W_v"], Q=self.Q, G=self.G, C=self.C,
                              K=self.K, V=self.V)

    def attend(self):
        import causal_head_latent_b200 as g
        H = DM // D
        v = lambda x: x.view(L_B, L_T, H, D)
        g.gmla_attend_prefill(v(self.Q), v(self.K), v(self.V), v(self.O), G=self.G)

    def out(self):
        import causal_head_latent_b200 as g
        g.gmla_gate_out(self.O, self.t["W_o"], self.Y)

    def run(self):
        self.project()
        self.attend()
        self.out()


# ------------------------------------------------------------------ CPU baseline (oracle)


def oracle_prefill_sample(seconds_target=15.0, rows=None, inp=None):
    """Time the float64 oracle on a bounded sample of the prefill workload: `rows`
    query rows (b=0, random head and position) of the B=1, H=96, T=8192 problem."""
    import oracle as orc
    from synth_inputs import SEEDS, prefill_qkv
    if inp is None:
        # widened to float64 once, outside the timed call
        inp = {k: orc.widen(v) for k, v in prefill_qkv(SEEDS["prefill_attn"], P_B, P_T, P_H).items()}
    rng = np.random.default_rng(1)
    if rows is None:
        rows = 2000
    sel = np.stack([np.zeros(rows, np.int64), rng.integers(0, P_H, rows), rng.integers(0, P_T, rows)], 1)
    flops = float(np.sum(4.0 * D * (sel[:, 2] + 1)))
    t0 = time.perf_counter()
    orc.attention(inp["Q"], inp["K"], inp["V"], rows=sel)
    dt = time.perf_counter() - t0
    return flops, dt, rows, orc.num_threads(), inp


def cpu_baseline_prefill(target_s=15.0):
    flops, dt, rows, cores, inp = oracle_prefill_sample(rows=500)
    n = int(max(500, min(200000, 500 * target_s / max(dt, 1e-3))))
    flops, dt, rows, cores, _ = oracle_prefill_sample(rows=n, inp=inp)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} random query rows (b=0, random head, random position) of the B=1 H=96 T=8192 causal "
                      f"prefill, float64 C oracle, {dt:.1f} s"}


def cpu_baseline_decode(target_s=8.0):
    """Oracle decode (plain definition: K_h, V_h rebuilt from the cache) for a few
    (b, h) pairs over the first `L` latents; GB/s counts the cache bytes a full
    decode step would stream at the same per-(b,h) rate."""
    import oracle as orc
    from synth_inputs import Draw
    dr = Draw(77)
    L = 8192
    H = 96
    q = dr.normal((1, DM))
    cache = dr.normal((1, L, DC))
    Wk = dr.normal((DM, DC), 1 / math.sqrt(DC))
    Wv = dr.normal((DM, DC), 1 / math.sqrt(DC))
    heads = [(0, h) for h in range(0, H, 12)]
    t0 = time.perf_counter()
    orc.decode_latent(q, cache, L, Wk, Wv, H, heads=heads)
    dt = time.perf_counter() - t0
    # full step = DEC_B * H (b, h) pairs over DEC_L latents; per-(b,h) time scales with L
    t_full = dt / len(heads) * (DEC_B * H) * (DEC_L / L)
    return {"value": decode_bytes() / t_full / 1e9, "unit": "GB/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{len(heads)} (b,h) pairs over L={L} latents (non-absorbed float64 C oracle, {dt:.1f} s), "
                      f"scaled to B=32 x 96 heads x L=131072"}


# ------------------------------------------------------------------ main


def run_reference(args, rank, world):
    """Reference arm: the float64 oracle timed on the host cores."""
    if rank != 0:
        return
    flops0, dt0, _, cores, inp = oracle_prefill_sample(rows=200)
    rows = int(max(200, min(20000, 200 * 2.0 / max(dt0, 1e-3))))   # about 2 s per step
    for _ in range(args.warmup):
        oracle_prefill_sample(rows=rows, inp=inp)
    tot_f = tot_t = 0.0
    for _ in range(args.steps):
        f, dt, _, cores, _ = oracle_prefill_sample(rows=rows, inp=inp)
        tot_f += f
        tot_t += dt
    val = tot_f / tot_t / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_obj(args),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step {rows} random query rows of the B=1 H=96 T=8192 causal prefill"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_obj(args):
    if args.workload == "layer":
        return {"workload": f"Gated MLA layer prefill B={L_B} T={L_T} d_model={DM} H=96 D_h=128 d_c={DC} bf16",
                "global_batch": L_B * max(1, args.gpus), "seq_len": L_T, "parallelism": f"dp{args.gpus}",
                "l2": "inputs larger than L2"}
    return {"workload": f"causal prefill attention B={P_B} H={P_H} T={P_T} D_h={D} bf16 + latent-cache decode "
                        f"B={DEC_B} L={DEC_L} d_c={DC} H=96 d_model={DM} (projections, append, absorbed attention, "
                        f"LSE combine, gate, W_o) + decode over explicit K/V B={PL_B} H=96 Tk={PL_TK} + full layer "
                        f"prefill B={L_B} T={L_T} d_model={DM} d_c={DC}",
            "global_batch": P_B * max(1, args.gpus), "seq_len": P_T, "parallelism": f"dp{args.gpus}",
            "parts": args.parts, "l2": "inputs larger than L2 (Q/K/V 604 MB, cache 4.3 GB, layer 2.4 GB); no flush"}


def timed(fn_list, steps, world):
    """Run `steps` iterations of every fn in fn_list; per-fn CUDA-event time on the
    current stream; the whole region bracketed by barrier + synchronize."""
    import torch
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in fn_list]
          for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    start.record()
    for i in range(steps):
        for j, fn in enumerate(fn_list):
            ev[i][j][0].record()
            fn()
            ev[i][j][1].record()
    end.record()
    barrier(world)
    total = start.elapsed_time(end)
    per = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps)) for j in range(len(fn_list))]
    return total, per


def run_varlen(args, rank, world, local, peaks):
    """Variable-length batches: gmla_attend_prefill_varlen over VL_Q / VL_KV (H = VL_H;
    flops count each sequence's own causal pairs) and gmla_attend_decode_varlen at
    B = VL_DEC_B with seeded lengths in 1..VL_DEC_LMAX (bytes count visible latents)."""
    import torch

    import causal_head_latent_b200 as g
    from synth_inputs import Draw, prefill_qkv

    B = len(VL_Q)
    Tq, Tk = max(VL_Q), max(VL_KV)
    inp = prefill_qkv(1401, B, Tq, VL_H, Tk=Tk)
    Q, K, V = (dev(inp[k]) for k in ("Q", "K", "V"))
    del inp
    O = torch.empty_like(Q)
    wsp = torch.empty(g.gmla_attend_prefill_varlen_workspace_size(B), dtype=torch.uint8, device="cuda")
    pairs = sum(q * (kv - q) + q * (q + 1) // 2 for q, kv in zip(VL_Q, VL_KV))
    pf = 4.0 * D * VL_H * pairs

    dr = Draw(1402)
    lens = [int(x) for x in np.random.default_rng(1402).integers(1, VL_DEC_LMAX + 1, VL_DEC_B)]
    H, d = DM // D, DM
    q = dev(dr.normal((VL_DEC_B, d)))
    Wk = dev(dr.normal((d, DC), 1 / np.sqrt(DC)))
    Wv = dev(dr.normal((d, DC), 1 / np.sqrt(DC)))
    C = dev(dr.normal((VL_DEC_B, VL_DEC_LMAX, DC)))
    Od = torch.empty(VL_DEC_B, d, dtype=torch.bfloat16, device="cuda")
    wsd = torch.empty(g.gmla_attend_decode_varlen_workspace_size(VL_DEC_B, VL_DEC_LMAX, H, DC), dtype=torch.uint8,
                      device="cuda")
    db = 2.0 * (sum(lens) * DC + 2 * d * DC + 2 * VL_DEC_B * d)

    fp = lambda: g.gmla_attend_prefill_varlen(Q, K, V, O, VL_Q, VL_KV, workspace=wsp)
    fd = lambda: g.gmla_attend_decode_varlen(q, C, lens, Wk, Wv, Od, H, workspace=wsd)
    for _ in range(args.warmup):
        fp()
        fd()
    g.gmla_get_device_status()
    clk = ClockSampler(local)
    clk.start()
    total, per = timed([fp, fd], args.steps, world)
    clk.stop()
    clocks = clk.summary()
    g.gmla_get_device_status()
    total = max_over_ranks(total, world)
    p_ms = max_over_ranks(per[0], world) / args.steps
    d_ms = max_over_ranks(per[1], world) / args.steps
    p_tf = pf / (p_ms / 1e3) / 1e12
    d_gbs = db / (d_ms / 1e3) / 1e9
    line = {"metric": "variable-length batches: padded prefill attention TFLOP/s (per-sequence causal pairs) and "
                      "per-sequence-length latent decode GB/s",
            "value": p_tf, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"gmla_attend_prefill_varlen B={B} H={VL_H} D_h={D} q_lens={list(VL_Q)} "
                                   f"kv_lens={list(VL_KV)} + gmla_attend_decode_varlen B={VL_DEC_B} H=96 d_c={DC} "
                                   f"lengths seeded in 1..{VL_DEC_LMAX} (sum {sum(lens)})",
                       "l2": "inputs larger than L2; no flush"},
            "clocks": clocks, "gpu_launches": 4 * args.steps,
            "roofline": {"bound": "tensor", "achieved": p_tf, "peak": peaks["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": p_tf / peaks["bf16_tflops_sustained"], "traffic": None},
            "decode": {"value": d_gbs, "unit": "GB/s", "ms_per_step": d_ms,
                       "roofline": {"bound": "hbm", "achieved": d_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": d_gbs / peaks["hbm_gbs"], "traffic": None}},
            "prefill_ms": p_ms}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(args, rank, world, local, peaks):
    """Long-context sweep: causal prefill attention (B=1, SWEEP_H heads) and latent-cache
    decode (B=SWEEP_B, 96 heads, d_c=512) at each length of SWEEP_T, each timed with CUDA
    events after W warm-up calls; K per size is as many calls as fit ~2 s (at most --steps)."""
    import torch

    import causal_head_latent_b200 as g
    from synth_inputs import Draw, prefill_qkv

    def time_fn(fn, launches):
        for _ in range(args.warmup):
            fn()
        g.gmla_get_device_status()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, int(2000.0 / max(e0.elapsed_time(e1), 1e-3))))
        total, _ = timed([fn], steps, world)
        g.gmla_get_device_status()
        return max_over_ranks(total, world) / steps, steps * launches

    rows, launches = [], 0
    clk = ClockSampler(local)
    clk.start()
    for i, T in enumerate(SWEEP_T):
        inp = prefill_qkv(900 + i, 1, T, SWEEP_H)
        Q, K, V = (dev(inp[k]) for k in ("Q", "K", "V"))
        del inp
        O = torch.empty_like(Q)
        p_ms, n = time_fn(lambda: g.gmla_attend_prefill(Q, K, V, O, causal=True), 1)
        launches += n
        del Q, K, V, O
        dr = Draw(950 + i)
        H, d = DM // D, DM
        q = dev(dr.normal((SWEEP_B, d)))
        Wk = dev(dr.normal((d, DC), 1 / np.sqrt(DC)))
        Wv = dev(dr.normal((d, DC), 1 / np.sqrt(DC)))
        C = dev(dr.normal((SWEEP_B, T, DC)))
        Od = torch.empty(SWEEP_B, d, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(g.gmla_attend_decode_workspace_size(SWEEP_B, T, H, DC), dtype=torch.uint8, device="cuda")
        d_ms, n = time_fn(lambda: g.gmla_attend_decode(q, C, T, Wk, Wv, Od, H, workspace=ws), 3)
        launches += n
        del q, Wk, Wv, C, Od, ws
        torch.cuda.empty_cache()
        pf = prefill_flops(1, SWEEP_H, T)
        db = decode_bytes(SWEEP_B, T)
        rows.append({"T": T, "dot_products_per_head": T * (T + 1) / 2,
                     "prefill_ms": p_ms, "prefill_tflops": pf / (p_ms / 1e3) / 1e12,
                     "prefill_frac_of_sustained_bf16": pf / (p_ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"],
                     "decode_ms": d_ms, "decode_gbs": db / (d_ms / 1e3) / 1e9,
                     "decode_frac_of_hbm": db / (d_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "cache_bytes_per_sequence": T * DC * 2})
    clk.stop()
    clocks = clk.summary()
    ratios = {}
    for a, b in ((0, 1), (1, 2)):
        ta, tb = SWEEP_T[a], SWEEP_T[b]
        lab = lambda t: f"{t // 1048576}M" if t % 1048576 == 0 else f"{t // 1024}K"
        key = f"{lab(ta)}->{lab(tb)}"
        ratios[key] = {"dot_products": rows[b]["dot_products_per_head"] / rows[a]["dot_products_per_head"],
                       "prefill_time": rows[b]["prefill_ms"] / rows[a]["prefill_ms"],
                       "kv_cache": tb / ta, "decode_time": rows[b]["decode_ms"] / rows[a]["decode_ms"]}
    line = {"metric": "long-context sweep: causal prefill attention TFLOP/s and latent-cache decode time vs context "
                      "length (8K, 128K, 1M)",
            "value": rows[-1]["prefill_tflops"], "unit": "TFLOP/s", "n_gpus": world, "steps": None,
            "warmup": args.warmup, "ms_per_step": rows[-1]["prefill_ms"] + rows[-1]["decode_ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"causal prefill attention B=1 H={SWEEP_H} D_h={D} and latent-cache decode "
                                   f"B={SWEEP_B} H=96 d_c={DC} at T = L = 8192, 131072, 1048576",
                       "l2": "inputs larger than L2 at 128K and 1M; at 8K the decode cache (33.5 MB) fits in L2"},
            "clocks": clocks, "gpu_launches": launches, "sweep": rows, "ratios": ratios, "pages": SWEEP_PAGE}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    global DEC_L
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parts", default="all", choices=["all", "prefill", "decode", "plain", "layer"])
    ap.add_argument("--workload", default="step", choices=["step", "layer", "sweep", "varlen"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--dec-L", type=int, default=DEC_L,
                    help="cached latent length of the decode part (smaller only for profiling captures)")
    args = ap.parse_args()
    DEC_L = args.dec_L
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return

    import torch
    rank, world, local = dist_setup(args.gpus)
    import causal_head_latent_b200 as g
    peaks = load_peaks()

    if args.workload == "sweep":
        run_sweep(args, rank, world, local, peaks)
        return
    if args.workload == "varlen":
        run_varlen(args, rank, world, local, peaks)
        return

    if args.workload == "layer":
        part = LayerPart(4)
        for _ in range(args.warmup):
            part.run()
        g.gmla_get_device_status()
        clk = ClockSampler(local)
        clk.start()
        total, per = timed([part.run], args.steps, world)
        clk.stop()
        clocks = clk.summary()
        g.gmla_get_device_status()
        total = max_over_ranks(total, world)
        val = part.flops * args.steps * world / (total / 1e3) / 1e12
        line = {"metric": "Gated MLA layer prefill TFLOP/s", "value": val, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": config_obj(args), "clocks": clocks,
                "gpu_launches": part.launches * args.steps,
                "roofline": {"bound": "tensor", "achieved": val / world,
                             "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                             "frac": val / world / peaks["bf16_tflops_sustained"], "traffic": None,
                             "peak_kind": f"{peaks['source']} sustained bf16"}}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return

    pre = dec = plain = layer = None
    if args.parts in ("all", "prefill"):
        pre = PrefillPart(3)
    if args.parts in ("all", "decode"):
        dec = DecodePart(5)
    if args.parts in ("all", "layer"):
        layer = LayerPart(4)
    if args.parts in ("all", "plain"):
        plain = PlainDecodePart(2)
    # One step is one pass over every workload.  Each workload is warmed up and
    # timed in a region of its own (K steps), in this order, so that the power
    # drawn by the GEMM-heavy full layer does not lower the clock of the kernels
    # measured before it; each region reports the clocks sampled during it.
    regions = []
    if pre:
        regions.append(("prefill", [("prefill_attention", pre.run)]))
    if dec:
        regions.append(("decode", [("decode_project", dec.project), ("decode_attend", dec.attend),
                                   ("decode_out", dec.out)]))
    if plain:
        regions.append(("plain", [("plain_decode", plain.run)]))
    if layer:
        regions.append(("layer", [("layer_project", layer.project), ("layer_attend", layer.attend),
                                  ("layer_out", layer.out)]))
    K = args.steps
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)  # the sampler's first sample
    perd, region_ms, region_clocks = {}, {}, {}
    for rname, fl in regions:
        for _ in range(args.warmup):
            for _, fn in fl:
                fn()
        g.gmla_get_device_status()
        h0 = time.time()
        rt, per = timed([fn for _, fn in fl], K, world)
        h1 = time.time()
        g.gmla_get_device_status()
        region_ms[rname] = max_over_ranks(rt, world)
        region_clocks[rname] = (h0, h1)
        for (n, _), v in zip(fl, per):
            perd[n] = max_over_ranks(v, world)
    time.sleep(0.1)
    clk.stop()
    t_first, t_last = min(h[0] for h in region_clocks.values()), max(h[1] for h in region_clocks.values())
    region_clocks = {r: clk.summary(*hh) for r, hh in region_clocks.items()}
    clocks = clk.summary(t_first, t_last)  # every timed region, warm-ups between them included
    total = sum(region_ms.values())
    launches = sum(p.launches for p in (pre, dec, layer, plain) if p is not None)
    # the prefill region is tens of milliseconds at the sampled clock: the burst
    # peak (a short cuBLAS run) is its denominator; the sustained one (seconds
    # under the power cap) is reported beside it
    burst = peaks["bf16_tflops"]

    line = {"metric": METRIC, "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_obj(args), "clocks": clocks, "gpu_launches": launches * K,
            "kernel_ms_per_step": {k: v / K for k, v in perd.items()},
            "regions": {r: {"ms_per_step": region_ms[r] / K, "clocks": region_clocks[r]} for r in region_ms}}
    if pre:
        t_att = perd["prefill_attention"] / K
        val = pre.flops * world / (t_att / 1e3) / 1e12
        line.update(value=val, unit="TFLOP/s")
        ach = pre.flops / (t_att / 1e3) / 1e12
        tr, tr_how = profiled_traffic("attn_prefill_kernel")
        line["roofline"] = {"bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s",
                            "frac": ach / burst, "traffic": tr, "traffic_source": tr_how,
                            "algorithmic_bytes": 2.0 * 4 * P_B * P_T * P_H * D,
                            "kernel": "attn_prefill_kernel",
                            "peak_kind": f"{peaks['source']} burst bf16 (timed region of {region_ms['prefill']:.0f} ms "
                                         f"at {region_clocks['prefill']['sm_mhz']} MHz)",
                            "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
                            "frac_of_datasheet_2250": ach / 2250.0}
    if dec:
        t_dec = perd["decode_attend"] / K
        gbs = dec.bytes / (t_dec / 1e3) / 1e9
        t_step = (perd["decode_project"] + perd["decode_attend"] + perd["decode_out"]) / K
        tr, tr_how = profiled_traffic("gmla_attend_decode") if DEC_L == 131072 else (None, None)
        dobj = {"value": gbs * world, "unit": "GB/s", "ms_per_step": t_dec,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "traffic": tr, "traffic_source": tr_how,
                             "algorithmic_bytes": dec.bytes, "kernel": "gmla_attend_decode",
                             "peak_kind": f"{peaks['source']} HBM copy", "frac_of_datasheet_8000": gbs / 8000.0},
                "step_ms": t_step, "step_gbs": decode_step_bytes() / (t_step / 1e3) / 1e9,
                "workload": f"latent-cache decode B={DEC_B} L={DEC_L} d_c={DC} H=96 d_model={DM}",
                "clocks": region_clocks["decode"]}
        line["decode"] = dobj
        if not pre:
            line.update(value=gbs * world, unit="GB/s", roofline=dobj["roofline"])
    if layer:
        t_l = sum(perd[k] for k in ("layer_project", "layer_attend", "layer_out")) / K
        tf = layer.flops / (t_l / 1e3) / 1e12
        ltr, ltr_how = profiled_traffic("gemm_kernel")
        H = DM // D
        M = L_B * L_T
        parts_flops = {"layer_project": 2.0 * M * DM * (2 * DM + DC) + 2.0 * M * DC * 2 * DM,
                       "layer_attend": prefill_flops(L_B, H, L_T), "layer_out": 2.0 * M * DM * DM}
        lobj = {"value": tf * world, "unit": "TFLOP/s", "ms_per_step": t_l,
                "workload": f"Gated MLA layer prefill B={L_B} T={L_T} d_model={DM} H=96 D_h=128 d_c={DC}",
                "algorithmic_flops": layer.flops,
                "roofline": {"bound": "tensor", "achieved": tf, "peak": burst, "unit": "TFLOP/s", "frac": tf / burst,
                             "traffic": ltr, "traffic_source": ltr_how, "traffic_kernel": "gemm_kernel ([Q|G|C] launch)",
                             "peak_kind": f"{peaks['source']} burst bf16",
                             "frac_of_sustained": tf / peaks["bf16_tflops_sustained"]},
                "clocks": region_clocks["layer"],
                "calls": {k: {"ms": perd[k] / K, "tflops": f / (perd[k] / K / 1e3) / 1e12}
                          for k, f in parts_flops.items()}}
        line["layer"] = lobj
        if not (pre or dec):
            line.update(value=tf * world, unit="TFLOP/s", roofline=lobj["roofline"])
    if plain:
        t_p = perd["plain_decode"] / K
        gbs = plain.bytes / (t_p / 1e3) / 1e9
        ptr, ptr_how = profiled_traffic("attn_rows_kernel")
        pobj = {"value": gbs * world, "unit": "GB/s", "ms_per_step": t_p,
                "workload": f"decode attention over explicit K/V B={PL_B} H=96 Tq=1 Tk={PL_TK} D_h=128 [B,H,T,D]",
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "traffic": ptr, "traffic_source": ptr_how,
                             "algorithmic_bytes": plain.bytes,
                             "kernel": "attn_rows_kernel", "peak_kind": f"{peaks['source']} HBM copy",
                             "l2": "394 MB of K/V, timed back to back (a step reads them once; about 3x L2)"},
                "clocks": region_clocks["plain"]}
        line["decode_plain"] = pobj
        if not (pre or dec or layer):
            line.update(value=gbs * world, unit="GB/s", roofline=pobj["roofline"])

    # end-to-end through the public API with pinned host buffers
    if not args.no_e2e and (pre or dec):
        ke = max(1, min(K, 5))
        if pre:
            def time_e2e(fn):
                fn()
                barrier(world)
                t0 = torch.cuda.Event(enable_timing=True)
                t1 = torch.cuda.Event(enable_timing=True)
                t0.record()
                for _ in range(ke):
                    fn()
                t1.record()
                barrier(world)
                return max_over_ranks(t0.elapsed_time(t1), world) / ke
            te_serial = time_e2e(pre.run_e2e)
            te = time_e2e(pre.run_e2e_chunked)
            h2d, d2h = pre.e2e_bytes()
            line["e2e"] = {"value": pre.flops * world / (te / 1e3) / 1e12, "unit": "TFLOP/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": te,
                           "what": "H2D of Q, K, V from pinned host memory in 8 row pieces on a copy stream, "
                                   "gmla_attend_prefill per piece of query rows over the keys copied so far, "
                                   "D2H of each piece of O on a third stream (copies overlap the attention)",
                           "serial": {"value": pre.flops * world / (te_serial / 1e3) / 1e12, "ms_per_step": te_serial,
                                      "what": "H2D of Q, K, V, one gmla_attend_prefill, D2H of O, one after another"}}
        if dec:
            dec.run_e2e()
            barrier(world)
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(ke):
                dec.run_e2e()
            t1.record()
            barrier(world)
            te = max_over_ranks(t0.elapsed_time(t1), world) / ke
            e = {"value": dec.bytes * world / (te / 1e3) / 1e9, "unit": "GB/s",
                 "h2d_bytes_per_step": dec.X_host.numel() * 2, "d2h_bytes_per_step": dec.Y_host.numel() * 2,
                 "ms_per_step": te, "what": "H2D of the new tokens' hidden states + full decode step "
                                            "(projections, append, attend, W_o) + D2H of Y; cache and weights resident"}
            line["decode"]["e2e"] = e
            if not pre:
                line["e2e"] = e
        g.gmla_get_device_status()

    if rank == 0 and world >= 1 and not args.no_cpu:
        if pre:
            line["cpu_baseline"] = cpu_baseline_prefill()
        if dec:
            cb = cpu_baseline_decode()
            line["decode"]["cpu_baseline"] = cb
            if not pre:
                line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

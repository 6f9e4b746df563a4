"""bench.py without a GPU: the reference arm (the float64 oracle timed on the
host) prints one JSON line with the contract's keys, ranks other than 0 print
nothing, and the workload arithmetic matches the figures the timed
configurations are quoted with."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

from tests.conftest import ROOT

BENCH = os.path.join(ROOT, "bench.py")


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", BENCH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, BENCH] + args, cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_reference_arm_json_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_are_silent():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"],
             {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]


def test_workload_arithmetic():
    b = _load_bench()
    # causal pairs T(T+1)/2 per head, 4*D flop per pair (QK^T and PV): 1.6495e12 at B=1, H=96, T=8192
    assert b.prefill_flops(1, 96, 8192) == pytest.approx(1.6495e12, rel=1e-4)
    # the decode streams every visible latent once: B*L*d_c*2 bytes = 4.295e9 at B=32, L=131072
    latents = 32 * 131072 * 512 * 2
    assert latents == pytest.approx(4.295e9, rel=1e-3)
    extra = b.decode_bytes(32, 131072) - latents
    assert 0 < extra < 0.02 * latents  # W_k, W_v, q, G and O on top of the cache
    # decode over explicit K, V at the softmax page's shape: Q, K, V, O = 394.0 MB
    assert b.plain_decode_bytes() == 2 * 8 * 96 * 128 * (2 * 1001 + 2)
    assert b.plain_decode_bytes() == pytest.approx(393.8e6, rel=1e-3)
    # full layer prefill: a1 5.05e12 + a2 2.06e11 + a3 8.248e11 + a5 2.474e12 = 8.556e12 flop
    assert b.layer_flops() == pytest.approx(8.556e12, rel=1e-3)
    # the sweep's lengths are the cost table's, whose dot-product orders they reproduce
    assert b.SWEEP_T == (8192, 131072, 1048576)
    for t, order in zip(b.SWEEP_T, b.SWEEP_PAGE["dot_products_per_head"]):
        assert t * (t + 1) / 2 == pytest.approx(order, rel=0.06)


def test_traffic_records_follow_the_code_not_the_comments():
    """The recorded DRAM traffic of a kernel is reported only while the code it
    was captured from is unchanged: a comment or whitespace edit keeps it, any
    change of a token (inside a string literal too) drops it."""
    b = _load_bench()
    src = 'int a = 1;  // note\n/* block */ asm("x // y"); char q = \'"\';\n'
    assert b.code_only(src) == b.code_only(src.replace("note", "other note").replace("  ", " "))
    assert b.code_only(src) != b.code_only(src.replace("a = 1", "a = 2"))
    assert b.code_only(src) != b.code_only(src.replace("x // y", "x // z"))
    for kernel, ent in b.PROFILED_TRAFFIC.items():
        assert len(ent["sha1"]) == 40 and ent["bytes"] > 0, kernel
        assert all(os.path.exists(os.path.join(ROOT, "causal_head_latent_b200", "csrc", f)) for f in ent["sources"])

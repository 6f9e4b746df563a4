"""Workspace layouts, checked on the CPU (no GPU, nothing launched).

The calls that copy tensor maps into a caller workspace (the variable-length
decode and prefill) must place them on a 64-byte boundary -- TMA reads a map
from global memory at that alignment -- although the caller only promises a
16-byte-aligned pointer, and every region must fit in the size the matching
*_workspace_size function reports.  The layout arithmetic is a pure host
header (csrc/ws_layout.h), so a small C++ program compiled here evaluates it
for every 16-byte-aligned offset of the base within 256 bytes and for a range
of problem sizes; the sizes it derives must equal the library's own reports.
"""
import ctypes
import json
import os
import subprocess

import pytest

from tests.conftest import ROOT

CSRC = os.path.join(ROOT, "causal_head_latent_b200", "csrc")

CHECKER = r"""
#include <cstdio>
#include "ws_layout.h"
using namespace gmla;
int main() {
  const long long cases[][4] = {{1, 1, 1, 64}, {2, 100, 2, 64}, {3, 4163, 96, 512}, {32, 131072, 96, 512},
                                {7, 999, 5, 192}, {113, 5000, 96, 512}, {1000, 64, 96, 512}};
  std::printf("[");
  bool first = true;
  for (auto &c : cases) {
    const long long B = c[0], L = c[1], H = c[2], dc = c[3];
    int S, kps;
    latent_plan(B, L, kLatentTileKeys, &S, &kps);
    for (int per_seq = 0; per_seq < 2; ++per_seq) {
      const size_t need = latent_layout_bytes(B, H, dc, S, per_seq);
      for (unsigned long long k = 0; k < 16; ++k) {
        const unsigned long long base = 0x7f0000000000ull + 16 * k;
        const LatentLayout o = latent_layout(base, B, H, dc, S, per_seq);
        std::printf("%s{\"kind\":\"decode\",\"B\":%lld,\"L\":%lld,\"H\":%lld,\"dc\":%lld,\"S\":%d,\"kps\":%d,"
                    "\"tile\":%d,\"per_seq\":%d,\"base\":%llu,\"need\":%zu,\"qt\":%zu,\"pm\":%zu,\"pl\":%zu,\"pacc\":%zu,"
                    "\"lse2\":%zu,\"maps\":%zu,\"lens\":%zu,\"end\":%zu}",
                    first ? "" : ",", B, L, H, dc, S, kps, kLatentTileKeys, per_seq, base, need, o.qt, o.pm, o.pl, o.pacc, o.lse2,
                    o.maps, o.lens, o.end);
        first = false;
      }
    }
    const size_t pneed = prefill_varlen_layout_bytes(B);
    for (unsigned long long k = 0; k < 16; ++k) {
      const unsigned long long base = 0x7f0000000000ull + 16 * k;
      const PrefillVarlenLayout o = prefill_varlen_layout(base, B);
      std::printf(",{\"kind\":\"prefill\",\"B\":%lld,\"base\":%llu,\"need\":%zu,\"maps\":%zu,\"lens\":%zu,"
                  "\"end\":%zu}", B, base, pneed, o.maps, o.lens, o.end);
    }
  }
  std::printf("]\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def layouts(tmp_path_factory):
    d = tmp_path_factory.mktemp("wslayout")
    src, exe = d / "check.cpp", d / "check"
    src.write_text(CHECKER)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    return json.loads(subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout)


def test_tensor_maps_land_on_64_byte_boundaries(layouts):
    for r in layouts:
        if r["kind"] == "decode" and not r["per_seq"]:
            continue
        assert (r["base"] + r["maps"]) % 64 == 0, r
        assert (r["base"] + r["lens"]) % 4 == 0, r


def test_regions_are_ordered_disjoint_and_fit(layouts):
    for r in layouts:
        if r["kind"] == "prefill":
            B = r["B"]
            assert r["lens"] - r["maps"] >= 3 * B * 128
            assert r["end"] - r["lens"] >= 2 * B * 4
        else:
            B, H, dc, S = r["B"], r["H"], r["dc"], r["S"]
            assert r["pm"] - r["qt"] >= 2 * B * H * dc
            assert r["pl"] - r["pm"] >= 4 * S * B * H
            assert r["pacc"] - r["pl"] >= 4 * S * B * H
            assert r["lse2"] - r["pacc"] >= 4 * S * B * H * dc
            assert r["maps"] - r["lse2"] >= 4 * B * H
            if r["per_seq"]:
                assert r["lens"] - r["maps"] >= 128 * B
                assert r["end"] - r["lens"] >= 4 * B
            # float4 loads and TMA: the float32 states and q~ start 16-byte aligned
            for k in ("qt", "pm", "pl", "pacc", "lse2"):
                assert (r["base"] + r[k]) % 16 == 0, (k, r)
        assert r["end"] <= r["need"], r


def test_split_plan_covers_every_key_once(layouts):
    for r in layouts:
        if r["kind"] != "decode":
            continue
        S, kps, L = r["S"], r["kps"], r["L"]
        assert kps % r["tile"] == 0 and S >= 1
        assert (S - 1) * kps < L <= S * kps, r   # no empty split, nothing left over


def test_library_reports_the_same_sizes(layouts):
    from causal_head_latent_b200 import build
    build.build()
    import causal_head_latent_b200 as g
    L = g.lib
    for r in layouts:
        if r["kind"] == "prefill":
            assert L.gmla_attend_prefill_varlen_workspace_size(r["B"]) == r["need"]
        elif r["per_seq"]:
            assert L.gmla_attend_decode_varlen_workspace_size(r["B"], r["L"], r["H"], r["dc"]) == r["need"]
        else:
            assert L.gmla_attend_decode_workspace_size(r["B"], r["L"], r["H"], r["dc"]) == r["need"]
            assert L.gmla_attend_decode_partial_workspace_size(r["B"], 5, 5 + r["L"], r["H"], r["dc"]) == r["need"]

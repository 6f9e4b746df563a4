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
      const long long R = per_seq ? latent_varlen_records(B, L, kLatentTileKeys) : (long long)S * B;
      const size_t need = latent_layout_bytes(B, H, dc, R, per_seq);
      for (unsigned long long k = 0; k < 16; ++k) {
        const unsigned long long base = 0x7f0000000000ull + 16 * k;
        const LatentLayout o = latent_layout(base, B, H, dc, R, per_seq);
        std::printf("%s{\"kind\":\"decode\",\"B\":%lld,\"L\":%lld,\"H\":%lld,\"dc\":%lld,\"S\":%d,\"kps\":%d,"
                    "\"R\":%lld,\"tile\":%d,\"per_seq\":%d,\"base\":%llu,\"need\":%zu,\"qt\":%zu,\"pm\":%zu,"
                    "\"pl\":%zu,\"pacc\":%zu,\"lse2\":%zu,\"maps\":%zu,\"lens\":%zu,\"items\":%zu,\"offs\":%zu,"
                    "\"end\":%zu}",
                    first ? "" : ",", B, L, H, dc, S, kps, R, kLatentTileKeys, per_seq, base, need, o.qt, o.pm, o.pl,
                    o.pacc, o.lse2, o.maps, o.lens, o.items, o.offs, o.end);
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
            B, H, dc, R = r["B"], r["H"], r["dc"], r["R"]
            assert R >= r["S"] * B
            assert r["pm"] - r["qt"] >= 2 * B * H * dc
            assert r["pl"] - r["pm"] >= 4 * R * H
            assert r["pacc"] - r["pl"] >= 4 * R * H
            assert r["lse2"] - r["pacc"] >= 4 * R * H * dc
            assert r["maps"] - r["lse2"] >= 4 * B * H
            if r["per_seq"]:
                assert r["lens"] - r["maps"] >= 128 * B
                assert r["items"] - r["lens"] >= 4 * B
                assert r["offs"] - r["items"] >= 16 * R
                assert r["end"] - r["offs"] >= 4 * (B + 1)
                assert (r["base"] + r["items"]) % 16 == 0, r
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


PLAN_CHECKER = r"""
#include <cstdio>
#include <vector>
#include "ws_layout.h"
using namespace gmla;
int main() {
  // each case: B, Lmax, then B lengths
  std::vector<std::vector<long long>> cases = {
      {1, 1, 1}, {3, 100, 100, 1, 47}, {4, 131072, 131072, 131072, 131072, 131072},
      {5, 131072, 131072, 4096, 4096, 49, 97}, {2, 1000000, 1000000, 17}};
  // a skewed batch: one long sequence and 31 short ones
  std::vector<long long> sk = {32, 131072, 131072};
  for (int b = 1; b < 32; ++b) sk.push_back(4096 + 37 * b);
  cases.push_back(sk);
  // 64 sequences of random-looking lengths
  std::vector<long long> rnd = {64, 70000};
  unsigned long long x = 12345;
  for (int b = 0; b < 64; ++b) {
    x = x * 6364136223846793005ull + 1442695040888963407ull;
    rnd.push_back(1 + (long long)((x >> 33) % 70000));
  }
  cases.push_back(rnd);
  std::printf("[");
  for (size_t c = 0; c < cases.size(); ++c) {
    const long long B = cases[c][0], Lmax = cases[c][1];
    const long long *lens = cases[c].data() + 2;
    const long long R = latent_varlen_records(B, Lmax, kLatentTileKeys);
    int kps = 0;
    const long long n = latent_varlen_plan(lens, B, kLatentTileKeys, R, &kps, nullptr, nullptr);
    std::vector<LatentItem> it((size_t)n);
    std::vector<int> off((size_t)B + 1);
    int kps2 = 0;
    const long long n2 = latent_varlen_plan(lens, B, kLatentTileKeys, R, &kps2, it.data(), off.data());
    std::printf("%s{\"B\":%lld,\"R\":%lld,\"kps\":%d,\"kps2\":%d,\"n\":%lld,\"n2\":%lld,\"tile\":%d,\"lens\":[",
                c ? "," : "", B, R, kps, kps2, n, n2, kLatentTileKeys);
    for (long long b = 0; b < B; ++b) std::printf("%s%lld", b ? "," : "", lens[b]);
    std::printf("],\"off\":[");
    for (long long b = 0; b <= B; ++b) std::printf("%s%d", b ? "," : "", off[b]);
    std::printf("],\"items\":[");
    for (long long i = 0; i < n; ++i)
      std::printf("%s[%d,%d,%d,%d]", i ? "," : "", it[i].b, it[i].k_begin, it[i].k_end, it[i].slot);
    std::printf("]}");
  }
  std::printf("]\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def varlen_plans(tmp_path_factory):
    d = tmp_path_factory.mktemp("wsplan")
    src, exe = d / "plan.cpp", d / "plan"
    src.write_text(PLAN_CHECKER)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    return json.loads(subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout)


def test_varlen_items_cover_every_row_once(varlen_plans):
    """The work items of a per-sequence-length decode cover rows [0, lens[b]) of
    every sequence exactly once, each item within one sequence, no item empty
    or longer than kps (a whole number of tiles), and no more items than the
    workspace holds records."""
    for r in varlen_plans:
        B, R, kps, items = r["B"], r["R"], r["kps"], r["items"]
        assert r["kps2"] == kps and r["n2"] == r["n"] == len(items)
        assert kps % r["tile"] == 0 and kps > 0
        assert B <= len(items) <= R
        for b in range(B):
            spans = sorted((k0, k1) for (bb, k0, k1, _) in items if bb == b)
            assert spans[0][0] == 0 and spans[-1][1] == r["lens"][b], (b, spans)
            for (a0, a1), (c0, _) in zip(spans, spans[1:]):
                assert a1 == c0
            for k0, k1 in spans:
                assert 0 < k1 - k0 <= kps and k0 % kps == 0


def test_varlen_records_are_distinct_and_where_the_merge_reads(varlen_plans):
    """Record b holds the first piece of sequence b (the merge writes c^ of
    sequence b over it in place); the other pieces of b sit in records
    off[b] .. off[b+1]-1; no record is used twice; pieces of kps keys launch
    before the ragged ones, and those longest first."""
    for r in varlen_plans:
        B, R, off, items = r["B"], r["R"], r["off"], r["items"]
        slots = [it[3] for it in items]
        assert len(set(slots)) == len(slots) and all(0 <= s < R for s in slots)
        assert off[0] == B and off[B] == len(items)
        for b in range(B):
            mine = sorted((k0, s) for (bb, k0, _, s) in items if bb == b)
            assert mine[0] == (0, b)
            assert [s for _, s in mine[1:]] == list(range(off[b], off[b + 1]))
        sizes = [k1 - k0 for (_, k0, k1, _) in items]
        full = [s == r["kps"] for s in sizes]
        assert full == sorted(full, reverse=True)
        ragged = [s for s in sizes if s != r["kps"]]
        assert ragged == sorted(ragged, reverse=True)


def test_varlen_plan_balances_a_skewed_batch(varlen_plans):
    """One 128K-row sequence next to 31 of about 4K: the plan cuts the long one
    into many pieces instead of giving every CTA the split size of the longest
    sequence, so the largest item is far below 128K / (uniform split count)."""
    sk = [r for r in varlen_plans if r["B"] == 32][0]
    total = sum(sk["lens"])
    assert sk["kps"] <= 4 * total / 148
    assert max(k1 - k0 for (_, k0, k1, _) in sk["items"]) == sk["kps"]

"""Host-side launch plans of csrc/launch_plan.h (pure integer arithmetic),
compiled with g++ and checked on the CPU: the few-row GEMM plan of a decode
step's products and the CTA order of the prefill attention."""
import json
import os
import subprocess

import pytest

from tests.conftest import ROOT

CSRC = os.path.join(ROOT, "causal_head_latent_b200", "csrc")

CHECKER = r"""
#include <cstdio>
#include "launch_plan.h"
using namespace gmla;
int main() {
  std::printf("{\"few\":[");
  struct Case { int rows, batches, np, N[3], k_chunks; };
  const Case cases[] = {
      {32, 1, 3, {12288, 12288, 512}, 192},  // decode-step [Q | G | C], d_model = 12288
      {32, 1, 1, {12288, 0, 0}, 192},        // decode-step W_o
      {20, 1, 1, {16384, 0, 0}, 8},          // a few cached rows expanded to K only
      {20, 1, 2, {16384, 16384, 0}, 8},      // ... to K and V
      {7, 1, 3, {1536, 1536, 64}, 24},
      {33, 1, 1, {12288, 0, 0}, 192},        // more rows than the kernel holds
      {32, 2, 1, {12288, 0, 0}, 192},        // several batches
      {32, 1, 1, {12288, 0, 0}, 3},          // too few K chunks
      {32, 1, 1, {65536, 0, 0}, 192}};       // more tiles than SMs at any width
  bool first = true;
  for (const Case &c : cases) {
    const FewRowsPlan f = few_rows_plan(c.rows, c.batches, c.N, c.np, c.k_chunks, 148);
    std::printf("%s[%d,%d,%d]", first ? "" : ",", f.nb, f.sk, f.tiles);
    first = false;
  }
  // every single-problem width from 64 to 40000 (multiples of 64) at 32 rows
  std::printf("],\"sweep\":[");
  first = true;
  for (int n = 64; n <= 40000; n += 64) {
    const int N[1] = {n};
    const FewRowsPlan f = few_rows_plan(32, 1, N, 1, 16, 148);
    std::printf("%s[%d,%d,%d,%d]", first ? "" : ",", n, f.nb, f.sk, f.tiles);
    first = false;
  }
  std::printf("],\"group\":[");
  const long long tks[] = {1, 300, 4096, 8192, 16384, 65536, 131072, 1048576};
  first = true;
  for (long long tk : tks) {
    std::printf("%s[%lld,%d]", first ? "" : ",", tk, prefill_head_group(tk, 128));
    first = false;
  }
  std::printf("],\"order\":[");
  struct Ord { int BH, n_ct, G, causal; };
  const Ord ords[] = {{96, 32, 8, 1}, {192, 16, 16, 1}, {20, 8, 16, 1}, {21, 5, 16, 1}, {6, 3, 16, 0},
                      {7, 1, 3, 1}, {1, 4, 1, 1}, {13, 7, 4, 0}};
  first = true;
  for (const Ord &o : ords) {
    std::printf("%s{\"BH\":%d,\"n_ct\":%d,\"G\":%d,\"causal\":%d,\"map\":[", first ? "" : ",", o.BH, o.n_ct, o.G,
                o.causal);
    for (int idx = 0; idx < o.BH * o.n_ct; ++idx) {
      int bh = -1, ct = -1;
      prefill_cta_item(idx, o.BH, o.n_ct, o.G, o.causal != 0, &bh, &ct);
      std::printf("%s[%d,%d]", idx ? "," : "", bh, ct);
    }
    std::printf("]}");
    first = false;
  }
  std::printf("]}\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def plans(tmp_path_factory):
    d = tmp_path_factory.mktemp("launchplan")
    src, exe = d / "plan.cpp", d / "plan"
    src.write_text(CHECKER)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    return json.loads(subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout)


def test_few_row_plans_of_the_decode_step(plans):
    """The decode step at d_model = 12288: [Q | G | C] in 131 unsplit tiles of 192
    columns (98 of 256 would leave 50 SMs idle), W_o in 64 tiles of 192 split
    over two-CTA clusters (128 CTAs); the wide expansions keep 256-column tiles,
    split when two CTAs per tile still fit one wave; the kernel is not used for
    more than 32 rows, several batches, fewer than 4 K chunks per CTA, or more
    tiles than SMs."""
    assert plans["few"] == [[192, 1, 131], [192, 2, 64], [256, 2, 64], [256, 1, 128], [192, 2, 17],
                            [0, 0, 0], [0, 0, 0], [0, 0, 0], [0, 0, 0]]


def test_few_row_plan_invariants(plans):
    """For every width: the launch fits one wave of 148 SMs, covers N with its
    tiles, and no other choice (256 or 192 columns, split in 1 or 2) gives more CTAs."""
    for n, nb, sk, tiles in plans["sweep"]:
        if nb == 0:
            assert -(-n // 192) > 148  # not even unsplit 192-column tiles fit one wave
            continue
        assert sk * tiles <= 148 and tiles == -(-n // nb) and tiles * nb >= n
        best = max(s * -(-n // w) for w in (256, 192) for s in (1, 2) if s * -(-n // w) <= 148)
        assert sk * tiles == best


def test_prefill_head_groups(plans):
    """Groups of (b, h) pairs whose K and V take about 32 MB: 8 heads at 8K keys,
    16 (the cap) at 4K and below, one from 64K keys on."""
    assert dict(plans["group"]) == {1: 16, 300: 16, 4096: 16, 8192: 8, 16384: 4, 65536: 1, 131072: 1,
                                    1048576: 1}


def test_prefill_cta_order_covers_every_item_once(plans):
    """Every (b, h, query pair) gets exactly one CTA; the CTAs of a group of
    head pairs are contiguous in the launch, and within a group the query pairs
    go longest first (causal) or in order (non-causal) across the group's heads."""
    for o in plans["order"]:
        BH, n_ct, G, causal, m = o["BH"], o["n_ct"], o["G"], o["causal"], [tuple(x) for x in o["map"]]
        assert sorted(m) == [(bh, ct) for bh in range(BH) for ct in range(n_ct)]
        for idx, (bh, ct) in enumerate(m):
            assert bh // G == idx // (G * n_ct)  # group of pairs by launch position
        for g0 in range(0, BH, G):
            seq = [ct for (bh, ct) in m if g0 <= bh < g0 + G]
            assert seq == sorted(seq, reverse=bool(causal))

// Launch plans that are pure integer arithmetic (no CUDA types): shared by the
// kernels' host code (and, for the prefill's CTA order, the kernel itself) and
// checked on the CPU by the tests.
#pragma once

#ifdef __CUDACC__
#define GMLA_HD __host__ __device__
#else
#define GMLA_HD
#endif

namespace gmla {

// ---------------------------------------------------------------- few-row GEMM
// A product with at most kFewRowsMax output rows in one batch (a decode step:
// one new token per sequence) has fewer 128 x 256 tiles than SMs, so each CTA
// is capped by what it can pull in while the other SMs idle.  The few-row
// kernel takes tiles nb columns wide and may split each tile's K chunks over a
// cluster of sk CTAs.  The plan: the choice with the most CTAs within one wave
// of `sms`, the wider tile on a tie; nb = 0 when the kernel does not apply
// (more rows, several batches, fewer than 4 K chunks per CTA, or more tiles
// than SMs).
constexpr int kFewRowsMax = 32;
constexpr int kFewRowsSplitMax = 2;

struct FewRowsPlan {
  int nb = 0, sk = 0, tiles = 0;
};

inline FewRowsPlan few_rows_plan(int a_rows, int a_batches, const int *N, int n_problems, int k_chunks, int sms) {
  FewRowsPlan best;
  if (a_batches != 1 || a_rows > kFewRowsMax) return best;
  const int widths[2] = {256, 192};
  for (int w = 0; w < 2; ++w) {
    const int nb = widths[w];
    int tiles = 0;
    for (int i = 0; i < n_problems; ++i) tiles += (N[i] + nb - 1) / nb;
    for (int sk = kFewRowsSplitMax; sk >= 1; --sk) {
      if ((long long)sk * tiles > sms || k_chunks < 4 * sk) continue;
      if (sk * tiles > best.sk * best.tiles) best = FewRowsPlan{nb, sk, tiles};
      break;  // the largest split that fits gives this width its most CTAs
    }
  }
  return best;
}

// ---------------------------------------------------------------- prefill CTA order
// K and V of one head take Tk * head_dim * 4 bytes; the prefill launches its
// CTAs in groups of (b, h) pairs whose K and V take about kHeadGroupBytes
// (8 heads at 8K keys, one from 64K keys on), so that the K and V in flight
// stay in L2.
constexpr long long kHeadGroupBytes = 32ll << 20;

inline int prefill_head_group(long long Tk, int head_dim) {
  const long long kv_head = Tk * (long long)head_dim * 4;
  long long g = kHeadGroupBytes / (kv_head > 0 ? kv_head : 1);
  if (g < 1) g = 1;
  if (g > 16) g = 16;
  return (int)g;
}

// The (b, h) pair `bh` and query pair `ct` of CTA `idx` of a launch of
// BH * n_ct CTAs: groups of head_group pairs (the last group may be smaller),
// within a group the query pairs longest (latest) first across all of the
// group's pairs when causal, so that the launch ends on short CTAs.
GMLA_HD inline void prefill_cta_item(int idx, int BH, int n_ct, int head_group, bool causal, int *bh, int *ct) {
  const int per_group = head_group * n_ct;
  const int grp = idx / per_group, rg = idx % per_group;
  const int gsize = (BH - grp * head_group) < head_group ? (BH - grp * head_group) : head_group;
  const int ci = rg / gsize;
  *bh = grp * head_group + rg % gsize;
  *ct = causal ? (n_ct - 1 - ci) : ci;
}

}  // namespace gmla

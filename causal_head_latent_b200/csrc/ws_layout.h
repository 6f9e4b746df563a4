// Host-side layout of the caller workspaces (pure integer arithmetic, no CUDA).
//
// A workspace only has to be 16-byte aligned, but the tensor maps that some
// calls copy into it are read by TMA from global memory and must sit on a
// 64-byte boundary, and the float32 partial states are loaded 16 bytes at a
// time.  So every layout starts at the first 256-byte boundary at or after
// the caller's pointer, and each region is rounded up to 256 bytes; the sizes
// the *_workspace_size functions report include the 255 bytes this rounding
// may skip at the start.
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace gmla {

constexpr size_t kWsAlign = 256;
constexpr size_t kTensorMapBytes = 128;  // sizeof(CUtensorMap)
constexpr int kLatentTileKeys = 48;      // keys per tile of the latent decode kernel (48 or 64)

inline size_t ws_round(size_t x) { return (x + kWsAlign - 1) & ~(kWsAlign - 1); }

// Split count for B sequences of L keys in tiles of `tile_keys`: fill whole
// waves of the 148 SMs of a B200 (one CTA per SM) while keeping the float32
// partial states small next to the cache.  A pure function of (B, L) so that
// a workspace size never depends on the device.  Every split but the last
// holds keys_per_split keys (a multiple of tile_keys); none is empty.
inline void latent_plan(long long B, long long L, int tile_keys, int *n_splits, int *keys_per_split) {
  const long long KT = tile_keys;
  const long long tiles = (L + KT - 1) / KT;
  double best = 1e30;
  long long best_s = 1;
  for (long long s = 1; s <= 64 && s <= tiles; ++s) {
    const long long ctas = B * s;
    const long long waves = (ctas + 147) / 148;
    const double eff = (double)ctas / (double)(waves * 148);
    const double overhead = (double)s * 96 * 512 * 8 / ((double)L * 512 * 2 + 1.0);
    const double cost = 1.0 / eff + overhead;
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s;
    }
  }
  const long long kps = ((tiles + best_s - 1) / best_s) * KT;
  *n_splits = (int)((L + kps - 1) / kps);
  *keys_per_split = (int)kps;
}

// Per-sequence lengths: the rows [0, lens[b]) of every sequence are cut into
// work items of at most kps keys (a multiple of the tile), so that the CTAs of
// one launch stream about equally many latents whatever the length mix (a
// split plan from the longest length would leave the CTAs of short sequences
// idle).  Item (b, 0) keeps its partial state in record b; the other items of
// sequence b in records seq_off[b] .. seq_off[b+1]-1 (from B on).
struct LatentItem {
  int b, k_begin, k_end, slot;
};

// Records (items) a workspace holds for B sequences of at most Lmax rows:
// those of the split plan of Lmax, or two waves of the 148 SMs plus one per
// sequence, whichever is more (never more than the tiles there are).
inline long long latent_varlen_records(long long B, long long Lmax, int tile_keys) {
  int S, kps;
  latent_plan(B, Lmax, tile_keys, &S, &kps);
  const long long tiles = B * ((Lmax + tile_keys - 1) / tile_keys);
  long long two_waves = 2 * 148 + B;
  if (two_waves > tiles) two_waves = tiles;
  return (long long)S * B > two_waves ? (long long)S * B : two_waves;
}

// Items for lengths lens[0..B) (each >= 1): kps is chosen among the sizes that
// split the longest sequence into 1..256 pieces, by a model of the launch in
// units of one latent row: whole waves of 148 CTAs times (kps + 256, the
// per-CTA cost of loading q~ and storing a partial state) plus the merge's
// read of 192 per item spread over the SMs; only item counts <= cap qualify.
// Returns the item count; with `items` and `seq_off` (B+1 entries) non-null,
// also writes the items in launch order (longest first) and the offsets.
inline long long latent_varlen_plan(const long long *lens, long long B, int tile_keys, long long cap, int *kps_out,
                                    LatentItem *items, int *seq_off) {
  const long long KT = tile_keys;
  long long maxlen = 1;
  for (long long b = 0; b < B; ++b)
    if (lens[b] > maxlen) maxlen = lens[b];
  long long best_kps = ((maxlen + KT - 1) / KT) * KT;  // one item per sequence always fits (cap >= B)
  double best = 1e300;
  for (long long s = 1; s <= 256; ++s) {
    const long long kps = (((maxlen + s - 1) / s + KT - 1) / KT) * KT;
    long long n = 0;
    for (long long b = 0; b < B; ++b) n += (lens[b] + kps - 1) / kps;
    if (n > cap) continue;
    const double cost = (double)((n + 147) / 148) * (double)(kps + 256) + (double)n * 192.0 / 148.0;
    if (cost < best - 1e-9) {
      best = cost;
      best_kps = kps;
    }
  }
  const long long kps = best_kps;
  long long n = 0;
  for (long long b = 0; b < B; ++b) n += (lens[b] + kps - 1) / kps;
  *kps_out = (int)kps;
  if (items && seq_off) {
    // records: b for the first piece of sequence b, B.. for the others in sequence order
    long long next = B;
    for (long long b = 0; b < B; ++b) {
      seq_off[b] = (int)next;
      next += (lens[b] + kps - 1) / kps - 1;
    }
    seq_off[B] = (int)next;
    // launch order: the full pieces (kps keys) first, then the ragged last pieces, longest first
    long long k = 0;
    for (long long b = 0; b < B; ++b)
      for (long long k0 = 0; k0 + kps <= lens[b]; k0 += kps)
        items[k++] = LatentItem{(int)b, (int)k0, (int)(k0 + kps), (int)(k0 == 0 ? b : seq_off[b] + k0 / kps - 1)};
    const long long first_ragged = k;
    for (long long b = 0; b < B; ++b) {
      const long long k0 = (lens[b] / kps) * kps;
      if (k0 < lens[b]) items[k++] = LatentItem{(int)b, (int)k0, (int)lens[b], (int)(k0 == 0 ? b : seq_off[b] + k0 / kps - 1)};
    }
    // insertion sort of the ragged pieces by length, descending (at most B of them)
    for (long long i = first_ragged + 1; i < k; ++i) {
      const LatentItem t = items[i];
      long long j = i;
      while (j > first_ragged && items[j - 1].k_end - items[j - 1].k_begin < t.k_end - t.k_begin) {
        items[j] = items[j - 1];
        --j;
      }
      items[j] = t;
    }
  }
  return n;
}

// Offsets (bytes from the caller's pointer) of the regions of a latent-decode
// workspace: q~ bf16 [B,H,dc] | m, l float [R,H] | acc float [R,H,dc] | lse2
// float [B,H] | with per-sequence lengths also one tensor map and one int32
// length per sequence, R work items and B+1 record offsets.  R is the number
// of partial-state records: S*B for S splits of every sequence ([S,B] order),
// latent_varlen_records(...) with per-sequence lengths.  `end` is the first
// byte past the layout.
struct LatentLayout {
  size_t qt, pm, pl, pacc, lse2, maps, lens, items, offs, end;
};

inline LatentLayout latent_layout(uintptr_t base, long long B, long long H, long long dc, long long R,
                                  bool per_sequence) {
  LatentLayout o;
  size_t off = ws_round(base) - base;
  o.qt = off;
  off += ws_round(2 * (size_t)B * H * dc);
  o.pm = off;
  off += ws_round(sizeof(float) * (size_t)R * H);
  o.pl = off;
  off += ws_round(sizeof(float) * (size_t)R * H);
  o.pacc = off;
  off += ws_round(sizeof(float) * (size_t)R * H * dc);
  o.lse2 = off;
  off += ws_round(sizeof(float) * (size_t)B * H);
  o.maps = o.lens = o.items = o.offs = off;
  if (per_sequence) {
    off += ws_round((size_t)B * kTensorMapBytes);
    o.lens = off;
    off += ws_round((size_t)B * sizeof(int));
    o.items = off;
    off += ws_round((size_t)R * sizeof(LatentItem));
    o.offs = off;
    off += ws_round((size_t)(B + 1) * sizeof(int));
  }
  o.end = off;
  return o;
}

// Bytes a caller must provide for that layout at any 16-byte-aligned pointer.
inline size_t latent_layout_bytes(long long B, long long H, long long dc, long long R, bool per_sequence) {
  return (kWsAlign - 16) + latent_layout(0, B, H, dc, R, per_sequence).end;
}

// Prefill with per-sequence lengths: three tensor maps and two int32 lengths
// per sequence.
struct PrefillVarlenLayout {
  size_t maps, lens, end;
};

inline PrefillVarlenLayout prefill_varlen_layout(uintptr_t base, long long B) {
  PrefillVarlenLayout o;
  size_t off = ws_round(base) - base;
  o.maps = off;
  off += ws_round(3 * (size_t)B * kTensorMapBytes);
  o.lens = off;
  off += ws_round(2 * (size_t)B * sizeof(int));
  o.end = off;
  return o;
}

inline size_t prefill_varlen_layout_bytes(long long B) { return (kWsAlign - 16) + prefill_varlen_layout(0, B).end; }

// Gated output projection: the gated context sigmoid(G) (.) O, bf16 [M, N].
inline size_t gate_out_layout_offset(uintptr_t base) { return ws_round(base) - base; }
inline size_t gate_out_layout_bytes(long long M, long long N) { return (kWsAlign - 16) + ws_round(2 * (size_t)M * N); }

}  // namespace gmla

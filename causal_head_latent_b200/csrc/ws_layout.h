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

// Offsets (bytes from the caller's pointer) of the regions of a latent-decode
// workspace: q~ bf16 [B,H,dc] | m, l float [S,B,H] | acc float [S,B,H,dc] |
// lse2 float [B,H] | optionally one tensor map and one int32 length per
// sequence.  `end` is the first byte past the layout.
struct LatentLayout {
  size_t qt, pm, pl, pacc, lse2, maps, lens, end;
};

inline LatentLayout latent_layout(uintptr_t base, long long B, long long H, long long dc, long long S,
                                  bool per_sequence) {
  LatentLayout o;
  size_t off = ws_round(base) - base;
  o.qt = off;
  off += ws_round(2 * (size_t)B * H * dc);
  o.pm = off;
  off += ws_round(sizeof(float) * (size_t)S * B * H);
  o.pl = off;
  off += ws_round(sizeof(float) * (size_t)S * B * H);
  o.pacc = off;
  off += ws_round(sizeof(float) * (size_t)S * B * H * dc);
  o.lse2 = off;
  off += ws_round(sizeof(float) * (size_t)B * H);
  o.maps = o.lens = off;
  if (per_sequence) {
    off += ws_round((size_t)B * kTensorMapBytes);
    o.lens = off;
    off += ws_round((size_t)B * sizeof(int));
  }
  o.end = off;
  return o;
}

// Bytes a caller must provide for that layout at any 16-byte-aligned pointer.
inline size_t latent_layout_bytes(long long B, long long H, long long dc, long long S, bool per_sequence) {
  return (kWsAlign - 16) + latent_layout(0, B, H, dc, S, per_sequence).end;
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

// Decode over the latent cache with W_k absorbed into the query and W_v into
// the output.
//
// For a new token with query q (heads h = 0..H-1 of width D) and visible
// latents c_0..c_{L-1} ("Gated MLA" page: K = C W_k^T, V = C W_v^T), the
// head-h scores are q_h . (W_k^(h) c_s) = (W_k^(h)T q_h) . c_s and the head
// context is sum_s a_s W_v^(h) c_s = W_v^(h) (sum_s a_s c_s), with W^(h) the
// rows h*D .. h*D+D-1.  Three launches:
//   absorb   q~[b,h,:] = scale * log2(e) * W_k^(h)T q_h, stored as bfloat16
//   stream   tensor-core split-KV pass over the latents (attn_latent_tc.cu):
//            per split the running max m, sum l and acc[h,:] = sum_s p_s c_s
//   merge    exact log-sum-exp merge of the splits, c^ = acc / l (the
//            partial form over a key range stops here: c^ and its
//            log-sum-exp, which gmla_decode_combine later merges with the
//            states of other key ranges)
//   W_v      o_h = W_v^(h) c^_h, gate sigmoid(G), bfloat16 store.
// gmla_decode_combine, which has no scratch for c^, does the last two in one
// kernel (combine_kernel).
#include <math.h>

#include <mutex>
#include <vector>

#include "internal.h"
#include "ptx.cuh"
#include "ws_layout.h"

namespace gmla {

int launch_latent_tc(const CUtensorMap &tmQt, const CUtensorMap &tmC, const uint16_t *C, long long Lmax, int B, int L,
                     int k_base, int H, int dc, int n_splits, int keys_per_split, float *part_m, float *part_l,
                     float *part_acc, float *weights, int w_ld, const CUtensorMap *tmC_seq, const int *lens,
                     const LatentItem *items, int n_items, unsigned *status, cudaStream_t stream);
int latent_tc_tile_keys();

namespace latent {

constexpr int HD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- combine (gmla_decode_combine)
// Merge of n states and W_v in one kernel, for gmla_decode_combine, which has
// no scratch for c^.  grid (H, ceil(B / CB)), CT threads.  Phase 1: warp bb
// computes the weights 2^(m_s - M) / sum_s l_s 2^(m_s - M) of the states of
// sequence b0 + bb (lanes over s).  Phase 2: c^ = sum_s w_s acc_s over all
// (sequence, column) pairs into shared memory.  Phase 3: o_h = W_v^(h) c^ with
// W_v read in whole rows, then the gate and the bfloat16 store.
constexpr int CB = 8;
constexpr int CT = 256;
static_assert(CT / 32 == CB, "one warp per sequence in phase 1");

struct CombineParams {
  const float *part_m, *part_l, *part_acc;  // [S,B,H] (m scaled by m_scale to log2 units), [S,B,H] or null (= 1),
                                            // [S,B,H,dc]
  float m_scale;
  int n_splits, B, H, dc;
  const uint16_t *Wv, *G;
  uint16_t *O;
  float *lse2;  // [B,H] log2-domain log-sum-exp, may be null
};

__global__ void __launch_bounds__(CT) combine_kernel(const CombineParams P) {
  extern __shared__ __align__(16) float csm[];  // chat [CB][dc] | split weights [CB][n_splits]
  const int h = blockIdx.x, b0 = blockIdx.y * CB;
  const int nb = min(CB, P.B - b0);
  const int dc = P.dc, S = P.n_splits;
  float *chat = csm;
  float *wsp = csm + CB * dc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < nb) {
    const int b = b0 + warp;
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, P.part_m[((size_t)s * P.B + b) * P.H + h] * P.m_scale);
    M = warp_max(M);
    float Lsum = 0.f;
    for (int s = lane; s < S; s += 32) {
      const size_t i = ((size_t)s * P.B + b) * P.H + h;
      const float m = P.part_m[i] * P.m_scale;
      const float e = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
      wsp[warp * S + s] = e;
      Lsum += (P.part_l ? P.part_l[i] : 1.f) * e;
    }
    Lsum = warp_sum(Lsum);
    // no visible key in any state: every weight 0, c^ = 0, log-sum-exp -inf
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    __syncwarp();
    for (int s = lane; s < S; s += 32) wsp[warp * S + s] *= inv;
    if (lane == 0 && P.lse2) P.lse2[(size_t)b * P.H + h] = Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY;
  }
  __syncthreads();
  {
    const size_t split_stride4 = (size_t)P.B * P.H * dc / 4;
    for (int i4 = threadIdx.x; i4 < nb * dc / 4; i4 += CT) {
      const int bb = (i4 * 4) / dc, c = (i4 * 4) % dc;
      const float4 *src = reinterpret_cast<const float4 *>(P.part_acc + ((size_t)(b0 + bb) * P.H + h) * dc + c);
      const float *w = wsp + bb * S;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < S; s0 += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          // an empty state (weight 0) left no acc: never read it
          v[u] = (s0 + u < S && w[s0 + u] != 0.f) ? src[(size_t)(s0 + u) * split_stride4]
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float ws = (s0 + u < S) ? w[s0 + u] : 0.f;
          a.x = fmaf(ws, v[u].x, a.x);
          a.y = fmaf(ws, v[u].y, a.y);
          a.z = fmaf(ws, v[u].z, a.z);
          a.w = fmaf(ws, v[u].w, a.w);
        }
      }
      *reinterpret_cast<float4 *>(chat + bb * dc + c) = a;
    }
  }
  __syncthreads();
  // o_h[b, r] = sum_c W_v[h*128 + r, c] c^[b, c].  Warp w owns rows
  // 64*(w >> 2) .. +63 and sequences bp, bp+1 (bp = 2*(w & 3)); lane l owns the
  // columns 16l .. 16l+15 (d_c <= 512) of every row, so a warp reads whole rows
  // of W_v (coalesced) and keeps its columns of c^ in registers.  Per block of
  // 32 rows each lane holds 32 partial sums per sequence; a transpose-reduce
  // across the warp (31 shuffles) leaves lane l with the full sum of row l.
  const int bp = 2 * (warp & 3), rbase = 64 * (warp >> 2);
  const int c0 = 16 * lane;
  const bool cols_ok = c0 < dc;
  float cx[2][16];
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int e = 0; e < 16; ++e) cx[k][e] = (cols_ok && bp + k < nb) ? chat[(bp + k) * dc + c0 + e] : 0.f;
#pragma unroll 1
  for (int rb = 0; rb < 64; rb += 32) {
    float part[2][32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float w[16];
      if (cols_ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(P.Wv + ((size_t)h * HD + rbase + rb + i) * dc + c0);
        const uint4 v0 = src[0], v1 = src[1];
        const uint32_t ww[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w[2 * e] = __uint_as_float(ww[e] << 16);
          w[2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) a = fmaf(w[e], cx[k][e], a);
        part[k][i] = a;
      }
    }
    // transpose-reduce: after the step with offset o each lane keeps the half
    // of its rows whose index has lane's bit o, adding its partner's copy
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = up ? part[k][i] : part[k][i + o];
          const float keep = up ? part[k][i + o] : part[k][i];
          part[k][i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (bp + k < nb) {
        const size_t oi = (size_t)(b0 + bp + k) * P.H * HD + (size_t)h * HD + rbase + rb + lane;
        float v = part[k][0];
        if (P.G) v *= sigmoidf_(bf16_to_f32(P.G[oi]));
        P.O[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
  }
}

// ---------------------------------------------------------------- merge (decode path)
// The exact log-sum-exp merge of the S split states, one thread per float4 of
// the [B*H, d_c] state: thread i reads its four columns of every split (all
// loads in flight), the S maxima and sums of its (b, h) row (shared by the
// d_c/4 threads of the row: served from L1), and writes c^ = sum_s w_s acc_s
// -- in place over split 0 (each thread reads its own slot before writing it)
// or into the caller's buffer (partial form), with the row's log-sum-exp.
struct MergeParams {
  const float *part_m, *part_l;  // [S, BH]; part_l null: every sum is 1
  const float *part_acc;         // [S, BH, dc]
  float *chat;                   // [BH, dc]
  float m_scale;                 // to log2 units
  int S, BH, dc;
  float *lse2;                   // [BH] log2 domain, or null
  float *lse_nat;                // [BH] natural log, or null
  // Work-item records (null: S splits per sequence in [S, BH] order): the
  // states of sequence b are records b and seq_off[b] .. seq_off[b+1]-1 of
  // [R, H] (and [R, H, dc]); H heads per sequence.
  const int *seq_off;
  int H;
};

constexpr int MT = 256;

__global__ void __launch_bounds__(MT) merge_kernel(const MergeParams P) {
  const int per_row = P.dc / 4;
  const size_t i4 = blockIdx.x * (size_t)MT + threadIdx.x;
  if (i4 >= (size_t)P.BH * per_row) return;
  const size_t bh = i4 / per_row;
  const int col4 = (int)(i4 % per_row);
  // record of state s of this (b, h)
  int S = P.S;
  size_t b_seq = 0, h = bh, x0 = 0;
  if (P.seq_off) {
    b_seq = bh / P.H;
    h = bh % P.H;
    x0 = (size_t)P.seq_off[b_seq];
    S = 1 + (P.seq_off[b_seq + 1] - P.seq_off[b_seq]);
  }
  auto rec = [&](int st) -> size_t {
    if (!P.seq_off) return (size_t)st * P.BH + bh;
    return (st == 0 ? b_seq : x0 + st - 1) * (size_t)P.H + h;
  };
  float M = -INFINITY;
  for (int st = 0; st < S; ++st) M = fmaxf(M, P.part_m[rec(st)] * P.m_scale);
  const float4 *src = reinterpret_cast<const float4 *>(P.part_acc);
  float Lsum = 0.f;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < S; s0 += 8) {
    float e[8];
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int st = s0 + u;
      const size_t r = st < S ? rec(st) : 0;
      const float m = st < S ? P.part_m[r] * P.m_scale : -INFINITY;
      e[u] = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
      // an empty state (weight 0) left no acc: never read it
      v[u] = e[u] != 0.f ? src[r * per_row + col4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int st = s0 + u;
      if (st < S) Lsum += (P.part_l ? P.part_l[rec(st)] : 1.f) * e[u];
      a.x = fmaf(e[u], v[u].x, a.x);
      a.y = fmaf(e[u], v[u].y, a.y);
      a.z = fmaf(e[u], v[u].z, a.z);
      a.w = fmaf(e[u], v[u].w, a.w);
    }
  }
  // no visible key in any state: c^ = 0, log-sum-exp -inf
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  reinterpret_cast<float4 *>(P.chat)[i4] = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
  if (i4 % per_row == 0) {
    const float l2 = Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY;
    if (P.lse2) P.lse2[bh] = l2;
    if (P.lse_nat) P.lse_nat[bh] = l2 * kLn2;
  }
}

__global__ void weights_fix_kernel(float *w, const float *lse2, int BH, int L) {
  const size_t n = (size_t)BH * L;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    w[i] = fast_exp2(w[i] - lse2[i / L]);
}

// Per-sequence lengths: rows of [B, H, Lmax]; columns at or past lens[b] are 0.
__global__ void weights_fix_varlen_kernel(float *w, const float *lse2, const int *lens, int H, int BH, long long Lmax) {
  const size_t n = (size_t)BH * Lmax;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / Lmax;
    const long long col = (long long)(i % Lmax);
    w[i] = col < lens[r / H] ? fast_exp2(w[i] - lse2[r]) : 0.f;
  }
}

// The state of an empty key range: log-sum-exp -inf, c^ = 0.
__global__ void empty_state_kernel(float *lse, float *chat, size_t n_lse, size_t n_chat) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_chat; i += (size_t)gridDim.x * blockDim.x) {
    chat[i] = 0.f;
    if (i < n_lse) lse[i] = -INFINITY;
  }
}

}  // namespace latent

// ------------------------------------------------------------------ split planning and workspace

void latent_plan(long long B, long long L, int *n_splits, int *keys_per_split) {
  latent_plan(B, L, latent_tc_tile_keys(), n_splits, keys_per_split);
}

size_t latent_workspace_bytes(long long B, long long L, long long H, long long dc) {
  int S, kps;
  latent_plan(B, L, &S, &kps);
  return latent_layout_bytes(B, H, dc, (long long)S * B, false);
}

// With per-sequence lengths the workspace holds the states of up to
// latent_varlen_records(B, cache_len_max) work items, and per sequence a
// 128-byte tensor map, an int32 length and a record offset.
size_t latent_varlen_workspace_bytes(long long B, long long cache_len_max, long long H, long long dc) {
  return latent_layout_bytes(B, H, dc, latent_varlen_records(B, cache_len_max, latent_tc_tile_keys()), true);
}

// The launches for a given split plan (S splits of kps keys over the key
// range [a.k0, a.L)) and workspace; with per-sequence lengths (a.lens) the
// plan is the work-item plan of those lengths and S, kps are not used.
static int launch_attend_latent_plan(const LatentArgs &a, int S, int kps, cudaStream_t stream) {
  using namespace latent;
  static_assert(sizeof(CUtensorMap) == kTensorMapBytes, "tensor map size");
  static_assert(sizeof(LatentItem) == 16, "work item size");
  uint8_t *base = static_cast<uint8_t *>(a.workspace);
  const long long records =
      a.lens ? latent_varlen_records(a.B, a.cache_len_max, latent_tc_tile_keys()) : (long long)S * a.B;
  const LatentLayout lay = latent_layout(reinterpret_cast<uintptr_t>(base), a.B, a.H, a.dc, records, a.lens != nullptr);
  uint16_t *qt = reinterpret_cast<uint16_t *>(base + lay.qt);
  float *pm = reinterpret_cast<float *>(base + lay.pm);
  float *pl = reinterpret_cast<float *>(base + lay.pl);
  float *pacc = reinterpret_cast<float *>(base + lay.pacc);
  float *lse2 = reinterpret_cast<float *>(base + lay.lse2);
  CUtensorMap *maps = nullptr;
  int *lens_dev = nullptr, *offs_dev = nullptr;
  LatentItem *items_dev = nullptr;
  long long n_items = 0;
  if (a.lens) {
    // per-sequence 2-D latent maps (d_c, lens[b]), lengths, work items and record
    // offsets, copied before the launches; the map region starts on a 256-byte
    // boundary (TMA reads maps at 64-byte alignment)
    maps = reinterpret_cast<CUtensorMap *>(base + lay.maps);
    lens_dev = reinterpret_cast<int *>(base + lay.lens);
    items_dev = reinterpret_cast<LatentItem *>(base + lay.items);
    offs_dev = reinterpret_cast<int *>(base + lay.offs);
    std::vector<CUtensorMap> hm((size_t)a.B);
    std::vector<int> hl((size_t)a.B), ho((size_t)a.B + 1);
    for (int b = 0; b < a.B; ++b) {
      const long long dims[2] = {a.dc, a.lens[b]}, strides[1] = {a.dc};
      const unsigned box[2] = {64, (unsigned)latent_tc_tile_keys()};
      if (!make_tmap_bf16(&hm[b], a.C + (size_t)b * a.cache_len_max * a.dc, 2, dims, strides, box)) return -1;
      hl[b] = (int)a.lens[b];
    }
    int kps_v = 0;
    n_items = latent_varlen_plan(a.lens, a.B, latent_tc_tile_keys(), records, &kps_v, nullptr, nullptr);
    if (n_items < 1 || n_items > records) return -1;
    std::vector<LatentItem> hi((size_t)n_items);
    latent_varlen_plan(a.lens, a.B, latent_tc_tile_keys(), records, &kps_v, hi.data(), ho.data());
    S = 1;
    // pageable sources: the copies are staged before cudaMemcpyAsync returns
    if (cudaMemcpyAsync(maps, hm.data(), hm.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpyAsync(lens_dev, hl.data(), hl.size() * sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(items_dev, hi.data(), hi.size() * sizeof(LatentItem), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpyAsync(offs_dev, ho.data(), ho.size() * sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return -1;
  }

  if (launch_absorb_tc(a.Q, a.Wk, a.B, a.H, a.dc, a.scale * kLog2e, qt, a.status, stream) != 0) return -1;
  {
    CUtensorMap tq, tc;
    const long long dq[3] = {a.dc, a.H, a.B}, sq[2] = {a.dc, (long long)a.H * a.dc};
    const unsigned bq[3] = {64, 96, 1};
    if (!make_tmap_bf16(&tq, qt, 3, dq, sq, bq)) return -1;
    // The key extent is L (the end of the key range), not cache_len_max: rows of
    // a ragged last tile past L read as zeros, never as whatever the unwritten
    // cache rows hold.
    const long long dcm[3] = {a.dc, a.L, a.B}, scm[2] = {a.dc, a.cache_len_max * a.dc};
    const unsigned bc[3] = {64, (unsigned)latent_tc_tile_keys(), 1};
    if (!make_tmap_bf16(&tc, a.C, 3, dcm, scm, bc)) return -1;
    const int w_ld = a.lens ? (int)a.cache_len_max : a.L;
    if (launch_latent_tc(tq, tc, a.C, a.cache_len_max, a.B, a.L, (int)a.k0, a.H, a.dc, S, kps, pm, pl, pacc,
                         a.weights, w_ld, maps, lens_dev, items_dev, (int)n_items, a.status, stream) != 0)
      return -1;
  }
  {
    // merge the split states: in place over split 0 of the partial accumulators,
    // or into the caller's buffers for the partial form
    MergeParams M;
    M.part_m = pm;
    M.part_l = pl;
    M.part_acc = pacc;
    M.chat = a.out_chat ? a.out_chat : pacc;
    M.m_scale = 1.f;
    M.S = S;
    M.BH = a.B * a.H;
    M.dc = a.dc;
    M.lse2 = a.out_chat ? nullptr : lse2;
    M.lse_nat = a.out_lse;
    M.seq_off = offs_dev;
    M.H = a.H;
    const size_t n4 = (size_t)M.BH * a.dc / 4;
    merge_kernel<<<(unsigned)((n4 + MT - 1) / MT), MT, 0, stream>>>(M);
  }
  if (!a.out_chat && launch_wv_tc(pacc, a.Wv, a.G, a.O, a.B, a.H, a.dc, a.status, stream) != 0) return -1;
  if (a.weights && a.lens)
    weights_fix_varlen_kernel<<<4 * num_sms(), 256, 0, stream>>>(a.weights, lse2, lens_dev, a.H, a.B * a.H,
                                                                 a.cache_len_max);
  else if (a.weights)
    weights_fix_kernel<<<4 * num_sms(), 256, 0, stream>>>(a.weights, lse2, a.B * a.H, a.L);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_attend_latent(const LatentArgs &a, cudaStream_t stream) {
  int S, kps;
  latent_plan(a.B, a.lens ? a.cache_len_max : a.L - a.k0, &S, &kps);
  return launch_attend_latent_plan(a, S, kps, stream);
}

int launch_latent_empty_state(float *lse, float *chat, long long B, long long H, long long dc, cudaStream_t stream) {
  latent::empty_state_kernel<<<2 * num_sms(), 256, 0, stream>>>(lse, chat, (size_t)(B * H), (size_t)(B * H * dc));
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Merge n partial states (natural-log lse [n,B,H], c^ [n,B,H,dc]), apply
// W_v^(h) and the gate.
int launch_latent_combine(const float *lse, const float *chat, int n, int B, int H, int dc, const uint16_t *Wv,
                          const uint16_t *G, uint16_t *O, cudaStream_t stream) {
  using namespace latent;
  CombineParams P;
  P.part_m = lse;
  P.part_l = nullptr;
  P.part_acc = chat;
  P.m_scale = kLog2e;
  P.n_splits = n;
  P.B = B;
  P.H = H;
  P.dc = dc;
  P.Wv = Wv;
  P.G = G;
  P.O = O;
  P.lse2 = nullptr;
  combine_kernel<<<dim3(H, (B + CB - 1) / CB), CT, sizeof(float) * (CB * dc + CB * n), stream>>>(P);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// ------------------------------------------------------------------ decode without a caller workspace
//
// Some callers cannot allocate device memory when they decode: a runtime that
// reserved all of the device memory for its own pool up front, or host code
// that runs where the CUDA allocator must not be called (it can synchronise
// the device, or the caller holds a lock the allocator may wait on).  For
// them the decode scratch (q~, the per-split partial states and the
// log-sum-exp) lives in the fixed array below, which every GPU that loads this
// library holds until the process exits.
//
// Every call uses the same array and leaves its contents behind.  Each call
// overwrites all of the scratch it reads before reading it (q~ by the absorb
// kernel, every split's m, l and acc by the streaming kernel, the
// log-sum-exp by the combine kernel), so nothing needs clearing.  Calls whose
// GPU work overlaps -- on different streams, or from different host threads
// without ordering -- race on the array.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

static constexpr int kNoAllocMaxDevices = 64;
static void *g_decode_scratch_addr[kNoAllocMaxDevices];
static std::mutex g_decode_scratch_mu;

// Device address of the scratch array on the current device.  The symbol's
// name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.  The lookup also loads this
// file's device code on that device, which commits the array's memory; the
// per-device set-up of every entry point calls this, so the first call of
// any entry point on a device is the one that commits it.
void *latent_noalloc_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_decode_scratch_mu);
  if (!g_decode_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
    g_decode_scratch_addr[dev] = p;
  }
  return g_decode_scratch_addr[dev];
}

size_t latent_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Returns 0 on success, -1 on a CUDA error, -3 when the problem does not fit in
// the scratch array even with a single split.  Allocates nothing.
int launch_attend_latent_noalloc(const LatentArgs &args, cudaStream_t stream) {
  int S, kps;
  latent_plan(args.B, args.L, &S, &kps);
  // fewer splits when the default plan's partial states do not fit (the array
  // is 256-byte aligned, so the layout starts at its first byte)
  auto fits = [&](int s) {
    return latent_layout(0, args.B, args.H, args.dc, (long long)s * args.B, false).end <= kNoAllocScratchBytes;
  };
  while (S > 1 && !fits(S)) --S;
  if (!fits(S)) return -3;
  const int KT = latent_tc_tile_keys();
  const long long tiles = (args.L + KT - 1) / KT;
  kps = (int)(((tiles + S - 1) / S) * KT);
  S = (int)((args.L + kps - 1) / kps);  // no empty split
  void *scratch = latent_noalloc_scratch_address();
  if (!scratch) return -1;
  LatentArgs a = args;
  a.workspace = scratch;
  return launch_attend_latent_plan(a, S, kps, stream);
}

}  // namespace gmla

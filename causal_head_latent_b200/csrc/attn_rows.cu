// Attention for a few query rows over explicit K/V (decode mode), on CUDA cores.
//
// Decode attends one query to Tk cached keys ("Kimi K3 - Softmax over keys",
// decode mode: scores [B, 96, 1, 1001]), which is bound by reading K and V
// (one multiply-add per loaded element), so it streams K and V rather than
// using tensor cores.
//
// One CTA per (b, h, t) query row.  A producer warp streams the row's keys and
// values through shared memory in tiles of 64 keys by TMA (three stages of
// 16 KB of K and 16 KB of V, so about 192 KB per SM stay in flight with two
// CTAs resident), and 256 threads = 16 half-warps consume them: a half-warp
// owns one key at a time (16 lanes x 8 dims = one 128-wide head row, read
// from the 128-byte-swizzled tile), the half-warps take keys round-robin,
// keep a private online softmax state (max, sum, 8 accumulators per lane) and
// are merged exactly at the end through shared memory (log-sum-exp combine).
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace rows {

constexpr int HD = 128;
constexpr int CT = 256;                   // consumer threads
constexpr int THREADS = CT + 32;          // + the producer warp
constexpr int HALF_WARPS = CT / 16;
constexpr int KEYS = 64;                  // keys per tile
constexpr int UNROLL = KEYS / HALF_WARPS;  // keys per half-warp per tile
constexpr int STAGES = 3;
constexpr int HALF_BYTES = KEYS * 128;    // 64 keys x 64 dims, 128-byte swizzled
constexpr int TILE_BYTES = 2 * HALF_BYTES;
constexpr float kLog2e = 1.4426950408889634f;

struct Smem {
  uint8_t k[STAGES][TILE_BYTES];
  uint8_t v[STAGES][TILE_BYTES];
  uint64_t full[STAGES], empty[STAGES];
  float m[HALF_WARPS], l[HALF_WARPS];
  float acc[HALF_WARPS][HD];
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

struct Params {
  RowsArgs a;
  float scale_log2;
};

__device__ __forceinline__ void load8(const uint16_t *p, float (&f)[8]) {
  const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Dims 8*sub .. 8*sub+7 of key row r of a swizzled tile.
__device__ __forceinline__ void tile8(const uint8_t *tile, int r, int sub, float (&f)[8]) {
  const uint4 v = *reinterpret_cast<const uint4 *>(tile + (sub >> 3) * HALF_BYTES + r * 128 + (((sub & 7) ^ (r & 7)) << 4));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(THREADS) attn_rows_kernel(const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmV, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const RowsArgs &a = P.a;
  const int t = blockIdx.x % a.Tq;
  const int bh = blockIdx.x / a.Tq;
  const int b = bh / a.H, h = bh % a.H;
  const int pos = a.Tk - a.Tq + t;
  const int lim = a.causal ? min(pos, a.Tk - 1) : a.Tk - 1;  // last visible key
  const int n_tiles = lim / KEYS + 1;
  const float sl2 = P.scale_log2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], CT / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int hw = threadIdx.x / 16;   // half-warp index
  const int sub = threadIdx.x % 16;  // lane within the half-warp: dims [8*sub, 8*sub+8)
  float *wrow = a.weights ? a.weights + (((size_t)b * a.H + h) * a.Tq + t) * (size_t)a.Tk : nullptr;

  if (threadIdx.x >= CT) {
    // ---------------------------------------------------------------- producer
    if (threadIdx.x == CT) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (!mbar_wait(&sm.empty[s], ((j / STAGES) & 1) ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&sm.full[s], 2 * TILE_BYTES);
        for (int hc = 0; hc < 2; ++hc) {
          tma_load_4d(sm.k[s] + hc * HALF_BYTES, &tmK, &sm.full[s], hc * 64, j * KEYS, h, b);
          tma_load_4d(sm.v[s] + hc * HALF_BYTES, &tmV, &sm.full[s], hc * 64, j * KEYS, h, b);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    float q[8];
    load8(a.Q + b * a.qs[0] + t * a.qs[1] + h * a.qs[2] + sub * 8, q);
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % STAGES;
      // warp-uniform: the half-warp shuffles below need every lane of the warp
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (j / STAGES) & 1, a.status))) break;
      float x[UNROLL];
      float mx = m;
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int r = hw + u * HALF_WARPS;  // key within the tile
        const int key = j * KEYS + r;
        float kf[8];
        tile8(sm.k[s], r, sub, kf);
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) d = fmaf(q[i], kf[i], d);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o, 16);
        x[u] = key <= lim ? d * sl2 : -INFINITY;
        mx = fmaxf(mx, x[u]);
        if (wrow && key <= lim && sub == 0) wrow[key] = x[u];
      }
      const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int r = hw + u * HALF_WARPS;
        const float pu = (x[u] == -INFINITY) ? 0.f : fast_exp2(x[u] - mx);
        // P is rounded to bfloat16 before it multiplies V, as the eager path does.
        const float pb = __bfloat162float(__float2bfloat16_rn(pu));
        l += pu;
        if (pu != 0.f) {
          float vf[8];
          tile8(sm.v[s], r, sub, vf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(pb, vf[i], acc[i]);
        }
      }
      m = mx;
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.empty[s]);
    }
  }

  // merge the 16 half-warp states
  __syncwarp();  // lane 0 of the producer warp ran its loop alone
  if (threadIdx.x < CT) {
    if (sub == 0) {
      sm.m[hw] = m;
      sm.l[hw] = l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) sm.acc[hw][sub * 8 + i] = acc[i];
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < HALF_WARPS; ++i) M = fmaxf(M, sm.m[i]);
  float L = 0.f;
#pragma unroll
  for (int i = 0; i < HALF_WARPS; ++i) L += (sm.m[i] == -INFINITY) ? 0.f : sm.l[i] * fast_exp2(sm.m[i] - M);
  if (threadIdx.x < HD) {
    const int d = threadIdx.x;
    float o = 0.f;
#pragma unroll
    for (int i = 0; i < HALF_WARPS; ++i)
      if (sm.m[i] != -INFINITY) o += sm.acc[i][d] * fast_exp2(sm.m[i] - M);
    o /= L;
    if (a.G) o *= sigmoidf_(bf16_to_f32(a.G[((size_t)b * a.Tq + t) * (size_t)(a.H * HD) + (size_t)h * HD + d]));
    a.O[b * a.os[0] + t * a.os[1] + h * a.os[2] + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  }
  const float lg = M + __log2f(L);
  if (threadIdx.x == 0 && a.lse) a.lse[((size_t)b * a.H + h) * a.Tq + t] = lg * 0.6931471805599453f;
  if (wrow) {
    __syncthreads();  // raw scores written by other threads
    for (int s2 = threadIdx.x; s2 < a.Tk; s2 += THREADS) wrow[s2] = (s2 <= lim) ? fast_exp2(wrow[s2] - lg) : 0.f;
  }
}

}  // namespace rows

int launch_attn_rows(const RowsArgs &a, cudaStream_t stream) {
  using namespace rows;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(attn_rows_kernel), (int)kSmemBytes, kSmemRows)) return -1;
  Params P;
  P.a = a;
  P.scale_log2 = a.scale * kLog2e;
  const long long grid = (long long)a.B * a.H * a.Tq;
  if (grid <= 0) return 0;
  if (grid > 0x7fffffffLL) return -2;
  // K and V as (D, T, H, B) tiled maps: tiles of 64 keys x 64 dims
  CUtensorMap tk, tv;
  const long long dk[4] = {HD, a.Tk, a.H, a.B}, sk[3] = {a.ks[1], a.ks[2], a.ks[0]};
  const long long sv[3] = {a.vs[1], a.vs[2], a.vs[0]};
  const unsigned box[4] = {64, KEYS, 1, 1};
  if (!make_tmap_bf16(&tk, a.K, 4, dk, sk, box) || !make_tmap_bf16(&tv, a.V, 4, dk, sv, box)) return -1;
  attn_rows_kernel<<<(unsigned)grid, THREADS, kSmemBytes, stream>>>(tk, tv, P);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

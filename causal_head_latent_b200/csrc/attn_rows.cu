// Attention for a few query rows over explicit K/V (decode mode), on CUDA cores.
//
// Decode attends one query to Tk cached keys ("Kimi K3 - Softmax over keys",
// decode mode: scores [B, 96, 1, 1001]), which is bound by reading K and V
// (one multiply-add per loaded element), so it streams K and V with coalesced
// 16-byte loads rather than using tensor cores.
//
// One CTA per (b, h, t) query row, 256 threads = 16 half-warps.  A half-warp
// owns one key at a time (16 lanes x 8 dims = one 128-wide head row); the
// half-warps take keys round-robin, keep a private online softmax state
// (max, sum, 8 accumulators per lane) and are merged exactly at the end
// through shared memory (log-sum-exp combine).
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace rows {

constexpr int HD = 128;
constexpr int THREADS = 256;
constexpr int HALF_WARPS = THREADS / 16;
constexpr int UNROLL = 4;
constexpr float kLog2e = 1.4426950408889634f;

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

__global__ void __launch_bounds__(THREADS) attn_rows_kernel(const Params P) {
  const RowsArgs &a = P.a;
  const int t = blockIdx.x % a.Tq;
  const int bh = blockIdx.x / a.Tq;
  const int b = bh / a.H, h = bh % a.H;
  const int hw = threadIdx.x / 16;    // half-warp index
  const int sub = threadIdx.x % 16;   // lane within the half-warp: dims [8*sub, 8*sub+8)
  const int pos = a.Tk - a.Tq + t;
  const int lim = a.causal ? min(pos, a.Tk - 1) : a.Tk - 1;  // last visible key
  const float sl2 = P.scale_log2;

  float q[8];
  load8(a.Q + b * a.qs[0] + t * a.qs[1] + h * a.qs[2] + sub * 8, q);
  const uint16_t *kb = a.K + b * a.ks[0] + h * a.ks[2] + sub * 8;
  const uint16_t *vb = a.V + b * a.vs[0] + h * a.vs[2] + sub * 8;
  float *wrow = a.weights ? a.weights + (((size_t)b * a.H + h) * a.Tq + t) * (size_t)a.Tk : nullptr;

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  // The trip count depends only on lim, never on hw: both half-warps of a warp
  // run every iteration, since the full-warp shuffles below need all 32 lanes.
  for (int base = 0; base <= lim; base += HALF_WARPS * UNROLL) {
    const int s0 = base + hw;
    float kf[UNROLL][8], vf[UNROLL][8];
    bool valid[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int s = s0 + u * HALF_WARPS;
      valid[u] = s <= lim;
      if (valid[u]) {
        load8(kb + (long long)s * a.ks[1], kf[u]);
        load8(vb + (long long)s * a.vs[1], vf[u]);
      }
    }
    float x[UNROLL];
    float mx = m;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) d = fmaf(q[i], valid[u] ? kf[u][i] : 0.f, d);
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o, 16);
      x[u] = valid[u] ? d * sl2 : -INFINITY;
      mx = fmaxf(mx, x[u]);
      if (wrow && valid[u] && sub == 0) wrow[s0 + u * HALF_WARPS] = x[u];
    }
    const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const float pu = valid[u] ? fast_exp2(x[u] - mx) : 0.f;
      // P is rounded to bfloat16 before it multiplies V, as the eager path does.
      const float pb = __bfloat162float(__float2bfloat16_rn(pu));
      l += pu;
      if (valid[u]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(pb, vf[u][i], acc[i]);
      }
    }
    m = mx;
  }

  // merge the 16 half-warp states
  __shared__ float sm_m[HALF_WARPS], sm_l[HALF_WARPS];
  __shared__ float sm_acc[HALF_WARPS][HD];
  if (sub == 0) {
    sm_m[hw] = m;
    sm_l[hw] = l;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) sm_acc[hw][sub * 8 + i] = acc[i];
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < HALF_WARPS; ++i) M = fmaxf(M, sm_m[i]);
  float L = 0.f;
#pragma unroll
  for (int i = 0; i < HALF_WARPS; ++i) L += (sm_m[i] == -INFINITY) ? 0.f : sm_l[i] * fast_exp2(sm_m[i] - M);
  if (threadIdx.x < HD) {
    const int d = threadIdx.x;
    float o = 0.f;
#pragma unroll
    for (int i = 0; i < HALF_WARPS; ++i)
      if (sm_m[i] != -INFINITY) o += sm_acc[i][d] * fast_exp2(sm_m[i] - M);
    o /= L;
    if (a.G) o *= sigmoidf_(bf16_to_f32(a.G[((size_t)b * a.Tq + t) * (size_t)(a.H * HD) + (size_t)h * HD + d]));
    a.O[b * a.os[0] + t * a.os[1] + h * a.os[2] + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  }
  const float lg = M + __log2f(L);
  if (threadIdx.x == 0 && a.lse) a.lse[((size_t)b * a.H + h) * a.Tq + t] = lg * 0.6931471805599453f;
  if (wrow) {
    __syncthreads();  // raw scores written by other threads
    for (int s = threadIdx.x; s < a.Tk; s += THREADS) wrow[s] = (s <= lim) ? fast_exp2(wrow[s] - lg) : 0.f;
  }
}

}  // namespace rows

int launch_attn_rows(const RowsArgs &a, cudaStream_t stream) {
  rows::Params P;
  P.a = a;
  P.scale_log2 = a.scale * rows::kLog2e;
  const long long grid = (long long)a.B * a.H * a.Tq;
  if (grid <= 0) return 0;
  if (grid > 0x7fffffffLL) return -2;
  rows::attn_rows_kernel<<<(unsigned)grid, rows::THREADS, 0, stream>>>(P);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

// Decode over the latent cache with W_k absorbed into the query and W_v into
// the output.
//
// For a new token with query q (heads h = 0..H-1 of width D) and visible
// latents c_0..c_{L-1} ("Gated MLA" page: K = C W_k^T, V = C W_v^T), the
// head-h scores are q_h . (W_k^(h) c_s) = (W_k^(h)T q_h) . c_s and the head
// context is sum_s a_s W_v^(h) c_s = W_v^(h) (sum_s a_s c_s), with W^(h) the
// rows h*D .. h*D+D-1.  Three steps:
//   absorb   q~[b,h,:] = scale * log2(e) * W_k^(h)T q_h          (float32)
//   stream   per key split: running max m, sum l and acc[h,:] = sum_s p_s c_s
//            over the latents, every latent read once for all heads
//   combine  exact log-sum-exp merge of the splits, c^ = acc / l, then
//            o_h = W_v^(h) c^_h, gate sigmoid(G), bf16 store.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace latent {

constexpr int HD = 128;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- absorb
// grid (H, d_c / 128), 128 threads: thread j owns latent column c = 128*y + j.
__global__ void __launch_bounds__(128) absorb_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ Wk,
                                                     int B, int H, int dc, float sl2, float *__restrict__ qt) {
  extern __shared__ float qs[];  // [B][HD]
  const int h = blockIdx.x;
  const int c = blockIdx.y * 128 + threadIdx.x;
  for (int i = threadIdx.x; i < B * HD; i += 128) {
    const int b = i / HD, d = i % HD;
    qs[i] = bf16_to_f32(Q[(size_t)b * H * HD + (size_t)h * HD + d]);
  }
  __syncthreads();
  if (c >= dc) return;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int nb = min(32, B - b0);
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.f;
    for (int d = 0; d < HD; ++d) {
      const float w = bf16_to_f32(Wk[((size_t)h * HD + d) * dc + c]);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nb) acc[j] = fmaf(qs[(b0 + j) * HD + d], w, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nb) qt[((size_t)(b0 + j) * H + h) * dc + c] = acc[j] * sl2;
  }
}

// ---------------------------------------------------------------- stream (CUDA-core version)
// grid (n_splits, H / HG, B), 256 threads; HG heads per CTA, KT keys per tile.
constexpr int HG = 8;
constexpr int KT = 32;
constexpr int ST = 256;

struct StreamParams {
  const uint16_t *C;
  long long cache_len_max;
  int L, H, dc, n_splits, keys_per_split;
  const float *qt;       // [B,H,dc]
  float *part_m, *part_l, *part_acc;  // [S,B,H], [S,B,H], [S,B,H,dc]
  float *weights;        // optional raw scores [B,H,L]
  int B;
};

__global__ void __launch_bounds__(ST) stream_kernel(const StreamParams P) {
  extern __shared__ float sm[];
  const int dc = P.dc;
  float *q_s = sm;                 // [HG][dc]
  float *c_s = q_s + HG * dc;      // [KT][dc]
  float *p_s = c_s + KT * dc;      // [HG][KT]
  float *m_s = p_s + HG * KT;      // [HG]
  float *a_s = m_s + HG;           // [HG] rescale factors
  const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int h0 = hg * HG;
  const int k_begin = split * P.keys_per_split;
  const int k_end = min(P.L, k_begin + P.keys_per_split);
  for (int i = threadIdx.x; i < HG * dc; i += ST) {
    const int hh = i / dc, c = i % dc;
    q_s[i] = (h0 + hh < P.H) ? P.qt[((size_t)b * P.H + h0 + hh) * dc + c] : 0.f;
  }
  // each thread owns outputs (head hh, column c) for idx = tid + ST*j
  const int per = (HG * dc) / ST;  // dc multiple of 64 -> per = dc/32
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // meaningful in threads < HG
  if (threadIdx.x < HG) m_s[threadIdx.x] = -INFINITY;
  __syncthreads();
  for (int k0 = k_begin; k0 < k_end; k0 += KT) {
    const int nk = min(KT, k_end - k0);
    for (int i = threadIdx.x; i < KT * dc; i += ST) {
      const int kk = i / dc, c = i % dc;
      c_s[i] = kk < nk ? bf16_to_f32(P.C[((size_t)b * P.cache_len_max + k0 + kk) * dc + c]) : 0.f;
    }
    __syncthreads();
    // scores: thread -> (head, key)
    {
      const int hh = threadIdx.x / KT, kk = threadIdx.x % KT;
      float s = -INFINITY;
      if (kk < nk) {
        float d = 0.f;
        for (int c = 0; c < dc; ++c) d = fmaf(q_s[hh * dc + c], c_s[kk * dc + c], d);
        s = d;
        if (P.weights && h0 + hh < P.H) P.weights[((size_t)b * P.H + h0 + hh) * P.L + k0 + kk] = s;
      }
      p_s[hh * KT + kk] = s;
    }
    __syncthreads();
    if (threadIdx.x < HG) {
      const int hh = threadIdx.x;
      float mx = m_run;
      for (int kk = 0; kk < nk; ++kk) mx = fmaxf(mx, p_s[hh * KT + kk]);
      const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mx);
      float ls = 0.f;
      for (int kk = 0; kk < KT; ++kk) {
        const float pv = kk < nk ? fast_exp2(p_s[hh * KT + kk] - mx) : 0.f;
        ls += pv;
        p_s[hh * KT + kk] = __bfloat162float(__float2bfloat16_rn(pv));
      }
      l_run = l_run * alpha + ls;
      m_run = mx;
      a_s[hh] = alpha;
    }
    __syncthreads();
    for (int j = 0; j < per; ++j) {
      const int idx = threadIdx.x + ST * j;
      const int hh = idx / dc, c = idx % dc;
      float a = acc[j] * a_s[hh];
      for (int kk = 0; kk < nk; ++kk) a = fmaf(p_s[hh * KT + kk], c_s[kk * dc + c], a);
      acc[j] = a;
    }
    __syncthreads();
  }
  const size_t base = ((size_t)split * P.B + b) * P.H;
  if (threadIdx.x < HG && h0 + threadIdx.x < P.H) {
    P.part_m[base + h0 + threadIdx.x] = m_run;
    P.part_l[base + h0 + threadIdx.x] = l_run;
  }
  for (int j = 0; j < per; ++j) {
    const int idx = threadIdx.x + ST * j;
    const int hh = idx / dc, c = idx % dc;
    if (h0 + hh < P.H) P.part_acc[(base + h0 + hh) * dc + c] = acc[j];
  }
}

// ---------------------------------------------------------------- combine + W_v + gate
// grid (H, B), 128 threads (one per output channel of the head).
struct CombineParams {
  const float *part_m, *part_l, *part_acc;
  int n_splits, B, H, dc;
  const uint16_t *Wv, *G;
  uint16_t *O;
  float *lse2;  // [B,H] log2-domain lse (for debug weights)
};

__global__ void __launch_bounds__(128) combine_kernel(const CombineParams P) {
  extern __shared__ float chat[];  // [dc]
  const int h = blockIdx.x, b = blockIdx.y;
  const int dc = P.dc;
  float M = -INFINITY;
  for (int s = 0; s < P.n_splits; ++s) M = fmaxf(M, P.part_m[((size_t)s * P.B + b) * P.H + h]);
  float Lsum = 0.f;
  for (int s = 0; s < P.n_splits; ++s) {
    const float ms = P.part_m[((size_t)s * P.B + b) * P.H + h];
    if (ms != -INFINITY) Lsum += P.part_l[((size_t)s * P.B + b) * P.H + h] * fast_exp2(ms - M);
  }
  const float inv = 1.f / Lsum;
  for (int c = threadIdx.x; c < dc; c += 128) {
    float a = 0.f;
    for (int s = 0; s < P.n_splits; ++s) {
      const size_t i = ((size_t)s * P.B + b) * P.H + h;
      const float ms = P.part_m[i];
      if (ms != -INFINITY) a += P.part_acc[i * dc + c] * fast_exp2(ms - M);
    }
    chat[c] = a * inv;
  }
  if (threadIdx.x == 0 && P.lse2) P.lse2[(size_t)b * P.H + h] = M + __log2f(Lsum);
  __syncthreads();
  const int i = threadIdx.x;
  const uint16_t *w = P.Wv + ((size_t)h * HD + i) * dc;
  float o = 0.f;
  for (int c = 0; c < dc; c += 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(w + c);
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o = fmaf(__uint_as_float(ww[e] << 16), chat[c + 2 * e], o);
      o = fmaf(__uint_as_float(ww[e] & 0xFFFF0000u), chat[c + 2 * e + 1], o);
    }
  }
  const size_t oi = (size_t)b * P.H * HD + (size_t)h * HD + i;
  if (P.G) o *= sigmoidf_(bf16_to_f32(P.G[oi]));
  P.O[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
}

__global__ void weights_fix_kernel(float *w, const float *lse2, int BH, int L) {
  const size_t n = (size_t)BH * L;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    w[i] = fast_exp2(w[i] - lse2[i / L]);
}

}  // namespace latent

// Workspace layout (bytes, each region 256-aligned):
//   q~  float [B,H,dc] | m, l float [S,B,H] each | acc float [S,B,H,dc] | lse2 float [B,H]
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int latent_num_splits(long long B, long long L) {
  // enough CTAs (splits x head groups x batches) to fill the GPU a few times
  long long s = (4LL * num_sms() + B * 12 - 1) / (B * 12);
  if (s < 1) s = 1;
  long long max_s = (L + 255) / 256;
  if (s > max_s) s = max_s;
  if (s > 256) s = 256;
  return (int)s;
}

size_t latent_workspace_bytes(long long B, long long L, long long H, long long dc) {
  const long long S = latent_num_splits(B, L);
  return align256(sizeof(float) * B * H * dc) + 2 * align256(sizeof(float) * S * B * H) +
         align256(sizeof(float) * S * B * H * dc) + align256(sizeof(float) * B * H);
}

int launch_attend_latent(const LatentArgs &a, cudaStream_t stream) {
  using namespace latent;
  const int S = latent_num_splits(a.B, a.L);
  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  float *qt = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * a.B * a.H * a.dc);
  float *pm = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H);
  float *pl = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H);
  float *pacc = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H * a.dc);
  float *lse2 = reinterpret_cast<float *>(ws);

  const float sl2 = a.scale * kLog2e;
  {
    const size_t shm = sizeof(float) * a.B * HD;
    if (shm > 48 * 1024) cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    absorb_kernel<<<dim3(a.H, (a.dc + 127) / 128), 128, shm, stream>>>(a.Q, a.Wk, a.B, a.H, a.dc, sl2, qt);
  }
  {
    StreamParams P;
    P.C = a.C;
    P.cache_len_max = a.cache_len_max;
    P.L = a.L;
    P.H = a.H;
    P.dc = a.dc;
    P.n_splits = S;
    P.keys_per_split = (int)(((a.L + S - 1) / S + KT - 1) / KT * KT);
    P.qt = qt;
    P.part_m = pm;
    P.part_l = pl;
    P.part_acc = pacc;
    P.weights = a.weights;
    P.B = a.B;
    const size_t shm = sizeof(float) * ((size_t)HG * a.dc + (size_t)KT * a.dc + HG * KT + 2 * HG);
    cudaFuncSetAttribute(stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    stream_kernel<<<dim3(S, (a.H + HG - 1) / HG, a.B), ST, shm, stream>>>(P);
  }
  {
    CombineParams P;
    P.part_m = pm;
    P.part_l = pl;
    P.part_acc = pacc;
    P.n_splits = S;
    P.B = a.B;
    P.H = a.H;
    P.dc = a.dc;
    P.Wv = a.Wv;
    P.G = a.G;
    P.O = a.O;
    P.lse2 = lse2;
    combine_kernel<<<dim3(a.H, a.B), 128, sizeof(float) * a.dc, stream>>>(P);
  }
  if (a.weights) weights_fix_kernel<<<4 * num_sms(), 256, 0, stream>>>(a.weights, lse2, a.B * a.H, a.L);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

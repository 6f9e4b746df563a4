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
//   combine  exact log-sum-exp merge of the splits, c^ = acc / l, then
//            o_h = W_v^(h) c^_h, gate sigmoid(G), bfloat16 store.
#include <mutex>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace gmla {

int launch_latent_tc(const CUtensorMap &tmQt, const CUtensorMap &tmC, const uint16_t *C, long long Lmax, int B, int L,
                     int H, int dc, int n_splits, int keys_per_split, float *part_m, float *part_l, float *part_acc,
                     float *weights, int w_ld, const CUtensorMap *tmC_seq, const int *lens, unsigned *status,
                     cudaStream_t stream);
int latent_tc_tile_keys();

namespace latent {

constexpr int HD = 128;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- absorb
// grid (H, ceil(d_c / 128)), 128 threads: thread j owns latent column c = 128*y + j.
__global__ void __launch_bounds__(128) absorb_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ Wk,
                                                     int B, int H, int dc, float sl2, uint16_t *__restrict__ qt) {
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
    // four rows d of W_k per step, so q is read from shared memory as one
    // 16-byte broadcast per sequence instead of four
#pragma unroll 1
    for (int d = 0; d < HD; d += 4) {
      float w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = bf16_to_f32(Wk[((size_t)h * HD + d + e) * dc + c]);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nb) {
          const float4 q4 = *reinterpret_cast<const float4 *>(qs + (b0 + j) * HD + d);
          acc[j] = fmaf(q4.x, w[0], acc[j]);
          acc[j] = fmaf(q4.y, w[1], acc[j]);
          acc[j] = fmaf(q4.z, w[2], acc[j]);
          acc[j] = fmaf(q4.w, w[3], acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nb) qt[((size_t)(b0 + j) * H + h) * dc + c] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j] * sl2));
  }
}

// ---------------------------------------------------------------- combine + W_v + gate
// grid (H, ceil(B / CB)), 128 threads (one per output channel of the head).
constexpr int CB = 8;

struct CombineParams {
  const float *part_m, *part_l, *part_acc;
  int n_splits, B, H, dc;
  const uint16_t *Wv, *G;
  uint16_t *O;
  float *lse2;  // [B,H] log2-domain log-sum-exp (for the debug weights)
};

// grid (H, ceil(B / CB)), CT threads.  Per-split weights exp2(m_s - M) / L are
// computed once per sequence; the merge runs over all (sequence, column) pairs;
// two threads share one output row of W_v^(h) (one half of d_c each).
constexpr int CT = 256;

__global__ void __launch_bounds__(CT) combine_kernel(const CombineParams P) {
  extern __shared__ float sm[];  // chat [CB][dc] | split weights [CB][n_splits]
  const int h = blockIdx.x, b0 = blockIdx.y * CB;
  const int nb = min(CB, P.B - b0);
  const int dc = P.dc, S = P.n_splits;
  float *chat = sm;
  float *wsp = sm + CB * dc;
  if (threadIdx.x < nb) {
    const int b = b0 + threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, P.part_m[((size_t)s * P.B + b) * P.H + h]);
    float Lsum = 0.f;
    for (int s = 0; s < S; ++s) {
      const size_t i = ((size_t)s * P.B + b) * P.H + h;
      const float e = (P.part_m[i] == -INFINITY) ? 0.f : fast_exp2(P.part_m[i] - M);
      wsp[threadIdx.x * S + s] = e;
      Lsum += P.part_l[i] * e;
    }
    const float inv = 1.f / Lsum;
    for (int s = 0; s < S; ++s) wsp[threadIdx.x * S + s] *= inv;
    if (P.lse2) P.lse2[(size_t)b * P.H + h] = M + __log2f(Lsum);
  }
  __syncthreads();
  // c^ = sum_s w_s acc_s: four latent columns per thread (16-byte loads) and
  // eight splits' loads in flight before their multiply-adds.
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
          // an empty split (weight 0) left no acc: never read it
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
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int c_lo = half * (dc / 2), c_hi = c_lo + dc / 2;
  const uint16_t *w = P.Wv + ((size_t)h * HD + r) * dc;
  float o[CB];
#pragma unroll
  for (int bb = 0; bb < CB; ++bb) o[bb] = 0.f;
#pragma unroll 4
  for (int c = c_lo; c < c_hi; c += 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(w + c);
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float w0 = __uint_as_float(ww[e] << 16), w1 = __uint_as_float(ww[e] & 0xFFFF0000u);
#pragma unroll
      for (int bb = 0; bb < CB; ++bb) {
        if (bb < nb) {
          o[bb] = fmaf(w0, chat[bb * dc + c + 2 * e], o[bb]);
          o[bb] = fmaf(w1, chat[bb * dc + c + 2 * e + 1], o[bb]);
        }
      }
    }
  }
#pragma unroll
  for (int bb = 0; bb < CB; ++bb) o[bb] += __shfl_xor_sync(0xffffffffu, o[bb], 1);
  if (half == 0) {
#pragma unroll
    for (int bb = 0; bb < CB; ++bb) {
      if (bb < nb) {
        const size_t oi = (size_t)(b0 + bb) * P.H * HD + (size_t)h * HD + r;
        float v = o[bb];
        if (P.G) v *= sigmoidf_(bf16_to_f32(P.G[oi]));
        P.O[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
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

}  // namespace latent

// ------------------------------------------------------------------ split planning and workspace

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split count for B sequences of L keys: fill whole waves of the 148 SMs of a
// B200 (one CTA per SM) while keeping the float32 partial states small next to
// the cache.  A pure function of (B, L) so the workspace size never depends on
// the device.
void latent_plan(long long B, long long L, int *n_splits, int *keys_per_split) {
  const int KT = latent_tc_tile_keys();
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
  long long kps = ((tiles + best_s - 1) / best_s) * KT;
  long long s = (L + kps - 1) / kps;  // no empty split
  *n_splits = (int)s;
  *keys_per_split = (int)kps;
}

// Workspace layout (each region 256-byte aligned):
//   q~ bf16 [B,H,dc] | m, l float [S,B,H] each | acc float [S,B,H,dc] | lse2 float [B,H]
static size_t latent_workspace_bytes_for(long long B, long long H, long long dc, long long S) {
  return align256(2 * B * H * dc) + 2 * align256(sizeof(float) * S * B * H) + align256(sizeof(float) * S * B * H * dc) +
         align256(sizeof(float) * B * H);
}

size_t latent_workspace_bytes(long long B, long long L, long long H, long long dc) {
  int S, kps;
  latent_plan(B, L, &S, &kps);
  return latent_workspace_bytes_for(B, H, dc, S);
}

// With per-sequence lengths the plan follows cache_len_max, and the workspace
// also holds one 128-byte tensor map and one int32 length per sequence.
size_t latent_varlen_workspace_bytes(long long B, long long cache_len_max, long long H, long long dc) {
  return latent_workspace_bytes(B, cache_len_max, H, dc) + align256((size_t)B * sizeof(CUtensorMap)) +
         align256((size_t)B * sizeof(int));
}

// The three launches for a given split plan (S splits of kps keys) and workspace.
static int launch_attend_latent_plan(const LatentArgs &a, int S, int kps, cudaStream_t stream) {
  using namespace latent;
  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  uint16_t *qt = reinterpret_cast<uint16_t *>(ws);
  ws += align256(2 * (size_t)a.B * a.H * a.dc);
  float *pm = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H);
  float *pl = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H);
  float *pacc = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)S * a.B * a.H * a.dc);
  float *lse2 = reinterpret_cast<float *>(ws);
  ws += align256(sizeof(float) * (size_t)a.B * a.H);
  CUtensorMap *maps = nullptr;
  int *lens_dev = nullptr;
  if (a.lens) {
    // per-sequence 2-D latent maps (d_c, lens[b]) and lengths, copied before the launches
    maps = reinterpret_cast<CUtensorMap *>(ws);
    ws += align256((size_t)a.B * sizeof(CUtensorMap));
    lens_dev = reinterpret_cast<int *>(ws);
    std::vector<CUtensorMap> hm((size_t)a.B);
    std::vector<int> hl((size_t)a.B);
    for (int b = 0; b < a.B; ++b) {
      const long long dims[2] = {a.dc, a.lens[b]}, strides[1] = {a.dc};
      const unsigned box[2] = {64, (unsigned)latent_tc_tile_keys()};
      if (!make_tmap_bf16(&hm[b], a.C + (size_t)b * a.cache_len_max * a.dc, 2, dims, strides, box)) return -1;
      hl[b] = (int)a.lens[b];
    }
    // pageable sources: the copies are staged before cudaMemcpyAsync returns
    if (cudaMemcpyAsync(maps, hm.data(), hm.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpyAsync(lens_dev, hl.data(), hl.size() * sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return -1;
  }

  {
    const size_t shm = sizeof(float) * a.B * HD;
    if (shm > 48 * 1024 &&
        cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm) != cudaSuccess)
      return -1;
    absorb_kernel<<<dim3(a.H, (a.dc + 127) / 128), 128, shm, stream>>>(a.Q, a.Wk, a.B, a.H, a.dc,
                                                                      a.scale * kLog2e, qt);
  }
  {
    CUtensorMap tq, tc;
    const long long dq[3] = {a.dc, a.H, a.B}, sq[2] = {a.dc, (long long)a.H * a.dc};
    const unsigned bq[3] = {64, 96, 1};
    if (!make_tmap_bf16(&tq, qt, 3, dq, sq, bq)) return -1;
    // The key extent is L, not cache_len_max: rows of a ragged last tile past
    // L read as zeros, never as whatever the unwritten cache rows hold.
    const long long dcm[3] = {a.dc, a.L, a.B}, scm[2] = {a.dc, a.cache_len_max * a.dc};
    const unsigned bc[3] = {64, (unsigned)latent_tc_tile_keys(), 1};
    if (!make_tmap_bf16(&tc, a.C, 3, dcm, scm, bc)) return -1;
    const int w_ld = a.lens ? (int)a.cache_len_max : a.L;
    if (launch_latent_tc(tq, tc, a.C, a.cache_len_max, a.B, a.L, a.H, a.dc, S, kps, pm, pl, pacc, a.weights, w_ld, maps,
                         lens_dev, a.status, stream) != 0)
      return -1;
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
    combine_kernel<<<dim3(a.H, (a.B + CB - 1) / CB), CT, sizeof(float) * (CB * a.dc + CB * S), stream>>>(P);
  }
  if (a.weights && a.lens)
    weights_fix_varlen_kernel<<<4 * num_sms(), 256, 0, stream>>>(a.weights, lse2, lens_dev, a.H, a.B * a.H,
                                                                 a.cache_len_max);
  else if (a.weights)
    weights_fix_kernel<<<4 * num_sms(), 256, 0, stream>>>(a.weights, lse2, a.B * a.H, a.L);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_attend_latent(const LatentArgs &a, cudaStream_t stream) {
  int S, kps;
  latent_plan(a.B, a.lens ? a.cache_len_max : a.L, &S, &kps);
  return launch_attend_latent_plan(a, S, kps, stream);
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
// device (with that device current) and cached.
static void *decode_scratch_address() {
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
  // fewer splits when the default plan's partial states do not fit
  while (S > 1 && latent_workspace_bytes_for(args.B, args.H, args.dc, S) > kNoAllocScratchBytes) --S;
  if (latent_workspace_bytes_for(args.B, args.H, args.dc, S) > kNoAllocScratchBytes) return -3;
  const int KT = latent_tc_tile_keys();
  const long long tiles = (args.L + KT - 1) / KT;
  kps = (int)(((tiles + S - 1) / S) * KT);
  S = (int)((args.L + kps - 1) / kps);  // no empty split
  void *scratch = decode_scratch_address();
  if (!scratch) return -1;
  LatentArgs a = args;
  a.workspace = scratch;
  return launch_attend_latent_plan(a, S, kps, stream);
}

}  // namespace gmla

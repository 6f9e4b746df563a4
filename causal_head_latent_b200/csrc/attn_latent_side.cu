// The two small products around the latent-cache decode, on tcgen05 tensor
// cores ("Gated MLA" page, "Start from familiar attention": K = C W_k^T and
// V = C W_v^T, folded into the query and the output by associativity):
//
//   absorb:  q~[b, h, c] = s * sum_r q[b, 128h + r] W_k[128h + r, c]
//            (s = scale * log2 e; the decode's scores are then base-2 logits)
//   W_v:     o[b, 128h + r] = sigmoid(G[b, 128h + r]) * sum_c W_v[128h + r, c] c^[b, h, c]
//
// The products are M = 128 x N = 32 MMAs accumulating in 32 TMEM columns, with
// W^(h) brought into shared memory by TMA in 64-column chunks:
//   absorb  one CTA per (head h, 128 columns c of d_c, 32 sequences):
//           D[c, b] = A B with A = 128 columns of W_k^(h) read MN-major (c
//           contiguous), B = the 32 query rows of head h (K-major), K = 128;
//   W_v     one CTA per (head h, 32 sequences): D[r, b] with A = W_v^(h)
//           (K-major, 128 KB at d_c = 512), B = c^ of the 32 sequences, K = d_c.
// c^ is float32; it is split into c^ = hi + lo with hi = bf16(c^) and lo =
// bf16(c^ - hi), and both halves go through the MMA (2 x d_c / 16 of them), so
// the product keeps about 16 bits of c^ instead of bf16's 8.  Both kernels are
// bound by reading W^(h) once per CTA (about 3 us at d_c = 512, B <= 32).
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace side {

constexpr int HD = 128;
constexpr int NB = 32;                    // sequences per CTA (the MMA's N)
constexpr int WCHUNK = 128 * 64 * 2;      // 128 rows x 64 columns of W, 128-byte swizzled
constexpr int MAX_CHUNKS = 8;             // d_c <= 512
constexpr int BCHUNK = NB * 64 * 2;       // 32 rows x 64 columns of a B operand
constexpr int THREADS = 128;

struct SmemAbsorb {
  uint8_t w[2][WCHUNK];   // W_k^(h), columns c in [128 y + 64k, + 64) of all 128 rows r
  uint8_t q[2][BCHUNK];   // the 32 query rows of head h, r in [64j, 64j + 64)
  uint64_t full, done;
  uint32_t tmem_base;
};
struct SmemWv {
  uint8_t w[MAX_CHUNKS][WCHUNK];    // W_v^(h): chunk k holds columns c in [64k, 64k + 64) of all 128 rows r
  uint8_t hi[MAX_CHUNKS][BCHUNK];   // bf16(c^) of the 32 sequences, same column chunks
  uint8_t lo[MAX_CHUNKS][BCHUNK];   // bf16(c^ - hi)
  uint64_t full, done;
  uint32_t tmem_base;
};
constexpr size_t kSmemAbsorb = sizeof(SmemAbsorb) + 1024;
constexpr size_t kSmemWvTc = sizeof(SmemWv) + 1024;

struct Params {
  const float *chat;  // W_v: [B, H, dc] float32
  const uint16_t *G;  // W_v: optional gate logits [B, H*128]
  uint16_t *out;      // absorb: q~ [B, H, dc]; W_v: O [B, H*128]
  int B, H, dc;
  float sl2;          // absorb: scale * log2 e
  unsigned *status;
};

template <typename S>
__device__ __forceinline__ S &smem_of(uint8_t *raw) {
  return *reinterpret_cast<S *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__global__ void __launch_bounds__(THREADS, 1)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmQ, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  SmemAbsorb &sm = smem_of<SmemAbsorb>(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x, c0 = blockIdx.y * 128, b0 = blockIdx.z * NB;
  const int nchunk = min(2, (p.dc - c0) / 64);  // 1 or 2 (d_c is a multiple of 64)
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, NB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&sm.full, (uint32_t)(nchunk * WCHUNK + 2 * BCHUNK));
    for (int k = 0; k < nchunk; ++k) tma_load_2d(sm.w[k], &tmW, &sm.full, c0 + 64 * k, HD * h);
    for (int j = 0; j < 2; ++j) tma_load_2d(sm.q[j], &tmQ, &sm.full, HD * h + 64 * j, b0);
    if (mbar_wait(&sm.full, 0, p.status)) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, NB, true, false);
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        // A: the 128 columns c (two 64-wide chunks, LBO apart; a missing second chunk only
        // feeds rows c >= d_c, which are not stored), K-rows r = 16 kk ..
        const uint64_t a = sdesc_sw128(smem_u32(sm.w[0]) + kk * 2048, WCHUNK, 1024);
        const uint64_t bq = sdesc_sw128(smem_u32(sm.q[kk >> 2]) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(tmem, a, bq, idesc, kk > 0);
      }
    }
    umma_commit(&sm.done);
  }
  __syncwarp();
  const bool ok = mbar_wait(&sm.done, 0, p.status);
  tc_fence_after();
  float v[32];
  tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
  const int c = c0 + 32 * warp + lane;
  if (ok && c < p.dc) {
#pragma unroll
    for (int j = 0; j < NB; ++j)
      if (b0 + j < p.B)
        p.out[((size_t)(b0 + j) * p.H + h) * p.dc + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j] * p.sl2));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NB);
  }
}

__global__ void __launch_bounds__(THREADS, 1) wv_tc_kernel(const __grid_constant__ CUtensorMap tmW, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  SmemWv &sm = smem_of<SmemWv>(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x, b0 = blockIdx.y * NB;
  const int nchunk = p.dc / 64;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, NB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&sm.full, (uint32_t)(nchunk * WCHUNK));
    for (int k = 0; k < nchunk; ++k) tma_load_2d(sm.w[k], &tmW, &sm.full, 64 * k, HD * h);
  }
  // c^ of the 32 sequences as bf16 hi and lo parts, K-major in the 128-byte swizzle:
  // sequence b, columns 8u .. 8u+7 -> chunk u / 8, 16-byte slot (u % 8) ^ (b % 8) of row b
  // eight units (16 loads of 16 bytes) in flight per thread, then their conversions
  const int units = NB * (p.dc / 8);
  constexpr int UB = 8;
  for (int u0 = threadIdx.x; u0 < units; u0 += UB * THREADS) {
    float4 ld[UB][2];
#pragma unroll
    for (int k = 0; k < UB; ++k) {
      const int u = u0 + k * THREADS;
      const int b = u / (p.dc / 8), c8 = u % (p.dc / 8);
      if (u < units && b0 + b < p.B) {
        const float4 *src = reinterpret_cast<const float4 *>(p.chat + ((size_t)(b0 + b) * p.H + h) * p.dc + 8 * c8);
        ld[k][0] = src[0];
        ld[k][1] = src[1];
      } else {
        ld[k][0] = ld[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int k = 0; k < UB; ++k) {
      const int u = u0 + k * THREADS;
      if (u >= units) break;
      const int b = u / (p.dc / 8), c8 = u % (p.dc / 8);
      const float x[8] = {ld[k][0].x, ld[k][0].y, ld[k][0].z, ld[k][0].w, ld[k][1].x, ld[k][1].y, ld[k][1].z, ld[k][1].w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * i]), h1 = __float2bfloat16_rn(x[2 * i + 1]);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * i] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * i + 1] - __bfloat162float(h1));
        hw[i] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        lw[i] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
      }
      const uint32_t off = b * 128 + ((((c8 & 7) ^ (b & 7))) << 4);
      *reinterpret_cast<uint4 *>(sm.hi[c8 >> 3] + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(sm.lo[c8 >> 3] + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
  fence_proxy_async_smem();  // the MMAs read these through the async proxy
  __syncthreads();
  if (threadIdx.x == 0) {
    if (mbar_wait(&sm.full, 0, p.status)) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, NB, false, false);
      const int ksteps = p.dc / 16;
      for (int part = 0; part < 2; ++part) {
        uint8_t(*bsrc)[BCHUNK] = part ? sm.lo : sm.hi;
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint64_t a = sdesc_sw128(smem_u32(sm.w[kk >> 2]) + (kk & 3) * 32, 16, 1024);
          const uint64_t bc = sdesc_sw128(smem_u32(bsrc[kk >> 2]) + (kk & 3) * 32, 16, 1024);
          umma_bf16_ss(tmem, a, bc, idesc, (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
    }
    umma_commit(&sm.done);
  }
  __syncwarp();
  const bool ok = mbar_wait(&sm.done, 0, p.status);
  tc_fence_after();
  float v[32];
  tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
  const int r = 32 * warp + lane;  // row of W_v^(h): output channel 128h + r
  if (ok) {
    // the gate logits of all 32 sequences first (their loads in flight together), then the stores
    float gate[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j)
      gate[j] = (p.G && b0 + j < p.B) ? bf16_to_f32(p.G[(size_t)(b0 + j) * p.H * HD + (size_t)h * HD + r]) : 0.f;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (b0 + j < p.B) {
        const size_t oi = (size_t)(b0 + j) * p.H * HD + (size_t)h * HD + r;
        const float o = p.G ? v[j] * sigmoidf_(gate[j]) : v[j];
        p.out[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NB);
  }
}

}  // namespace side

// q~ [B, H, dc] = scale*log2(e) * (W_k^(h)T q_h) for every (b, h).
int launch_absorb_tc(const uint16_t *Q, const uint16_t *Wk, int B, int H, int dc, float sl2, uint16_t *qt,
                     unsigned *status, cudaStream_t stream) {
  using namespace side;
  if (dc % 64 || dc > 64 * MAX_CHUNKS) return -1;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(absorb_tc_kernel), (int)kSmemAbsorb, kSmemAbsorbTc))
    return -1;
  CUtensorMap tw, tq;
  const long long dw[2] = {dc, (long long)H * HD}, sw[1] = {dc};
  const unsigned bw[2] = {64, 128};
  const long long dq[2] = {(long long)H * HD, B}, sq[1] = {(long long)H * HD};
  const unsigned bq[2] = {64, NB};
  if (!make_tmap_bf16(&tw, Wk, 2, dw, sw, bw) || !make_tmap_bf16(&tq, Q, 2, dq, sq, bq)) return -1;
  Params p{};
  p.out = qt;
  p.B = B;
  p.H = H;
  p.dc = dc;
  p.sl2 = sl2;
  p.status = status;
  absorb_tc_kernel<<<dim3(H, (dc + 127) / 128, (B + NB - 1) / NB), THREADS, kSmemAbsorb, stream>>>(tw, tq, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// O [B, H*128] = (optionally gated) W_v^(h) c^[b, h] for every (b, h).
int launch_wv_tc(const float *chat, const uint16_t *Wv, const uint16_t *G, uint16_t *O, int B, int H, int dc,
                 unsigned *status, cudaStream_t stream) {
  using namespace side;
  if (dc % 64 || dc > 64 * MAX_CHUNKS) return -1;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(wv_tc_kernel), (int)kSmemWvTc, kSmemWv)) return -1;
  CUtensorMap tw;
  const long long dw[2] = {dc, (long long)H * HD}, sw[1] = {dc};
  const unsigned bw[2] = {64, 128};
  if (!make_tmap_bf16(&tw, Wv, 2, dw, sw, bw)) return -1;
  Params p{};
  p.chat = chat;
  p.G = G;
  p.out = O;
  p.B = B;
  p.H = H;
  p.dc = dc;
  p.status = status;
  wv_tc_kernel<<<dim3(H, (B + NB - 1) / NB), THREADS, kSmemWvTc, stream>>>(tw, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

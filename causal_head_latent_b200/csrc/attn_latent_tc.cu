// Split-KV decode over the latent cache on tcgen05 tensor cores.
//
// One CTA streams the latents [k_begin, k_end) of one sequence b and keeps an
// online-softmax state for all H (<= 96) heads at once; every latent tile is
// read from HBM once and used twice, as keys and as values:
//   S      [head, key]   = q~ C_tile^T          M=128 (heads, zero-padded by
//                                                overlap), N=KT, K=d_c
//   acc^T  [d_c, head]  += C_tile^T P^T         M=128 per d_c block, N=96,
//                                                K=KT  (C tile read MN-major)
// q~ = scale*log2(e) * W_k^(h)T q_h comes from the absorb kernel (bfloat16),
// so S is already in the exp2 domain.  P is rounded to bfloat16 before it
// multiplies the latents, as in the eager attention path ("Kimi K3 - Softmax
// over keys": float32 softmax, probabilities cast to the input type).
//
//   warp 0      TMA producer: q~ once, latent tiles into a STAGES-deep ring
//   warp 1      TMEM owner, MMA issuer (one thread)
//   warps 2..5  softmax (one head per TMEM lane), lazy rescale of acc^T when a
//               head's running max grows by more than 2^8, partial-state store
// TMEM columns: S double buffer [0, 2*64), acc^T blocks at 128 + 96*blk.
//
// q~ layout in shared memory: eight 64-column chunks of 96 rows (12 KB each)
// placed 12 KB apart.  The MMA reads 128-row A tiles, so rows 96..127 of chunk
// k alias rows 0..31 of chunk k+1 (a 4 KB tail follows the last chunk): those
// rows only feed S rows 96..127, which nothing reads.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace latent_tc {

constexpr int HMAX = 96;
constexpr int NUM_THREADS = 192;
constexpr int QCHUNK = HMAX * 128;         // 12 KB
constexpr int Q_BYTES = 8 * QCHUNK + 4096; // + tail read by the padded rows of the last chunk
constexpr int P_BYTES = HMAX * 128;        // P^T rows: one 128-byte swizzled row per head
constexpr float kRescaleThreshold = 8.0f;
constexpr int kPrefetchTiles = 8;          // L2 prefetch distance of the latent stream
constexpr int TM_S = 0;                    // two S buffers of 64 columns
constexpr int TM_ACC = 128;                // acc^T blocks: 128 + 96*blk

template <int KT>
struct Geo {
  static constexpr int CCHUNK = KT * 128;  // one 64-wide d_c chunk of a KT-key tile
  static constexpr int C_BYTES = 8 * CCHUNK;
};

struct Params {
  const uint16_t *C;  // latent cache [B, Lmax, dc] (for the L2 prefetch stream)
  long long Lmax;
  int B, L, H, dc, n_splits, keys_per_split;
  float *part_m, *part_l, *part_acc;  // [S,B,H], [S,B,H], [S,B,H,512]
  float *weights;                     // optional raw log2-domain scores [B,H,L]
  unsigned *status;
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// OR of `v` over the `count` threads of named barrier `id` (all of them must call).
__device__ __forceinline__ bool bar_or(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbarrier.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int KT, int STAGES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    latent_decode_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmC,
                         const Params p) {
  using G = Geo<KT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sq = base;
  uint8_t *sc = sq + Q_BYTES;                 // Q_BYTES is a multiple of 1024
  uint8_t *sp = sc + STAGES * G::C_BYTES;     // two P^T buffers
  float *alpha_s = reinterpret_cast<float *>(sp + 2 * P_BYTES);
  uint64_t *bars = reinterpret_cast<uint64_t *>(alpha_s + 128);
  uint64_t *bar_q = bars;
  uint64_t *c_full = bars + 1;
  uint64_t *c_empty = c_full + STAGES;
  uint64_t *s_full = c_empty + STAGES;  // [2]
  uint64_t *s_free = s_full + 2;        // [2]
  uint64_t *p_full = s_free + 2;
  uint64_t *pv_done = p_full + 1;       // [2]: PV of tile j arrives on pv_done[j & 1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.x / p.n_splits;
  const int split = blockIdx.x % p.n_splits;
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.L, k_begin + p.keys_per_split);
  const int n_tiles = (k_end - k_begin + KT - 1) / KT;  // >= 1 (the host leaves no split empty)

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQt);
      tma_prefetch_desc(&tmC);
      mbar_arrive_expect_tx(bar_q, 8 * QCHUNK);
      for (int kc = 0; kc < 8; ++kc) tma_load_3d(sq + kc * QCHUNK, &tmQt, bar_q, kc * 64, 0, b);
      // The latents of this split are one contiguous range; keep an L2 prefetch
      // stream kPrefetchTiles ahead of the shared-memory ring so DRAM latency is
      // hidden without more shared memory.
      const uint8_t *crow = reinterpret_cast<const uint8_t *>(p.C + ((size_t)b * p.Lmax) * p.dc);
      const size_t key_bytes = (size_t)p.dc * 2;
      auto prefetch_tile = [&](int jt) {
        const int kb = k_begin + jt * KT;
        if (jt < n_tiles) prefetch_l2_bulk(crow + (size_t)kb * key_bytes, (uint32_t)(min(KT, k_end - kb) * key_bytes));
      };
      for (int jt = 1; jt < kPrefetchTiles; ++jt) prefetch_tile(jt);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        prefetch_tile(j + kPrefetchTiles);
        if (!mbar_wait(&c_empty[s], ((j / STAGES) & 1) ^ 1, p.status)) break;
        mbar_arrive_expect_tx(&c_full[s], G::C_BYTES);
        uint8_t *dst = sc + s * G::C_BYTES;
        const int k0 = k_begin + j * KT;
        for (int kc = 0; kc < 8; ++kc) tma_load_3d(dst + kc * G::CCHUNK, &tmC, &c_full[s], kc * 64, k0, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, KT, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, HMAX, true, false);
      const uint32_t aq = smem_u32(sq), ac = smem_u32(sc), ap = smem_u32(sp);
      bool ok = mbar_wait(bar_q, 0, p.status);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % STAGES, sb = j & 1;
          ok = mbar_wait(&c_full[s], (j / STAGES) & 1, p.status);
          if (ok && j >= 2) ok = mbar_wait(&s_free[sb], ((j - 2) >> 1) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t cst = ac + s * G::C_BYTES;
          const uint32_t dS = tmem + TM_S + sb * 64;
#pragma unroll
          for (int kc = 0; kc < 8; ++kc)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(dS, sdesc_sw128(aq + kc * QCHUNK + kk * 32, 16, 1024),
                           sdesc_sw128(cst + kc * G::CCHUNK + kk * 32, 16, 1024), idS, (kc | kk) ? 1u : 0u);
          umma_commit(&s_full[sb]);
        }
        if (j >= 1) {
          const int jp = j - 1, s = jp % STAGES;
          ok = mbar_wait(p_full, jp & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t cst = ac + s * G::C_BYTES;
#pragma unroll
          for (int blk = 0; blk < 4; ++blk)
#pragma unroll
            for (int ks = 0; ks < KT / 16; ++ks)
              umma_bf16_ss(tmem + TM_ACC + blk * HMAX,
                           sdesc_sw128(cst + 2 * blk * G::CCHUNK + ks * 2048, G::CCHUNK, 1024),
                           sdesc_sw128(ap + (jp & 1) * P_BYTES + ks * 32, 16, 1024), idPV,
                           (jp > 0 || ks > 0) ? 1u : 0u);
          umma_commit(&pv_done[jp & 1]);
          umma_commit(&c_empty[s]);
        }
      }
    }
  } else {
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;  // head owned in the S phase; d_c row in the acc phase
    const bool head_ok = h < p.H;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    uint8_t *prow = sp + h * 128;
    const int sw = h & 7;
    float *wrow = (p.weights && head_ok) ? p.weights + ((size_t)b * p.H + h) * (size_t)p.L : nullptr;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, p.status)) { ok = false; break; }
      tc_fence_after();
      float x[KT];
      if (quarter < 3) {  // lanes 96..127 hold only padding rows
#pragma unroll
        for (int c = 0; c < KT; c += 16) tmem_ld16(tmem + lane_off + TM_S + sb * 64 + c, x + c);
      } else {
#pragma unroll
        for (int c = 0; c < KT; ++c) x[c] = -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      const int k0 = k_begin + j * KT;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < KT; ++c) {
        if (k0 + c >= k_end) x[c] = -INFINITY;
        mx = fmaxf(mx, x[c]);
      }
      if (wrow) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (k0 + c < k_end) wrow[k0 + c] = x[c];
      }
      float alpha = 1.f;
      bool resc = false;
      if (head_ok && mx > m_used + kRescaleThreshold) {
        if (m_used != -INFINITY) {
          alpha = fast_exp2(m_used - mx);
          resc = true;
        }
        m_used = mx;
      }
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      float rs = 0.f;
      uint32_t pk[KT / 2];
#pragma unroll
      for (int c = 0; c < KT; c += 2) {
        const float p0 = fast_exp2(x[c] - mref), p1 = fast_exp2(x[c + 1] - mref);
        rs += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      if (head_ok) l = l * alpha + rs;
      alpha_s[h] = alpha;
      const bool any = bar_or(1, 128, resc);

      // P^T buffer j&1 was last read by PV_{j-2}; a rescale of acc^T needs PV_{j-1} done.
      if (j >= 2 && !mbar_wait(&pv_done[j & 1], ((j >> 1) & 1) ^ 1, p.status)) { ok = false; break; }
      if (j > 0 && any) {
        if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.status)) { ok = false; break; }
        tc_fence_after();
        {
          // acc^T lanes are d_c rows; columns are heads: scale column h by alpha_s[h]
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
            for (int c = 0; c < HMAX; c += 32) {
              float v[32];
              const uint32_t ta = tmem + lane_off + TM_ACC + blk * HMAX + c;
              tmem_ld32(ta, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha_s[c + i];
              tmem_st32(ta, v);
            }
          }
        }
      }
      if (any) bar_sync(1, 128);  // alpha_s is rewritten by the next tile
      if (head_ok) {
        uint8_t *pr = prow + (j & 1) * P_BYTES;
#pragma unroll
        for (int u = 0; u < KT / 8; ++u)
          *reinterpret_cast<uint4 *>(pr + ((u ^ sw) << 4)) =
              make_uint4(pk[u * 4 + 0], pk[u * 4 + 1], pk[u * 4 + 2], pk[u * 4 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }

    // partial state of this split: m, l per head and acc^T
    if (ok && mbar_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.status)) {
      tc_fence_after();
      const size_t rec = ((size_t)split * p.B + b) * p.H;
      if (head_ok) {
        p.part_m[rec + h] = m_used;
        p.part_l[rec + h] = l;
      }
      const int row = quarter * 32 + lane;  // d_c row within a block
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        const int col = blk * 128 + row;  // latent column
#pragma unroll 1
        for (int c = 0; c < HMAX; c += 32) {
          float v[32];
          tmem_ld32(tmem + lane_off + TM_ACC + blk * HMAX + c, v);
          if (col < p.dc) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i < p.H) p.part_acc[(rec + c + i) * (size_t)p.dc + col] = v[i];
          }
        }
      }
    }
    tc_fence_before();
  }

  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int KT, int STAGES>
size_t smem_bytes() {
  return 1024 + Q_BYTES + STAGES * Geo<KT>::C_BYTES + 2 * P_BYTES + 128 * 4 + 8 * (1 + 2 * STAGES + 7) + 16;
}

}  // namespace latent_tc

// Keys per tile and pipeline depth of the tensor-core decode.
constexpr int kLatentKT = 32;
constexpr int kLatentStages = 3;

int latent_tc_tile_keys() { return kLatentKT; }

int launch_latent_tc(const CUtensorMap &tmQt, const CUtensorMap &tmC, const uint16_t *C, long long Lmax, int B, int L,
                     int H, int dc, int n_splits, int keys_per_split, float *part_m, float *part_l, float *part_acc,
                     float *weights, unsigned *status, cudaStream_t stream) {
  using namespace latent_tc;
  auto kern = latent_decode_kernel<kLatentKT, kLatentStages>;
  const size_t smem = smem_bytes<kLatentKT, kLatentStages>();
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return -1;
    configured = true;
  }
  Params p;
  p.C = C;
  p.Lmax = Lmax;
  p.B = B;
  p.L = L;
  p.H = H;
  p.dc = dc;
  p.n_splits = n_splits;
  p.keys_per_split = keys_per_split;
  p.part_m = part_m;
  p.part_l = part_l;
  p.part_acc = part_acc;
  p.weights = weights;
  p.status = status;
  kern<<<B * n_splits, NUM_THREADS, smem, stream>>>(tmQt, tmC, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

// Causal prefill attention on tcgen05 tensor cores.
//
// Computes, per (batch b, head h), O = softmax(Q K^T * scale + M) V with the
// float32 softmax over keys and P cast to bfloat16 before P V ("Gated MLA"
// page, "Start from familiar attention"; "Kimi K3 - Softmax over keys";
// mask of "Kimi K2 - Construct causal mask").  Query t of Tq sits at absolute
// position Tk - Tq + t.  The softmax runs online over key tiles (running max
// and sum with rescaling, Milakov & Gimelshein 2018), which is exact in real
// arithmetic.
//
// One CTA owns one 128-row query tile of one (b, h):
//   warp 0      TMA producer: Q once, then K/V tiles into a 2-stage ring
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S = Q K^T   (M=128, N=128, K=128, both operands K-major)
//                 O += P V    (P from shared memory, V MN-major)
//   warps 2..5  softmax warpgroup, one query row per thread (TMEM lane):
//                 S row from TMEM, mask, online max/sum in the exp2 domain,
//                 P row (bf16) into shared memory, O rescale in TMEM when the
//                 running max grows by more than 2^8, final 1/l, gate, store.
// TMEM: S in columns [0,128), O in [128,256).
// Tiles above the diagonal are skipped; only diagonal / tail tiles are masked.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace prefill {

constexpr int BM = 128;           // query rows per CTA
constexpr int BN = 128;           // keys per tile
constexpr int HD = 128;           // head dimension
constexpr int STAGES = 2;         // K/V ring depth
constexpr int TILE_BYTES = BM * HD * 2;  // one 128x128 bf16 operand tile = 2 swizzled 64-column chunks
constexpr int CHUNK_BYTES = TILE_BYTES / 2;
constexpr int NUM_THREADS = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest p we let through unrescaled

struct Smem {
  uint8_t q[TILE_BYTES];
  uint8_t k[STAGES][TILE_BYTES];
  uint8_t v[STAGES][TILE_BYTES];
  uint8_t p[TILE_BYTES];
  uint64_t bar_q;
  uint64_t bar_k_full[STAGES];
  uint64_t bar_v_full[STAGES];
  uint64_t bar_kv_empty[STAGES];
  uint64_t bar_s_full;
  uint64_t bar_s_free;
  uint64_t bar_p_full;
  uint64_t bar_o_done;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

struct Params {
  const uint16_t *G;  // optional gate logits [B, Tq, H*HD]
  uint16_t *O;
  long long o_sb, o_st, o_sh;
  float *lse;
  float *weights;
  int B, H, Tq, Tk, causal;
  int n_qt;
  float scale_log2;  // scale * log2(e)
  unsigned *status;
};

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) { return sdesc_sw128(addr, 16, 1024); }

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // Heavy (late) query tiles first; consecutive CTAs take different heads.
  const int BH = p.B * p.H;
  const int lin = blockIdx.x;
  const int qt = p.causal ? (p.n_qt - 1 - lin / BH) : (lin / BH);
  const int bh = lin % BH;
  const int b = bh / p.H, h = bh % p.H;
  const int q0 = qt * BM;
  const int shift = p.Tk - p.Tq;  // absolute position of query 0
  // Keys needed by this tile: 0 .. last_key
  const int last_row = min(q0 + BM - 1, p.Tq - 1);
  const int last_key = p.causal ? min(p.Tk - 1, shift + last_row) : (p.Tk - 1);
  const int n_kv = last_key / BN + 1;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.bar_k_full[s], 1);
      mbar_init(&sm.bar_v_full[s], 1);
      mbar_init(&sm.bar_kv_empty[s], 1);
    }
    mbar_init(&sm.bar_s_full, 1);
    mbar_init(&sm.bar_s_free, 4);
    mbar_init(&sm.bar_p_full, 4);
    mbar_init(&sm.bar_o_done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + 128;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&sm.bar_q, TILE_BYTES);
      tma_load_4d(sm.q, &tmQ, &sm.bar_q, 0, q0, h, b);
      tma_load_4d(sm.q + CHUNK_BYTES, &tmQ, &sm.bar_q, 64, q0, h, b);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % STAGES, r = j / STAGES;
        if (!mbar_wait(&sm.bar_kv_empty[s], (r & 1) ^ 1, p.status)) { sm.abort_flag = 1; break; }
        const int k0 = j * BN;
        mbar_arrive_expect_tx(&sm.bar_k_full[s], TILE_BYTES);
        tma_load_4d(sm.k[s], &tmK, &sm.bar_k_full[s], 0, k0, h, b);
        tma_load_4d(sm.k[s] + CHUNK_BYTES, &tmK, &sm.bar_k_full[s], 64, k0, h, b);
        mbar_arrive_expect_tx(&sm.bar_v_full[s], TILE_BYTES);
        tma_load_4d(sm.v[s], &tmV, &sm.bar_v_full[s], 0, k0, h, b);
        tma_load_4d(sm.v[s] + CHUNK_BYTES, &tmV, &sm.bar_v_full[s], 64, k0, h, b);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 128, false, true);
      const uint32_t aQ = smem_u32(sm.q);
      const uint32_t aP = smem_u32(sm.p);
      bool ok = mbar_wait(&sm.bar_q, 0, p.status);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int s = j % STAGES;
          ok = mbar_wait(&sm.bar_k_full[s], (j / STAGES) & 1, p.status);
          if (ok && j > 0) ok = mbar_wait(&sm.bar_s_free, (j - 1) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t aK = smem_u32(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
            umma_bf16_ss(tS, desc_kmajor(aQ + off), desc_kmajor(aK + off), idS, kk > 0);
          }
          umma_commit(&sm.bar_s_full);
        }
        if (j > 0) {
          const int jp = j - 1, s = jp % STAGES;
          ok = mbar_wait(&sm.bar_p_full, jp & 1, p.status);
          if (ok) ok = mbar_wait(&sm.bar_v_full[s], (jp / STAGES) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t aV = smem_u32(sm.v[s]);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t offP = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
            // V tile: rows = keys (128 B per row), two 64-wide D chunks 16 KB apart.
            umma_bf16_ss(tO, desc_kmajor(aP + offP), sdesc_sw128(aV + kk * 2048, CHUNK_BYTES, 1024), idPV,
                         (jp > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&sm.bar_o_done);
          umma_commit(&sm.bar_kv_empty[s]);
        }
      }
      if (!ok) sm.abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroup
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // query row within the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int t = q0 + row;                 // query index
    const bool row_valid = t < p.Tq;
    const int pos = shift + t;              // absolute position
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    float *wrow = (p.weights && row_valid) ? p.weights + (((size_t)b * p.H + h) * p.Tq + t) * (size_t)p.Tk : nullptr;
    uint8_t *prow = sm.p + row * 128;
    const int sw = row & 7;
    bool ok = true;

    for (int j = 0; j < n_kv; ++j) {
      const int k0 = j * BN;
      if (!mbar_wait(&sm.bar_s_full, j & 1, p.status)) { ok = false; break; }
      tc_fence_after();
      float x[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float tmp[32];
        tmem_ld32(tS + lane_off + c * 32, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = tmp[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_s_free);

      // scale into the log2 domain, mask, row max
      const bool need_mask = (k0 + BN > p.Tk) || (p.causal && (k0 + BN - 1 > shift + q0));
      float mx = -INFINITY;
      if (need_mask) {
        const int lim = p.causal ? min(pos, p.Tk - 1) : (p.Tk - 1);
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] = (k0 + c <= lim) ? x[c] * sl2 : -INFINITY;
          mx = fmaxf(mx, x[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] *= sl2;
          mx = fmaxf(mx, x[c]);
        }
      }
      if (wrow) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (k0 + c < p.Tk) wrow[k0 + c] = x[c];
      }
      // lazy rescale: keep the old reference max unless this tile exceeds it by > 2^8
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_used + kRescaleThreshold) {
        if (m_used != -INFINITY) {
          alpha = fast_exp2(m_used - mx);
          rescale = true;
        }
        m_used = mx;
      }
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      float rs = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = fast_exp2(x[c] - mref);
        const float p1 = fast_exp2(x[c + 1] - mref);
        rs += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;

      // PV of the previous tile must be done before O is rescaled or P overwritten.
      if (j > 0) {
        if (!mbar_wait(&sm.bar_o_done, (j - 1) & 1, p.status)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            float o[32];
            tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + lane_off + c * 32, o);
          }
        }
      }
      // P row -> shared memory in the 128-byte-swizzled K-major layout
#pragma unroll
      for (int u = 0; u < BN / 8; ++u) {
        const int chunk = u >> 3, uu = u & 7;
        uint4 val = make_uint4(pk[u * 4 + 0], pk[u * 4 + 1], pk[u * 4 + 2], pk[u * 4 + 3]);
        *reinterpret_cast<uint4 *>(prow + chunk * CHUNK_BYTES + ((uu ^ sw) << 4)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_p_full);
    }

    // ---------------------------------------------------------------- epilogue
    if (ok && mbar_wait(&sm.bar_o_done, (n_kv - 1) & 1, p.status)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      uint16_t *orow = p.O + (long long)b * p.o_sb + (long long)t * p.o_st + (long long)h * p.o_sh;
      const uint16_t *grow = p.G ? p.G + ((size_t)b * p.Tq + t) * (size_t)(p.H * HD) + (size_t)h * HD : nullptr;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tO + lane_off + c * 32, o);
        if (row_valid) {
          if (grow) {
            const uint4 *g4 = reinterpret_cast<const uint4 *>(grow + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 gv = g4[v];
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                o[v * 8 + e * 2] *= inv_l * sigmoidf_(bf16_to_f32(gw[e] & 0xFFFF));
                o[v * 8 + e * 2 + 1] *= inv_l * sigmoidf_(bf16_to_f32(gw[e] >> 16));
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= inv_l;
          }
          uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pack_bf16x2(o[v * 8 + 0], o[v * 8 + 1]), pack_bf16x2(o[v * 8 + 2], o[v * 8 + 3]),
                                pack_bf16x2(o[v * 8 + 4], o[v * 8 + 5]), pack_bf16x2(o[v * 8 + 6], o[v * 8 + 7]));
        }
      }
      if (row_valid && p.lse) p.lse[((size_t)b * p.H + h) * p.Tq + t] = (m_used + __log2f(l)) * 0.6931471805599453f;
      if (wrow) {
        // debug weights: raw log2-domain scores were stored above; normalise in place
        const int lim = p.causal ? min(pos, p.Tk - 1) : (p.Tk - 1);
        const float lg = m_used + __log2f(l);
        for (int s = 0; s < p.Tk; ++s) wrow[s] = (s <= lim) ? fast_exp2(wrow[s] - lg) : 0.f;
      }
    } else {
      sm.abort_flag = 1;
    }
    tc_fence_before();
  }

  __syncwarp();  // lane 0 of the producer / MMA warps ran its loop alone
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace prefill

int launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                        const PrefillArgs &a, cudaStream_t stream) {
  using namespace prefill;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return -1;
    configured = true;
  }
  Params p;
  p.G = a.G;
  p.O = a.O;
  p.o_sb = a.o_strides[0];
  p.o_st = a.o_strides[1];
  p.o_sh = a.o_strides[2];
  p.lse = a.lse;
  p.weights = a.weights;
  p.B = a.B;
  p.H = a.H;
  p.Tq = a.Tq;
  p.Tk = a.Tk;
  p.causal = a.causal;
  p.n_qt = (a.Tq + BM - 1) / BM;
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;
  const long long grid = (long long)p.n_qt * a.B * a.H;
  if (grid <= 0) return 0;
  if (grid > 0x7fffffffLL) return -2;
  attn_prefill_kernel<<<(unsigned)grid, NUM_THREADS, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

size_t attn_prefill_smem_bytes() { return prefill::kSmemBytes; }

}  // namespace gmla

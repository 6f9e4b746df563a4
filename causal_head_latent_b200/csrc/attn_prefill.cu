// Causal prefill attention on tcgen05 tensor cores.
//
// Computes, per (batch b, head h), O = softmax(Q K^T * scale + M) V with the
// float32 softmax over keys and P cast to bfloat16 before P V ("Gated MLA"
// page, "Start from familiar attention"; "Kimi K3 - Softmax over keys";
// mask of "Kimi K2 - Construct causal mask").  Query t of Tq sits at absolute
// position Tk - Tq + t.  The softmax runs online over key tiles (running max
// and sum with rescaling, Milakov & Gimelshein 2018), exact in real arithmetic.
//
// One CTA owns two 128-row query tiles (Q0, Q1) of one (b, h) and streams the
// K/V tiles they need once for both:
//   warp 0      TMA producer: Q0, K0, Q1, V0, then K and V tiles into 2-stage rings
//   warp 1      TMEM owner and MMA issuer (one thread).  Per key tile j the
//               tensor core runs   PV0_j, S0_{j+1}, PV1_j, S1_{j+1}
//               with S_i = Q_i K^T (both operands K-major, in shared memory)
//               and O_i += P_i V (P_i read from TMEM, V MN-major in shared
//               memory), so softmax of one tile overlaps MMAs of the other.
//   warps 2-5   softmax warpgroup of Q0, one query row per thread (TMEM lane)
//   warps 6-9   softmax warpgroup of Q1
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).  P_i
// (bfloat16, two per column) overwrites the first 64 columns of S_i.
// Because S_i of tile j+1 is issued after PV_i of tile j, its completion also
// means PV_i_j is done: the softmax may then rescale O_i (lazy: only when the
// running max grew by more than 2^8) and overwrite P_i without further waits.
// Tiles above the diagonal are skipped; only diagonal / tail tiles are masked.
#include "internal.h"
#include "launch_plan.h"
#include "ptx.cuh"

namespace gmla {
namespace prefill {

constexpr int BM = 128;                  // query rows per tile
constexpr int BN = 128;                  // keys per tile
constexpr int HD = 128;                  // head dimension
constexpr int STAGES = 2;                // K and V ring depth
constexpr int TILE_BYTES = BM * HD * 2;  // 128 x 128 bf16 = two 64-column swizzled chunks
constexpr int CHUNK_BYTES = TILE_BYTES / 2;
constexpr int NUM_THREADS = 320;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest p let through unrescaled

struct Smem {
  uint8_t q[2][TILE_BYTES];
  uint8_t k[STAGES][TILE_BYTES];
  uint8_t v[STAGES][TILE_BYTES];
  uint64_t bar_q[2];
  uint64_t k_full[STAGES], k_empty[STAGES];
  uint64_t v_full[STAGES], v_empty[STAGES];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint32_t tmem_base;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

struct Params {
  const uint16_t *G;  // optional gate logits [B, Tq, H*HD]
  uint16_t *O;
  long long o_sb, o_st, o_sh;
  float *lse;
  float *weights;
  int B, H, Tq, Tk, causal;  // Tq, Tk: the row strides of G, lse and weights (the maxima with lengths)
  // Per-sequence lengths (null: every sequence has Tq queries and Tk keys):
  // sequence b has q_lens[b] query rows and kv_lens[b] keys, read through
  // maps[3b .. 3b+2], 3-D maps (D, length, H) of Q, K and V whose row extent is
  // the sequence's length, so rows past it read as zeros.
  const int *q_lens, *kv_lens;
  const CUtensorMap *maps;
  int n_ct;          // CTAs (256-row query pairs) per (b, h)
  int head_group;    // (b, h) pairs per group of the launch order
  float scale_log2;  // scale * log2(e)
  unsigned *status;
};

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) { return sdesc_sw128(addr, 16, 1024); }

// D[tmem] (+)= A[tmem] * B[smem] (A from tensor memory, K-major).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Number of key tiles query tile `qt` needs (0 when the tile has no valid row).
__device__ __forceinline__ int kv_tiles(int Tq, int Tk, int causal, int qt) {
  const int q0 = qt * BM;
  if (q0 >= Tq) return 0;
  const int last_row = min(q0 + BM - 1, Tq - 1);
  const int last_key = causal ? min(Tk - 1, Tk - Tq + last_row) : (Tk - 1);
  return last_key / BN + 1;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // Launch order: the (b, h) pairs in groups of head_group, so that the K and V
  // of the few heads in flight stay in L2; within a group the query pairs go
  // longest (latest) first across all of the group's heads, so that the last
  // CTAs of the launch are short ones and no long CTA starts near the end.
  int bh, ct;
  prefill_cta_item((int)blockIdx.x, p.B * p.H, p.n_ct, p.head_group, p.causal != 0, &bh, &ct);
  const int b = bh / p.H, h = bh % p.H;
  const int Tq = p.q_lens ? p.q_lens[b] : p.Tq;  // this sequence's query rows and keys
  const int Tk = p.kv_lens ? p.kv_lens[b] : p.Tk;
  const int nkv0 = kv_tiles(Tq, Tk, p.causal, 2 * ct);
  const int nkv1 = kv_tiles(Tq, Tk, p.causal, 2 * ct + 1);
  const int nkv = max(nkv0, nkv1);
  // Query pairs past a shorter sequence's rows (per-sequence lengths only):
  // nothing to compute or store; the whole CTA leaves before any barrier.
  if (nkv == 0) return;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q[0], 1);
    mbar_init(&sm.bar_q[1], 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 4);
    }
    mbar_init(&sm.o_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const CUtensorMap *mq = p.maps ? p.maps + 3 * b : &tmQ;
      const CUtensorMap *mk = p.maps ? p.maps + 3 * b + 1 : &tmK;
      const CUtensorMap *mv = p.maps ? p.maps + 3 * b + 2 : &tmV;
      if (p.maps) {
        fence_tensormap_acquire(mq);
        fence_tensormap_acquire(mk);
        fence_tensormap_acquire(mv);
      }
      // one 64-column half of a 128-row tile (rows `row`.., head h of sequence b)
      auto load = [&](void *dst, const CUtensorMap *m, uint64_t *bar, int col, int row) {
        if (p.maps)
          tma_load_3d(dst, m, bar, col, row, h);
        else
          tma_load_4d(dst, m, bar, col, row, h, b);
      };
      tma_prefetch_desc(mq);
      tma_prefetch_desc(mk);
      tma_prefetch_desc(mv);
      const int q0 = 2 * ct * BM;
      // Q0 and K0 first: the first S product needs only them; Q1 follows K0
      auto load_q = [&](int i) {
        mbar_arrive_expect_tx(&sm.bar_q[i], TILE_BYTES);
        load(sm.q[i], mq, &sm.bar_q[i], 0, q0 + i * BM);
        load(sm.q[i] + CHUNK_BYTES, mq, &sm.bar_q[i], 64, q0 + i * BM);
      };
      load_q(0);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % STAGES, ph = ((j / STAGES) & 1) ^ 1;
        const int k0 = j * BN;
        if (!mbar_wait(&sm.k_empty[s], ph, p.status)) break;
        mbar_arrive_expect_tx(&sm.k_full[s], TILE_BYTES);
        load(sm.k[s], mk, &sm.k_full[s], 0, k0);
        load(sm.k[s] + CHUNK_BYTES, mk, &sm.k_full[s], 64, k0);
        if (j == 0) load_q(1);
        if (!mbar_wait(&sm.v_empty[s], ph, p.status)) break;
        mbar_arrive_expect_tx(&sm.v_full[s], TILE_BYTES);
        load(sm.v[s], mv, &sm.v_full[s], 0, k0);
        load(sm.v[s] + CHUNK_BYTES, mv, &sm.v_full[s], 64, k0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 128, false, true);
      const uint32_t aQ[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      const int nk[2] = {nkv0, nkv1};
      bool ok = mbar_wait(&sm.bar_q[0], 0, p.status);
      // S_i for key tile j (K-major Q_i and K_j)
      auto issue_s = [&](int i, int j) {
        const uint32_t aK = smem_u32(sm.k[j % STAGES]);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
          umma_bf16_ss(tmem + i * 128, desc_kmajor(aQ[i] + off), desc_kmajor(aK + off), idS, kk > 0);
        }
        umma_commit(&sm.s_full[i]);
      };
      // O_i += P_i V_j (P_i in TMEM columns [128 i, 128 i + 64), V_j MN-major)
      auto issue_pv = [&](int i, int j) {
        const uint32_t aV = smem_u32(sm.v[j % STAGES]);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ts(tmem + 256 + i * 128, tmem + i * 128 + kk * 8,
                       sdesc_sw128(aV + kk * 2048, CHUNK_BYTES, 1024), idPV, (j > 0 || kk > 0) ? 1u : 0u);
      };
      if (ok) ok = mbar_wait(&sm.k_full[0], 0, p.status);
      if (ok) {
        tc_fence_after();
        if (nk[0] > 0) issue_s(0, 0);
        if (nk[1] > 0) {
          ok = mbar_wait(&sm.bar_q[1], 0, p.status);
          tc_fence_after();
          if (ok) issue_s(1, 0);
        }
        umma_commit(&sm.k_empty[0]);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % STAGES;
        const bool next = j + 1 < nkv;
        ok = mbar_wait(&sm.v_full[s], (j / STAGES) & 1, p.status);
        if (ok && next) ok = mbar_wait(&sm.k_full[(j + 1) % STAGES], ((j + 1) / STAGES) & 1, p.status);
        for (int i = 0; ok && i < 2; ++i) {
          if (j < nk[i]) {
            if (!(ok = mbar_wait(&sm.p_full[i], j & 1, p.status))) break;
            tc_fence_after();
            issue_pv(i, j);
          }
          if (j + 1 < nk[i]) issue_s(i, j + 1);
        }
        if (!ok) break;
        umma_commit(&sm.v_empty[s]);
        if (next) umma_commit(&sm.k_empty[(j + 1) % STAGES]);
      }
      if (ok) umma_commit(&sm.o_done);
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int wg = (warp - 2) >> 2;         // 0: Q0, 1: Q1
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // query row within the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + wg * 128 + lane_off;
    const uint32_t tO = tmem + 256 + wg * 128 + lane_off;
    const int n_tiles = wg ? nkv1 : nkv0;
    const int q0 = (2 * ct + wg) * BM;
    const int t = q0 + row;
    const bool row_valid = t < Tq;
    const int shift = Tk - Tq;
    const int pos = shift + t;
    const int lim = p.causal ? min(pos, Tk - 1) : (Tk - 1);  // last visible key of this row
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    float *wrow = (p.weights && row_valid) ? p.weights + (((size_t)b * p.H + h) * p.Tq + t) * (size_t)p.Tk : nullptr;
    bool ok = true;

    for (int j = 0; j < n_tiles; ++j) {
      const int k0 = j * BN;
      if (!mbar_wait(&sm.s_full[wg], j & 1, p.status)) { ok = false; break; }
      tc_fence_after();
      float x[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float tmp[32];
        tmem_ld32(tS + c * 32, tmp);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = tmp[i];
      }
      const bool need_mask = k0 + BN - 1 > lim;  // a key of this tile lies past this row's last visible key
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (k0 + c > lim) x[c] = -INFINITY;
      }
      // the row maximum as 8 independent chains joined by a tree (a single
      // chain of BN - 1 dependent max operations is all latency)
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = x[i];
#pragma unroll
      for (int c = 8; c < BN; c += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], x[c + i]);
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mx *= sl2;  // scale > 0 commutes with max
      if (wrow) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (k0 + c < p.Tk) wrow[k0 + c] = x[c] * sl2;
      }
      // lazy rescale: keep the reference max unless this tile exceeds it by > 2^8
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_used + kRescaleThreshold) {
        if (m_used != -INFINITY) {
          alpha = fast_exp2(m_used - mx);
          rescale = true;
        }
        m_used = mx;
      }
      const float nref = (m_used == -INFINITY) ? 0.f : -m_used;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BN; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = fast_exp2(fmaf(x[c + e], sl2, nref));
          const float p1 = fast_exp2(fmaf(x[c + e + 1], sl2, nref));
          rs += p0 + p1;
          pk[e / 2] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c / 2, pk);
      }
      l = l * alpha + rs;
      // S_i of this tile completed after PV_i of the previous tile, so O_i is idle here.
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[wg]);
    }

    // ---------------------------------------------------------------- epilogue
    // The row's 128 gate logits, all sixteen 16-byte loads in flight while the
    // last P V products finish (loaded between the stores to O they would wait
    // for each store, as G and O may alias; each thread reads its own row first).
    const uint16_t *grow = p.G ? p.G + ((size_t)b * p.Tq + t) * (size_t)(p.H * HD) + (size_t)h * HD : nullptr;
    uint4 g16[HD / 8];
    if (n_tiles > 0 && ok && grow && row_valid) {
#pragma unroll
      for (int v = 0; v < HD / 8; ++v) g16[v] = reinterpret_cast<const uint4 *>(grow)[v];
    }
    if (n_tiles > 0 && ok && mbar_wait(&sm.o_done, 0, p.status)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      uint16_t *orow = p.O + (long long)b * p.o_sb + (long long)t * p.o_st + (long long)h * p.o_sh;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32, o);
        if (row_valid) {
          if (grow) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 gv = g16[c * 4 + v];
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
        const float lg = m_used + __log2f(l);
        for (int s = 0; s < p.Tk; ++s) wrow[s] = (s <= lim) ? fast_exp2(wrow[s] - lg) : 0.f;
      }
    }
    tc_fence_before();
  }

  __syncwarp();  // lane 0 of the producer / MMA warps ran its loop alone
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace prefill

int launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                        const PrefillArgs &a, cudaStream_t stream) {
  using namespace prefill;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(attn_prefill_kernel), (int)kSmemBytes, kSmemPrefill))
    return -1;
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
  p.q_lens = a.q_lens;
  p.kv_lens = a.kv_lens;
  p.maps = a.maps;
  p.causal = a.causal;
  p.n_ct = (a.Tq + 2 * BM - 1) / (2 * BM);
  p.head_group = prefill_head_group(a.Tk, HD);
  p.scale_log2 = a.scale * kLog2e;
  p.status = a.status;
  const long long grid = (long long)p.n_ct * a.B * a.H;
  if (grid <= 0) return 0;
  if (grid > 0x7fffffffLL) return -2;
  attn_prefill_kernel<<<(unsigned)grid, NUM_THREADS, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

size_t attn_prefill_smem_bytes() { return prefill::kSmemBytes; }

}  // namespace gmla

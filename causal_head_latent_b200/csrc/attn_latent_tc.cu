// Split-KV decode over the latent cache on tcgen05 tensor cores.
//
// One CTA streams the latents [k_begin, k_end) of one sequence b and keeps an
// online-softmax state for all H (<= 96) heads at once; every latent tile is
// read from HBM once and used twice, as keys and as values:
//   S^T    [key, head]  = C_tile q~^T         M=64 keys, N=96 heads, K=d_c
//   acc^T  [d_c, head] += C_tile^T P          M=128 per d_c block, N=96 heads,
//                                             K=64 keys (C tile read MN-major)
// with P [key, head] = 2^(S^T - m_head) held in shared memory as P^T rows.
// q~ = scale*log2(e) * W_k^(h)T q_h comes from the absorb kernel (bfloat16),
// so S is already in the exp2 domain.  P is rounded to bfloat16 before it
// multiplies the latents, as in the eager attention path ("Kimi K3 - Softmax
// over keys": float32 softmax, probabilities cast to the input type).
//
// Why keys on M: both products read their operands from shared memory, and on
// sm_100a an MMA with a small N is bound by those reads (A + B bytes per
// instruction), not by its arithmetic.  With keys on M, q~ is the 96-row B
// operand (no padding to 128 rows) and one 64-key tile costs 32 score MMAs,
// so the score product reads 2.5 KB of shared memory per key instead of the
// 5 KB a heads-on-M, 32-key-tile product needs.
//
//   warp 0      TMA producer: q~ once, then the latent stream in 64-column
//               chunks (8 KB: 64 keys x 64 d_c) through a 14-slot ring
//   warp 1      TMEM owner, MMA issuer (one thread)
//   warps 2..5  softmax: each thread holds 2 keys x 24 heads of S^T; lazy
//               rescale of acc^T when a head's running max grows by more than
//               2^8; partial-state store
//
// The ring holds 1.75 tiles, so the score MMAs of tile j are issued in two
// parts around the value MMAs of tile j-1: the first six chunks of tile j
// reuse slots tile j-2 released, the last two reuse the slots of chunks 0..1
// of tile j-1, which the first d_c block of its value product releases.
// Chunk pairs (2i, 2i+1) of a tile always sit in adjacent slots, so one
// MN-major descriptor with a slot-sized leading offset spans a 128-row d_c
// block.
//
// TMEM columns: S^T [0, 96) in the M=64 layout (rows 16r..16r+15 in lanes
// 32r..32r+15), acc^T blocks at 128 + 96*blk.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace latent_tc {

constexpr int HMAX = 96;
constexpr int KT = 64;                    // keys per tile: M of the score product
constexpr int NUM_THREADS = 192;
constexpr int NCHUNK = 8;                 // 64-wide d_c chunks per tile (d_c <= 512)
constexpr int QCHUNK = HMAX * 128;        // 12 KB: one d_c chunk of q~ for 96 heads
constexpr int Q_BYTES = NCHUNK * QCHUNK;  // 96 KB
constexpr int P_BYTES = HMAX * 128;       // P^T: one 128-byte swizzled row of 64 keys per head
constexpr int CCHUNK = KT * 128;          // 8 KB: one d_c chunk of a 64-key tile
constexpr int NSLOT = 14;                 // latent ring depth in chunks
constexpr int NEARLY = NSLOT - NCHUNK;    // score chunks issued before the previous tile's value product
constexpr float kRescaleThreshold = 8.0f;
constexpr int kPrefetchTiles = 8;         // L2 prefetch distance of the latent stream
constexpr int TM_S = 0;
constexpr int TM_ACC = 128;
constexpr unsigned long long kDrainLimitNs = 100000000ull;  // 100 ms: error-path drain of copies / MMAs

static_assert(NSLOT % 2 == 0 && NEARLY >= 2 && NEARLY <= NCHUNK, "ring depth");

struct Params {
  const uint16_t *C;  // latent cache [B, Lmax, dc] (for the L2 prefetch stream)
  long long Lmax;
  int B, L, H, dc, n_splits, keys_per_split;
  float *part_m, *part_l, *part_acc;  // [S,B,H], [S,B,H], [S,B,H,512]
  float *weights;                     // optional raw log2-domain scores [B,H,L]
  unsigned *status;
};

// 96 float32 columns of an M=64 accumulator in the 16x256b shape: this warp's
// 16 rows (lanes 32r..32r+15), thread t gets rows t/4 and t/4+8, column pair
// 2*(t%4) of every 8-column group.  v[4i + 2a + e] = (row t/4 + 8a, column
// 8i + 2*(t%4) + e).
__device__ __forceinline__ void tmem_ld_m64_96(uint32_t taddr, float *v) {
  uint32_t r[48];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47}, "
      "[%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47])
      : "r"(taddr), "r"(taddr + 64)
      : "memory");
#pragma unroll
  for (int i = 0; i < 48; ++i) v[i] = __uint_as_float(r[i]);
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

// Byte offset of P^T[h][key] in the 128-byte-swizzled K-major P^T buffer.
__device__ __forceinline__ uint32_t pt_offset(int h, int key) {
  return (uint32_t)(h * 128 + ((((key >> 3) ^ (h & 7)) << 4) | ((key & 7) << 1)));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    latent_decode_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmC,
                         const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sq = base;
  uint8_t *sp = sq + Q_BYTES;
  uint8_t *sc = sp + P_BYTES;  // Q_BYTES + P_BYTES is a multiple of 1024
  float *alpha_s = reinterpret_cast<float *>(sc + NSLOT * CCHUNK);
  float *red_s = alpha_s + 128;  // [4][HMAX]: per-quarter partial max / sum
  uint64_t *bars = reinterpret_cast<uint64_t *>(red_s + 4 * HMAX);
  uint64_t *bar_q = bars;
  uint64_t *c_full = bars + 1;           // [NSLOT]
  uint64_t *c_empty = c_full + NSLOT;    // [NSLOT]
  uint64_t *s_full = c_empty + NSLOT;
  uint64_t *s_free = s_full + 1;
  uint64_t *p_full = s_free + 1;
  uint64_t *acc_done = p_full + 1;
  uint64_t *mma_idle = acc_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_idle + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.x / p.n_splits;
  const int split = blockIdx.x % p.n_splits;
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.L, k_begin + p.keys_per_split);
  const int n_tiles = (k_end - k_begin + KT - 1) / KT;  // >= 1 (the host leaves no split empty)

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(acc_done, 1);
    mbar_init(mma_idle, 1);
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
      mbar_arrive_expect_tx(bar_q, Q_BYTES);
      for (int kc = 0; kc < NCHUNK; ++kc) tma_load_3d(sq + kc * QCHUNK, &tmQt, bar_q, kc * 64, 0, b);
      // The latents of this split are one contiguous range; an L2 prefetch
      // stream kPrefetchTiles ahead of the ring hides DRAM latency without
      // more shared memory.
      const uint8_t *crow = reinterpret_cast<const uint8_t *>(p.C + ((size_t)b * p.Lmax) * p.dc);
      const size_t key_bytes = (size_t)p.dc * 2;
      auto prefetch_tile = [&](int jt) {
        const int kb = k_begin + jt * KT;
        if (jt < n_tiles) prefetch_l2_bulk(crow + (size_t)kb * key_bytes, (uint32_t)(min(KT, k_end - kb) * key_bytes));
      };
      for (int jt = 1; jt < kPrefetchTiles; ++jt) prefetch_tile(jt);
      const int n_chunks = n_tiles * NCHUNK;
      int issued = 0;
      for (int g = 0; g < n_chunks; ++g) {
        const int s = g % NSLOT, use = g / NSLOT, j = g / NCHUNK, kc = g % NCHUNK;
        if (kc == 0) prefetch_tile(j + kPrefetchTiles);
        if (!mbar_wait(&c_empty[s], (use & 1) ^ 1, p.status)) break;
        mbar_arrive_expect_tx(&c_full[s], CCHUNK);
        tma_load_3d(sc + s * CCHUNK, &tmC, &c_full[s], kc * 64, k_begin + j * KT, b);
        issued = g + 1;
      }
      // Error path: let the copies still in flight land before the CTA exits.
      if (issued < n_chunks)
        for (int g = max(0, issued - NSLOT); g < issued; ++g)
          mbar_wait_limit(&c_full[g % NSLOT], (g / NSLOT) & 1, p.status, kDrainLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(KT, HMAX, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, HMAX, true, false);
      const uint32_t aq = smem_u32(sq), ac = smem_u32(sc), ap = smem_u32(sp);
      auto score_chunks = [&](int j, int kc0, int kc1) -> bool {
        for (int kc = kc0; kc < kc1; ++kc) {
          const int g = j * NCHUNK + kc;
          // TMA completion on the mbarrier orders the copy before the MMA's reads
          if (!mbar_wait(&c_full[g % NSLOT], (g / NSLOT) & 1, p.status)) return false;
          const uint32_t cst = ac + (g % NSLOT) * CCHUNK;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ss(tmem + TM_S, sdesc_sw128(cst + kk * 32, 16, 1024),
                         sdesc_sw128(aq + kc * QCHUNK + kk * 32, 16, 1024), idS, (kc | kk) ? 1u : 0u);
        }
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, p.status);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          // S^T is single-buffered: the softmax must have read S^T_{j-1}.
          if (j >= 1 && !mbar_wait(s_free, (j - 1) & 1, p.status)) break;
          tc_fence_after();
          if (!score_chunks(j, 0, NEARLY)) break;
        }
        if (j >= 1) {
          const int jp = j - 1;
          if (!mbar_wait(p_full, jp & 1, p.status)) break;
          tc_fence_after();
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
            const int g0 = jp * NCHUNK + 2 * blk;  // even, so g0 % NSLOT and the next slot are adjacent
            const uint32_t cst = ac + (g0 % NSLOT) * CCHUNK;
#pragma unroll
            for (int ks = 0; ks < KT / 16; ++ks)
              umma_bf16_ss(tmem + TM_ACC + blk * HMAX, sdesc_sw128(cst + ks * 2048, CCHUNK, 1024),
                           sdesc_sw128(ap + ks * 32, 16, 1024), idPV, (jp > 0 || ks > 0) ? 1u : 0u);
            umma_commit(&c_empty[g0 % NSLOT]);
            umma_commit(&c_empty[(g0 + 1) % NSLOT]);
          }
          if (jp == n_tiles - 1) umma_commit(acc_done);
        }
        if (j < n_tiles) {
          if (!score_chunks(j, NEARLY, NCHUNK)) break;
          umma_commit(s_full);  // also orders P^T and acc^T after the value MMAs of tile j-1
        }
      }
      // Every path: wait until the MMAs issued so far have finished before
      // the CTA releases TMEM.
      umma_commit(mma_idle);
      mbar_wait_limit(mma_idle, 0, p.status, kDrainLimitNs);
    }
  } else {
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int r8 = lane >> 2, c4 = lane & 3;
    const int keyA = 16 * quarter + r8;  // tile rows of v[4i + e] (keyA) and v[4i + 2 + e] (keyA + 8)
    float m[24], ls[24];
#pragma unroll
    for (int k = 0; k < 24; ++k) {
      m[k] = -INFINITY;
      ls[k] = 0.f;
    }
    float *wbase = p.weights ? p.weights + (size_t)b * p.H * (size_t)p.L : nullptr;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(s_full, j & 1, p.status));
      float v[48];
      if (got) {
        tc_fence_after();
        tmem_ld_m64_96(tmem + lane_off + TM_S, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
      }
      const int k0 = k_begin + j * KT;
      const bool okA = got && k0 + keyA < k_end, okB = got && k0 + keyA + 8 < k_end;
      float mx[24];
      bool need = !got;
#pragma unroll
      for (int i = 0; i < 12; ++i)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float a = okA ? v[4 * i + e] : -INFINITY;
          const float c = okB ? v[4 * i + 2 + e] : -INFINITY;
          v[4 * i + e] = a;
          v[4 * i + 2 + e] = c;
          mx[2 * i + e] = fmaxf(a, c);
          need |= mx[2 * i + e] > m[2 * i + e] + kRescaleThreshold;
        }
      if (wbase) {
#pragma unroll
        for (int i = 0; i < 12; ++i)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 8 * i + 2 * c4 + e;
            if (h < p.H) {
              float *w = wbase + (size_t)h * p.L + k0 + keyA;
              if (okA) w[0] = v[4 * i + e];
              if (okB) w[8] = v[4 * i + 2 + e];
            }
          }
      }
      if (bar_or(1, 128, need)) {
        if (bar_or(1, 128, !got)) {  // a wait gave up: every softmax thread leaves together
          ok = false;
          break;
        }
        // exact tile max per head: over the 8 threads sharing c4, then over the quarters
#pragma unroll
        for (int k = 0; k < 24; ++k) {
          mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 4));
          mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 8));
          mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 16));
        }
        if (r8 == 0) {
#pragma unroll
          for (int i = 0; i < 12; ++i)
#pragma unroll
            for (int e = 0; e < 2; ++e) red_s[quarter * HMAX + 8 * i + 2 * c4 + e] = mx[2 * i + e];
        }
        bar_sync(1, 128);
#pragma unroll
        for (int i = 0; i < 12; ++i)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 8 * i + 2 * c4 + e, k = 2 * i + e;
            const float tm = fmaxf(fmaxf(red_s[h], red_s[HMAX + h]), fmaxf(red_s[2 * HMAX + h], red_s[3 * HMAX + h]));
            float alpha = 1.f;
            if (tm > m[k] + kRescaleThreshold) {
              if (m[k] != -INFINITY) alpha = fast_exp2(m[k] - tm);
              m[k] = tm;
            }
            ls[k] *= alpha;
            if (quarter == 0 && r8 == 0) alpha_s[h] = alpha;
          }
        bar_sync(1, 128);  // alpha_s complete
        if (j > 0) {
          // acc^T lanes are d_c rows, columns are heads: scale column h by
          // alpha_s[h].  The value MMAs of tile j-1 have completed (s_full).
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
            for (int c = 0; c < HMAX; c += 32) {
              float a[32];
              const uint32_t ta = tmem + lane_off + TM_ACC + blk * HMAX + c;
              tmem_ld32(ta, a);
#pragma unroll
              for (int i = 0; i < 32; ++i) a[i] *= alpha_s[c + i];
              tmem_st32(ta, a);
            }
          }
        }
        bar_sync(1, 128);  // red_s and alpha_s are rewritten by a later tile
      }
      // probabilities, rounded to bfloat16 into P^T (free: the value MMAs of
      // tile j-1 completed before s_full of tile j)
#pragma unroll
      for (int i = 0; i < 12; ++i)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 8 * i + 2 * c4 + e, k = 2 * i + e;
          const float mref = (m[k] == -INFINITY) ? 0.f : m[k];
          const float pa = fast_exp2(v[4 * i + e] - mref), pb = fast_exp2(v[4 * i + 2 + e] - mref);
          ls[k] += pa + pb;
          *reinterpret_cast<uint16_t *>(sp + pt_offset(h, keyA)) = __bfloat16_as_ushort(__float2bfloat16_rn(pa));
          *reinterpret_cast<uint16_t *>(sp + pt_offset(h, keyA + 8)) = __bfloat16_as_ushort(__float2bfloat16_rn(pb));
        }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }

    // partial state of this split: m, l per head and acc^T
    if (ok) {
      const bool fin = !bar_or(1, 128, !mbar_wait(acc_done, 0, p.status));
      if (fin) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 24; ++k) {
          ls[k] += __shfl_xor_sync(0xffffffffu, ls[k], 4);
          ls[k] += __shfl_xor_sync(0xffffffffu, ls[k], 8);
          ls[k] += __shfl_xor_sync(0xffffffffu, ls[k], 16);
        }
        if (r8 == 0) {
#pragma unroll
          for (int i = 0; i < 12; ++i)
#pragma unroll
            for (int e = 0; e < 2; ++e) red_s[quarter * HMAX + 8 * i + 2 * c4 + e] = ls[2 * i + e];
        }
        bar_sync(1, 128);
        const size_t rec = ((size_t)split * p.B + b) * p.H;
        if (quarter == 0 && r8 == 0) {
#pragma unroll
          for (int i = 0; i < 12; ++i)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int h = 8 * i + 2 * c4 + e;
              if (h < p.H) {
                p.part_m[rec + h] = m[2 * i + e];
                p.part_l[rec + h] = (red_s[h] + red_s[HMAX + h]) + (red_s[2 * HMAX + h] + red_s[3 * HMAX + h]);
              }
            }
        }
        const int row = quarter * 32 + lane;  // d_c row within a block
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          const int col = blk * 128 + row;  // latent column
#pragma unroll 1
          for (int c = 0; c < HMAX; c += 32) {
            float a[32];
            tmem_ld32(tmem + lane_off + TM_ACC + blk * HMAX + c, a);
            if (col < p.dc) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c + i < p.H) p.part_acc[(rec + c + i) * (size_t)p.dc + col] = a[i];
            }
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

size_t smem_bytes() {
  return 1024 + Q_BYTES + P_BYTES + NSLOT * CCHUNK + 128 * 4 + 4 * HMAX * 4 + 8 * (1 + 2 * NSLOT + 5) + 16;
}

}  // namespace latent_tc

int latent_tc_tile_keys() { return latent_tc::KT; }

int launch_latent_tc(const CUtensorMap &tmQt, const CUtensorMap &tmC, const uint16_t *C, long long Lmax, int B, int L,
                     int H, int dc, int n_splits, int keys_per_split, float *part_m, float *part_l, float *part_acc,
                     float *weights, unsigned *status, cudaStream_t stream) {
  using namespace latent_tc;
  auto kern = latent_decode_kernel;
  const size_t smem = smem_bytes();
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

// Split-KV decode over the latent cache on tcgen05 tensor cores.
//
// One CTA streams the latents [k_begin, k_end) of one sequence b and keeps an
// online-softmax state for all H (<= 96) heads at once; every latent tile is
// read from HBM once and used twice, as keys and as values:
//   S      [head, key]  = q~ C_tile^T          M=128 (heads, zero-padded by
//                                               overlap), N=KT keys, K=d_c
//   acc^T  [d_c, head] += C_tile^T P^T^T       M=128 per d_c block, N=96 heads,
//                                               K=KT keys (C tile read MN-major)
// with P^T [head, key] = 2^(S - m_head) in shared memory.  q~ = scale*log2(e) *
// W_k^(h)T q_h comes from the absorb kernel (bfloat16), so S is already in
// the exp2 domain.  P is rounded to bfloat16 before it multiplies the
// latents, as in the eager attention path ("Kimi K3 - Softmax over keys":
// float32 softmax, probabilities cast to the input type).
//
// What bounds this kernel on sm_100a, and the shape that follows from it:
//  * an SM takes in at most ~22.5 bytes per cycle through TMA, from L2 as
//    from HBM, so the 1 KB latent row of a key costs >= 45 cycles of ingress
//    and the latent stream has to stay in flight without gaps;
//  * a tcgen05.mma with N <= 128 costs ~56-66 cycles whatever its M and N, so
//    the MMA count per key sets the compute floor: 32 score MMAs per tile
//    (d_c / 16, whatever KT) and 4 value MMAs per 16 keys (a probe without
//    one eighth of the score MMAs ran 8 % faster: the time follows the count;
//    the same MMAs with A read from TMEM instead ran slower);
//  * the MMA-issuing thread must not stall: a wait on its own recent MMAs
//    (through a barrier and another warp) drains the MMA pipe, an acquire
//    mbarrier wait between small MMAs costs ~270 cycles even when the phase
//    has completed (a relaxed poll plus fence.acq_rel costs ~90), and each
//    tcgen05.commit ~95.
// Tiles of KT = 48 keys (kLatentTileKeys; 64 also builds): 0.92 MMAs per key,
// and a 20-chunk latent ring (2.5 tiles) next to the 96 KB of q~ and the 9 KB
// of P^T, so every load of tile j reuses a slot of tile j-2 or j-3 and
// streams while tiles j-1 and j-2 are still in use.  64-key tiles need only
// 0.75 MMAs per key, but their 14-chunk ring (1.75 tiles: shared memory is
// full) makes the last chunk pair of tile j wait for the value MMAs of tile
// j-1, which measured slower.
// S is double-buffered in TMEM (2 x 64 columns next to the 384 of acc^T), so
// the score MMAs of the next tile never wait for the softmax; the score and
// value MMAs come from two threads, so the value MMAs of a tile go out as
// soon as its probabilities are ready (releasing ring slots early) while
// score MMAs keep the pipe busy; and the ring moves in chunk pairs, so a tile
// costs the score thread three waits and one commit and the value thread one
// wait and four commits (the value thread mostly waits for probabilities, so
// releasing each pair as soon as its value MMAs finish costs it nothing and
// starts the load that reuses the slot up to three blocks earlier).
//
//   warp 0      TMA producer: q~ once, then the latents in 64-column chunks
//               (KT keys x 64 d_c) through the ring
//   warp 1      TMEM owner; issues the score MMAs (one thread)
//   warps 2..5  softmax, one head per TMEM lane; lazy rescale of acc^T when a
//               head's running max grows by more than 2^8; partial-state store
//   warp 6      issues the value MMAs (one thread)
// Two issuing threads: a wait of one (for data, for the softmax) does not
// leave the tensor pipe idle while the other has MMAs to issue.
//
// q~ in shared memory: eight 64-column chunks of 96 rows (12 KB each) placed
// 12 KB apart.  The score MMA reads 128-row A tiles, so rows 96..127 of chunk
// k alias rows 0..31 of chunk k+1, and those of the last chunk the first 4 KB
// of the P^T buffer that follows q~: they only feed S rows 96..127, which
// nothing reads.
//
// TMEM columns: S buffers at 0 and 64 (KT columns each), acc^T blocks at
// 128 + 96*blk.
#include "internal.h"
#include "ptx.cuh"
#include "ws_layout.h"

namespace gmla {
namespace latent_tc {

constexpr int HMAX = 96;
constexpr int KT = kLatentTileKeys;       // keys per tile (48 or 64): N of the score product
static_assert(KT == 48 || KT == 64, "tile keys");
constexpr int NUM_THREADS = 224;
constexpr int NCHUNK = 8;                 // 64-wide d_c chunks per tile (d_c <= 512)
constexpr int QCHUNK = HMAX * 128;        // 12 KB: one d_c chunk of q~ for 96 heads
constexpr int Q_BYTES = NCHUNK * QCHUNK;  // 96 KB
// P^T [head, key] in 8-row x 16-byte core matrices without swizzle: heads
// 8g..8g+7 at g * P_SBO, their keys 8c..8c+7 at c * 128 within that group (no
// padding of a head's 96-byte row of 48 keys to the 128 bytes a swizzled row takes).
constexpr int P_SBO = (KT / 8) * 128;     // bytes per group of 8 heads
constexpr int P_BYTES = (HMAX / 8) * P_SBO;  // 9 KB (48-key tiles) or 12 KB (64)
constexpr int CCHUNK = KT * 128;          // one d_c chunk of a tile: KT keys x 64 d_c (6 or 8 KB)
constexpr int PBUF = 1;                   // P^T buffers (2: the softmax of tile j waits for tile j-2's value MMAs)
constexpr int NSLOT = KT == 64 ? 14 : (PBUF == 2 ? 18 : 20);  // latent ring depth in chunks
constexpr int NPAIR = NSLOT / 2;          // the ring moves in chunk pairs (one 128-row d_c block)
constexpr int NPT = NCHUNK / 2;           // chunk pairs per tile
constexpr int NEARLY_PAIRS = 2;           // chunk pairs of tile j behind the score thread's first data wait
constexpr int NTB = 4;                    // tile-indexed barriers rotate over 4 tiles
constexpr float kRescaleThreshold = 8.0f;
constexpr int kPrefetchTiles = 2;         // L2 prefetch distance of the latent stream
constexpr int TM_S = 0;                   // S buffers at TM_S + 64*i
constexpr int TM_ACC = 128;               // acc^T blocks: 128 + 96*blk
constexpr unsigned long long kDrainLimitNs = 100000000ull;  // 100 ms: error-path drain of copies / MMAs

// Ring reuse: the chunks move in pairs (2i, 2i+1) -- the two halves of d_c
// block i -- through NPAIR pair slots.  Pair q of tile j sits in pair slot
// (4j + q) % NPAIR, so its previous user is pair 4j + q - NPAIR: with 9 pair
// slots (48-key tiles) a pair of tile j-2 or j-3; with 7 (64-key tiles) pair
// q+1 of tile j-2 for q < 3 and pair 0 of tile j-1 for q = 3.  A load of tile
// j therefore waits only on tiles j-2 and before, whose value MMAs went out
// while the score MMAs of tile j-1 ran, or (64-key tiles, pair 3) on a
// release of tile j-1 that needs nothing of tile j.  No wait is on a later
// tile, so the ring cannot deadlock.  The two chunks of a pair are adjacent,
// so one MN-major descriptor with a chunk-sized leading offset spans the
// 128-row d_c block.
//
// Barriers are per tile (rotating over NTB tiles), not per slot: a tile costs
// the score thread two data waits (pairs 0..1, pairs 2..3) and the value
// thread one release commit per pair, after that d_c block's value MMAs.
// Waiting first for two pairs rather than three lets the score MMAs of a tile
// start one pair earlier; a first wait for a single pair leaves a longer
// second wait and measured slower.  A rotating barrier is never more than one
// phase away from the phase its waiter wants: the producer arms tile j only
// after a release of tile j-2 or j-3, by which time the MMA threads have
// consumed tile j-NTB; the producer waits for a release of tile j-2 or j-3
// only after it observed the releases of tiles j-4 and earlier.
static_assert(NSLOT % 2 == 0 && NPAIR >= NPT + NEARLY_PAIRS, "early pairs of tile j reuse slots of tile j-2");
static_assert(P_BYTES >= 32 * 128, "P^T buffer must cover the q~ tail");
static_assert(PBUF == 1 || (PBUF == 2 && KT == 48), "a second P^T buffer fits next to the 48-key ring only");

struct Params {
  const uint16_t *C;  // latent cache [B, Lmax, dc] (for the L2 prefetch stream)
  long long Lmax;
  int B, L, H, dc, n_splits, keys_per_split;
  int k_base;                         // first key of split 0 (the keys of a sequence are [k_base, L))
  float *part_m, *part_l, *part_acc;  // [S,B,H], [S,B,H], [S,B,H,512]
  float *weights;                     // optional raw log2-domain scores [B,H,w_ld]
  int w_ld;                           // row stride of weights (L, or Lmax with per-sequence lengths)
  // Per-sequence lengths (null: every sequence has L rows): lens[b] rows of
  // sequence b are visible, read through tmC_seq[b], a 2-D map (d_c, lens[b])
  // whose row extent makes a ragged last tile read zeros past lens[b].
  const CUtensorMap *tmC_seq;
  const int *lens;
  // Work items (null: blockIdx = b * n_splits + split): this CTA streams rows
  // [items[i].y, items[i].z) of sequence items[i].x into record items[i].w of
  // the [R, H] partial states.
  const int4 *items;
  unsigned *status;
};

// 48 consecutive float32 columns of this thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ld48(uint32_t taddr, float *v) {
  uint32_t r[48];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47}, "
      "[%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47])
      : "r"(taddr), "r"(taddr + 32)
      : "memory");
#pragma unroll
  for (int i = 0; i < 48; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive float32 columns of this thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float *v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr), "r"(taddr + 32)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
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

__global__ void __launch_bounds__(NUM_THREADS, 1)
    latent_decode_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmC,
                         const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sq = base;
  uint8_t *sp = sq + Q_BYTES;  // directly after q~: it holds the padded rows' tail
  uint8_t *sc = sp + PBUF * P_BYTES;  // Q_BYTES + P_BYTES is a multiple of 1024
  float *alpha_s = reinterpret_cast<float *>(sc + NSLOT * CCHUNK);
  uint64_t *bars = reinterpret_cast<uint64_t *>(alpha_s + 128);
  uint64_t *bar_q = bars;
  uint64_t *full_e = bars + 1;           // [NTB]: pairs 0..NEARLY_PAIRS-1 of tile j landed
  uint64_t *full_l = full_e + NTB;       // [NTB]: the remaining pairs of tile j landed
  uint64_t *rel = full_l + NTB;          // [NTB][NPT]: pair q of tile j released
  uint64_t *s_full = rel + NPT * NTB;    // [2]
  uint64_t *s_free = s_full + 2;         // [2]: the softmax has read S buffer i
  uint64_t *p_full = s_free + 2;
  uint64_t *acc_done = p_full + 1;
  uint64_t *mma_idle = acc_done + 1;     // [2]: one per issuing thread
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_idle + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int b, k_begin, k_end;
  size_t rec;  // first of this CTA's H partial-state records
  if (p.items) {
    const int4 it = p.items[blockIdx.x];
    b = it.x;
    k_begin = it.y;
    k_end = it.z;
    rec = (size_t)it.w * p.H;
  } else {
    b = blockIdx.x / p.n_splits;
    const int split = blockIdx.x % p.n_splits;
    const int Lb = p.lens ? p.lens[b] : p.L;
    k_begin = p.k_base + split * p.keys_per_split;
    k_end = min(Lb, k_begin + p.keys_per_split);
    rec = ((size_t)split * p.B + b) * p.H;
  }
  if (k_end <= k_begin) {
    // A split past the end of a shorter sequence: an empty partial state,
    // which the combine skips.  The whole CTA leaves before any barrier.
    for (int h = threadIdx.x; h < p.H; h += NUM_THREADS) {
      p.part_m[rec + h] = -INFINITY;
      p.part_l[rec + h] = 0.f;
    }
    return;
  }
  const int n_tiles = (k_end - k_begin + KT - 1) / KT;  // >= 1

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int t = 0; t < NTB; ++t) {
      mbar_init(&full_e[t], NEARLY_PAIRS);
      mbar_init(&full_l[t], NPT - NEARLY_PAIRS);
      for (int q = 0; q < NPT; ++q) mbar_init(&rel[NPT * t + q], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&mma_idle[i], 1);
    }
    mbar_init(p_full, 4);
    mbar_init(acc_done, 1);
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
      const CUtensorMap *mC = p.tmC_seq ? p.tmC_seq + b : &tmC;
      if (p.tmC_seq) fence_tensormap_acquire(mC);
      tma_prefetch_desc(&tmQt);
      tma_prefetch_desc(mC);
      mbar_arrive_expect_tx(bar_q, Q_BYTES);
      for (int kc = 0; kc < NCHUNK; ++kc) tma_load_3d(sq + kc * QCHUNK, &tmQt, bar_q, kc * 64, 0, b);
      // The latents of this split are one contiguous range; a short L2
      // prefetch stream ahead of the ring starts the DRAM reads early.
      const uint8_t *crow = reinterpret_cast<const uint8_t *>(p.C + ((size_t)b * p.Lmax) * p.dc);
      const size_t key_bytes = (size_t)p.dc * 2;
      auto prefetch_tile = [&](int jt) {
        const int kb = k_begin + jt * KT;
        if (jt < n_tiles) prefetch_l2_bulk(crow + (size_t)kb * key_bytes, (uint32_t)(min(KT, k_end - kb) * key_bytes));
      };
      for (int jt = 1; jt < kPrefetchTiles; ++jt) prefetch_tile(jt);
      const int n_pairs = n_tiles * NPT;
      int issued = 0;
      for (int g = 0; g < n_pairs; ++g) {
        const int ps = g % NPAIR, j = g / NPT, q = g % NPT;
        if (q == 0) prefetch_tile(j + kPrefetchTiles);
        if (g >= NPAIR) {  // the slot's previous pair: pair q' of tile t
          const int gp = g - NPAIR, t = gp / NPT, qp = gp % NPT;
          if (!mbar_wait(&rel[NPT * (t % NTB) + qp], (t / NTB) & 1, p.status)) break;
        }
        uint64_t *fb = q < NEARLY_PAIRS ? &full_e[j % NTB] : &full_l[j % NTB];
        mbar_arrive_expect_tx(fb, 2 * CCHUNK);
        for (int h2 = 0; h2 < 2; ++h2) {
          if (p.tmC_seq)
            tma_load_2d(sc + (2 * ps + h2) * CCHUNK, mC, fb, (2 * q + h2) * 64, k_begin + j * KT);
          else
            tma_load_3d(sc + (2 * ps + h2) * CCHUNK, mC, fb, (2 * q + h2) * 64, k_begin + j * KT, b);
        }
        issued = g + 1;
      }
      // Error path: let the copies still in flight land before the CTA exits
      // (the tiles whose loads were issued and not consumed: at most 3).
      if (issued < n_pairs)
        for (int j = max(0, (issued - NPAIR) / NPT); j * NPT < issued; ++j) {
          mbar_wait_limit(&full_e[j % NTB], (j / NTB) & 1, p.status, kDrainLimitNs);
          if ((j + 1) * NPT <= issued) mbar_wait_limit(&full_l[j % NTB], (j / NTB) & 1, p.status, kDrainLimitNs);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- score MMAs
      constexpr uint32_t idS = idesc_bf16_f32(128, KT, false, false);
      const uint32_t aq = smem_u32(sq), ac = smem_u32(sc);
      // Score MMAs of chunk pairs [q0, q1) of tile j into S buffer j&1.
      auto score_pairs = [&](int j, int q0, int q1) -> bool {
        const uint32_t dS = tmem + TM_S + (j & 1) * 64;
        // TMA completion on the mbarrier orders the copies before the MMA's reads
        if (!mbar_wait_relaxed(q0 == 0 ? &full_e[j % NTB] : &full_l[j % NTB], (j / NTB) & 1, p.status)) return false;
        for (int q = q0; q < q1; ++q) {
          const int g = j * NPT + q;
          const uint32_t cst = ac + (g % NPAIR) * 2 * CCHUNK;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(dS, sdesc_sw128(aq + (2 * q + h2) * QCHUNK + kk * 32, 16, 1024),
                           sdesc_sw128(cst + h2 * CCHUNK + kk * 32, 16, 1024), idS, (q | h2 | kk) ? 1u : 0u);
        }
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, p.status);
      for (int j = 0; ok && j < n_tiles; ++j) {
        // S buffer j&1 was last read by the softmax of tile j-2
        if (j >= 2 && !mbar_wait_relaxed(&s_free[j & 1], ((j - 2) >> 1) & 1, p.status)) break;
        tc_fence_after();
        if (!score_pairs(j, 0, NEARLY_PAIRS) || !score_pairs(j, NEARLY_PAIRS, NPT)) break;
        umma_commit(&s_full[j & 1]);
      }
      // Every path: wait until this thread's MMAs have finished before the
      // CTA releases TMEM.
      umma_commit(&mma_idle[0]);
      mbar_wait_limit(&mma_idle[0], 0, p.status, kDrainLimitNs);
    }
  } else if (warp == 6) {
    if (lane == 0) {
      // ---------------------------------------------------------------- value MMAs
      constexpr uint32_t idPV = idesc_bf16_f32(128, HMAX, true, false);
      const uint32_t ac = smem_u32(sc), ap = smem_u32(sp);
      for (int j = 0; j < n_tiles; ++j) {
        if (!mbar_wait_relaxed(p_full, j & 1, p.status)) break;
        tc_fence_after();
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const int g = j * NPT + blk;
          const uint32_t cst = ac + (g % NPAIR) * 2 * CCHUNK;
#pragma unroll
          for (int ks = 0; ks < KT / 16; ++ks)
            umma_bf16_ss(tmem + TM_ACC + blk * HMAX, sdesc_sw128(cst + ks * 2048, CCHUNK, 1024),
                         sdesc_noswizzle(ap + (j % PBUF) * P_BYTES + ks * 256, 128, P_SBO), idPV,
                         (j > 0 || ks > 0) ? 1u : 0u);
          // the last release also tells the softmax of tile j+1 that P^T and acc^T are free
          umma_commit(&rel[NPT * (j % NTB) + blk]);
        }
        if (j == n_tiles - 1) umma_commit(acc_done);
      }
      umma_commit(&mma_idle[1]);
      mbar_wait_limit(&mma_idle[1], 0, p.status, kDrainLimitNs);
    }
  } else {
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int h = quarter * 32 + lane;  // head owned in the S phase; d_c row in the acc phase
    const bool head_ok = h < p.H;
    const bool active = quarter < 3;  // lanes 96..127 of S hold only padding rows
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    uint8_t *prow = sp + (h >> 3) * P_SBO + (h & 7) * 16;
    float *wrow = (p.weights && head_ok) ? p.weights + ((size_t)b * p.H + h) * (size_t)p.w_ld : nullptr;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1;
      // a suspending wait: polling warps would take shared-memory bandwidth from the MMAs
      const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1, p.status));
      float x[KT];
      if (got) {
        tc_fence_after();
        if (active) {
          if constexpr (KT == 64)
            tmem_ld64(tmem + lane_off + TM_S + sb * 64, x);
          else
            tmem_ld48(tmem + lane_off + TM_S + sb * 64, x);
        } else {
#pragma unroll
          for (int c = 0; c < KT; ++c) x[c] = -INFINITY;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
      }
      const int k0 = k_begin + j * KT;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < KT; ++c) {
        if (!got || k0 + c >= k_end) x[c] = -INFINITY;
        mx = fmaxf(mx, x[c]);
      }
      if (wrow) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (k0 + c < k_end) wrow[k0 + c] = x[c];
      }
      const bool need = head_ok && mx > m_used + kRescaleThreshold;
      // P^T buffer j % PBUF is free once the value MMAs of tile j - PBUF have completed
      bool ready = got;
      if (got && j >= PBUF) {
        const int jp = j - PBUF;
        ready = __all_sync(0xffffffffu, mbar_wait(&rel[NPT * (jp % NTB) + NPT - 1], (jp / NTB) & 1, p.status));
        tc_fence_after();
      }
      if (bar_or(1, 128, need || !ready)) {
        if (bar_or(1, 128, !ready)) {  // a wait gave up: every softmax thread leaves together
          ok = false;
          break;
        }
        if (PBUF > 1 && j >= 1) {
          // the rescale below touches acc^T: the value MMAs of tile j-1 must have completed
          const int jp = j - 1;
          const bool r1 = __all_sync(0xffffffffu, mbar_wait(&rel[NPT * (jp % NTB) + NPT - 1], (jp / NTB) & 1, p.status));
          if (bar_or(1, 128, !r1)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        float alpha = 1.f;
        if (need) {
          if (m_used != -INFINITY) alpha = fast_exp2(m_used - mx);
          m_used = mx;
        }
        l *= alpha;
        alpha_s[h] = alpha;
        bar_sync(1, 128);  // alpha_s complete
        if (j > 0) {
          // acc^T lanes are d_c rows, columns are heads: scale column h by
          // alpha_s[h].  The value MMAs of tile j-1 have completed (rel).
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
        bar_sync(1, 128);  // alpha_s is rewritten by a later tile
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
      l += rs;
      // P^T row h of buffer j % PBUF (free: the value MMAs of tile j - PBUF have completed)
      if (active) {
#pragma unroll
        for (int u = 0; u < KT / 8; ++u)
          *reinterpret_cast<uint4 *>(prow + (j % PBUF) * P_BYTES + u * 128) =
              make_uint4(pk[u * 4 + 0], pk[u * 4 + 1], pk[u * 4 + 2], pk[u * 4 + 3]);
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

constexpr size_t smem_bytes() {
  return 1024 + Q_BYTES + PBUF * P_BYTES + NSLOT * CCHUNK + 128 * 4 + 8 * (1 + (2 + NPT) * NTB + 8) + 16;
}
static_assert(smem_bytes() <= 232448, "dynamic shared memory above the 227 KB a CTA may have");
static_assert((Q_BYTES + PBUF * P_BYTES) % 1024 == 0, "the latent ring must start on a 1024-byte boundary");

}  // namespace latent_tc

int latent_tc_tile_keys() { return latent_tc::KT; }

int launch_latent_tc(const CUtensorMap &tmQt, const CUtensorMap &tmC, const uint16_t *C, long long Lmax, int B, int L,
                     int k_base, int H, int dc, int n_splits, int keys_per_split, float *part_m, float *part_l,
                     float *part_acc, float *weights, int w_ld, const CUtensorMap *tmC_seq, const int *lens,
                     const LatentItem *items, int n_items, unsigned *status, cudaStream_t stream) {
  using namespace latent_tc;
  auto kern = latent_decode_kernel;
  const size_t smem = smem_bytes();
  if (!set_smem_limit_once(reinterpret_cast<const void *>(kern), (int)smem, kSmemLatentTc)) return -1;
  Params p;
  p.C = C;
  p.Lmax = Lmax;
  p.B = B;
  p.L = L;
  p.k_base = k_base;
  p.H = H;
  p.dc = dc;
  p.n_splits = n_splits;
  p.keys_per_split = keys_per_split;
  p.part_m = part_m;
  p.part_l = part_l;
  p.part_acc = part_acc;
  p.weights = weights;
  p.w_ld = w_ld;
  p.tmC_seq = tmC_seq;
  p.lens = lens;
  p.items = reinterpret_cast<const int4 *>(items);
  p.status = status;
  const long long grid = items ? (long long)n_items : (long long)B * n_splits;
  if (grid < 1 || grid > 0x7fffffffLL) return -1;
  kern<<<(unsigned)grid, NUM_THREADS, smem, stream>>>(tmQt, tmC, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

// Persistent tcgen05 GEMM:  D[m, n] = sum_k A[m, k] * B[n, k]  (bf16 in,
// float32 accumulate in TMEM, bf16 out), for the "X W^T" products of the
// "Gated MLA" page: [Q | G | C] = X [W_q; W_g; W_c]^T, [K | V] = C [W_k; W_v]^T
// and Y = O_gated W_o^T.  Up to three problems share the A operand and run
// in one launch (their N ranges are concatenated).
//
// Tiles are 128 x 256 with K chunks of 64 (one 128-byte swizzle atom wide).
//   warp 0      TMA producer, 4-stage ring (A 16 KB + B 32 KB per stage)
//   warp 1      TMEM owner and MMA issuer: per chunk 4 x tcgen05.mma
//               (M=128, N=256, K=16), both operands K-major
//   warps 2..5  epilogue: TMEM -> registers -> bf16, one output row per
//               thread; two TMEM accumulators (2 x 256 columns) let the
//               epilogue of tile i overlap the main loop of tile i+1.  Each
//               warp stages its 32 rows x 64 columns in shared memory (two
//               4 KB buffers, 128-byte swizzle) and one lane writes them out
//               with a TMA bulk store, so the store of one chunk overlaps the
//               conversion of the next and the writes leave as whole lines.
//               Boxes that would cross an output batch or the end of the rows
//               (and outputs whose layout TMA cannot address) are written by
//               per-thread 16-byte stores instead.
// The tile order walks groups of 16 m-tiles across all n-tiles so the CTAs
// resident at one time share A rows and B columns in L2.
#include "internal.h"
#include "launch_plan.h"
#include "ptx.cuh"

namespace gmla {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int NUM_THREADS = 192;
constexpr int GROUP_M = 16;

constexpr int OUT_ROWS = 32, OUT_COLS = 64;          // one epilogue warp's store box
constexpr int OUT_BYTES = OUT_ROWS * OUT_COLS * 2;    // 4 KB

struct Smem {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
  uint8_t out[4][2][OUT_BYTES];  // per epilogue warp, double-buffered
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

struct Params {
  GemmArgs g;
  int m_tiles_per_b;
  int m_tiles;        // over all batches
  int n_tiles[3];
  int n_tiles_total;
  int total_tiles;
  int k_chunks;
  int tma_out[3];     // problem i is written through tmO_i (3-D map: N, rows_per_b, batches; box 64 x 32 x 1)
};

struct TileCoord {
  int prob, mt, nt;
};

__device__ __forceinline__ TileCoord tile_coord(const Params &P, int idx) {
  // groups of GROUP_M m-tiles; inside a group n-tiles advance slowest
  const int group_span = GROUP_M * P.n_tiles_total;
  const int grp = idx / group_span;
  const int first_m = grp * GROUP_M;
  const int gm = min(GROUP_M, P.m_tiles - first_m);
  const int rem = idx - grp * group_span;
  const int ntg = rem / gm;
  TileCoord c;
  c.mt = first_m + rem % gm;
  int p = 0, nt = ntg;
  while (p < 2 && nt >= P.n_tiles[p]) {
    nt -= P.n_tiles[p];
    ++p;
  }
  c.prob = p;
  c.nt = nt;
  return c;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                const __grid_constant__ CUtensorMap tmO2, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  unsigned *status = P.g.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], 4);
    }
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
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      if (P.g.n_problems > 1) tma_prefetch_desc(&tmB1);
      if (P.g.n_problems > 2) tma_prefetch_desc(&tmB2);
      uint32_t g = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < P.total_tiles; idx += gridDim.x) {
        const TileCoord tc = tile_coord(P, idx);
        const CUtensorMap *mb = tc.prob == 0 ? &tmB0 : (tc.prob == 1 ? &tmB1 : &tmB2);
        const int bidx = tc.mt / P.m_tiles_per_b;
        const int row = P.g.a_row0 + (tc.mt % P.m_tiles_per_b) * BM;
        for (int kc = 0; kc < P.k_chunks; ++kc, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(&sm.empty[s], ((g / STAGES) & 1) ^ 1, status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
          tma_load_3d(sm.a[s], &tmA, &sm.full[s], kc * BK, row, bidx);
          tma_load_2d(sm.b[s], mb, &sm.full[s], kc * BK, tc.nt * BN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      uint32_t g = 0;
      int it = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < P.total_tiles; idx += gridDim.x, ++it) {
        const int ab = it & 1;
        if (!mbar_wait(&sm.acc_empty[ab], ((it >> 1) & 1) ^ 1, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tD = tmem + ab * BN;
        for (int kc = 0; kc < P.k_chunks; ++kc, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(&sm.full[s], (g / STAGES) & 1, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t aa = smem_u32(sm.a[s]), bb = smem_u32(sm.b[s]);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_ss(tD, sdesc_sw128(aa + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 32, 16, 1024), idesc,
                         (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&sm.empty[s]);
        }
        if (ok) umma_commit(&sm.acc_full[ab]);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint32_t staged = 0;  // boxes this warp has handed to TMA (buffer rotation)
    int it = 0;
    for (int idx = blockIdx.x; idx < P.total_tiles; idx += gridDim.x, ++it) {
      const TileCoord tc = tile_coord(P, idx);
      const int ab = it & 1;
      if (!mbar_wait(&sm.acc_full[ab], (it >> 1) & 1, status)) break;
      tc_fence_after();
      const GemmOut &o = P.g.prob[tc.prob];
      const CUtensorMap *mo = tc.prob == 0 ? &tmO0 : (tc.prob == 1 ? &tmO1 : &tmO2);
      const int bidx = tc.mt / P.m_tiles_per_b;
      const int t = (tc.mt % P.m_tiles_per_b) * BM + r;
      const bool row_ok = t < P.g.a_rows;
      const long long m = (long long)bidx * P.g.a_rows + t;
      uint16_t *orow = o.out + (m / o.rows_per_b) * o.sb + (m % o.rows_per_b) * o.st + o.off;
      // this warp's 32 rows as one box: all inside the problem's rows and inside one output batch
      const int t_box = t - lane;
      const long long m_box = m - lane;
      const bool boxed = P.tma_out[tc.prob] && t_box + OUT_ROWS <= P.g.a_rows &&
                         m_box % o.rows_per_b + OUT_ROWS <= o.rows_per_b;
      const uint32_t tD = tmem + ab * BN + lane_off;
#pragma unroll 1
      for (int c = 0; c < BN / OUT_COLS; ++c) {
        float v[OUT_COLS];
        tmem_ld32(tD + c * OUT_COLS, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(tD + c * OUT_COLS + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        const int n0 = tc.nt * BN + c * OUT_COLS;
        if (n0 >= o.N) continue;
        if (boxed) {
          uint8_t *buf = sm.out[quarter][staged & 1];
          if (staged >= 2) {
            if (lane == 0) bulk_wait_group_read<1>();  // the store that used this buffer has read it
            __syncwarp();
          }
          // row `lane` of the box: 16-byte chunk q at position q ^ (row % 8) (128-byte swizzle)
          uint4 *dst = reinterpret_cast<uint4 *>(buf + lane * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q ^ (lane & 7)] =
                make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]), pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                           pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]), pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(mo, buf, n0, (int)(m_box % o.rows_per_b), (int)(m_box / o.rows_per_b));
            bulk_commit_group();
          }
          ++staged;
        } else if (row_ok) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (n0 + 32 * h >= o.N) break;
            uint4 *dst = reinterpret_cast<uint4 *>(orow + n0 + 32 * h);
            const float *w = v + 32 * h;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(w[q * 8 + 0], w[q * 8 + 1]), pack_bf16x2(w[q * 8 + 2], w[q * 8 + 3]),
                                  pack_bf16x2(w[q * 8 + 4], w[q * 8 + 5]), pack_bf16x2(w[q * 8 + 6], w[q * 8 + 7]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
    }
    if (lane == 0) bulk_wait_group<0>();  // the bulk stores have finished before the CTA exits
    __syncwarp();
  }

  __syncwarp();  // lane 0 of the producer / MMA warps ran its loop alone
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ------------------------------------------------------------------ few rows
// With at most 32 output rows (a decode step: one new token per sequence) a
// launch of 128 x 256 tiles has fewer tiles than SMs (W_o at d_model = 12288:
// 48, the [Q | G | C] projection 98), and each CTA is capped by what it can
// pull in while the other SMs idle.  This kernel takes tiles NB columns wide
// (256 or 192: narrower tiles give more CTAs, each streaming fewer weight
// rows), and with sk = 2 a cluster of two CTAs shares one tile, each taking a
// contiguous half of the K chunks; CTA 1 stages its float32 partial rows in
// its own shared memory and sends them to CTA 0 with one bulk copy, and CTA 0
// adds them to its accumulator and writes the bf16 tile.  Only TMEM lanes
// 0..31 (the rows) carry data, so one epilogue warp per CTA does the work; the
// A loads bring in those 32 rows only, and the MMA's rows 32..127 read whatever
// the A buffer holds there, which reaches only lanes nothing reads.
constexpr int SK_MAX = 2;
constexpr int SK_STAGES = 4;
constexpr int SK_ROWS = 32;
constexpr int SK_A_BYTES = SK_ROWS * BK * 2;  // the A box: 32 rows (4 KB) at the start of a 128-row A buffer

template <int NB>
struct SmemSK {
  static constexpr int B_TILE = NB * BK * 2;    // 32 or 24 KB
  static constexpr int PART = SK_ROWS * NB * 4;  // one CTA's float32 partial rows
  uint8_t a[SK_STAGES][A_BYTES];
  uint8_t b[SK_STAGES][B_TILE];
  uint8_t part[SK_MAX - 1][PART];  // CTA 0: partials received; others: slot 0 stages their own
  uint64_t full[SK_STAGES];
  uint64_t empty[SK_STAGES];
  uint64_t acc_full;
  uint64_t recv;  // CTA 0: the partials of CTAs 1 .. SK-1 have landed
  uint32_t tmem_base;
};
template <int NB>
constexpr size_t smem_bytes_sk() { return sizeof(SmemSK<NB>) + 1024; }

// 16-byte chunk q (of NB/4) of row r of a partial, swizzled so that a warp
// whose lanes hold consecutive rows touches all banks.
template <int NB>
__device__ __forceinline__ uint32_t sk_off(int r, int q) { return r * (NB * 4) + ((q ^ (r & 7)) << 4); }

template <int NB>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                       const Params P, const int sk) {
  static_assert(NB == 256 || NB == 192, "few-row tile width");
  constexpr uint32_t TM_COLS = 256;  // NB float32 accumulator columns, allocated as a power of two
  using Sm = SmemSK<NB>;
  extern __shared__ uint8_t smem_raw[];
  Sm &sm = *reinterpret_cast<Sm *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  unsigned *status = P.g.status;
  const int rank = (int)cluster_ctarank();  // 0 without a cluster (sk = 1)
  const int tile = blockIdx.x / sk;
  const int kc0 = (int)((long long)P.k_chunks * rank / sk), kc1 = (int)((long long)P.k_chunks * (rank + 1) / sk);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.recv, 1);
    if (rank == 0) mbar_arrive_expect_tx(&sm.recv, (uint32_t)(sk - 1) * Sm::PART);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of every CTA initialised (CTA 0's receive barrier armed)
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const TileCoord tc = tile_coord(P, tile);

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap *mb = tc.prob == 0 ? &tmB0 : (tc.prob == 1 ? &tmB1 : &tmB2);
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(mb);
      for (int kc = kc0, g = 0; kc < kc1; ++kc, ++g) {
        const int s = g % SK_STAGES;
        if (!mbar_wait(&sm.empty[s], ((g / SK_STAGES) & 1) ^ 1, status)) break;
        mbar_arrive_expect_tx(&sm.full[s], SK_A_BYTES + Sm::B_TILE);
        tma_load_3d(sm.a[s], &tmA, &sm.full[s], kc * BK, P.g.a_row0, 0);
        tma_load_2d(sm.b[s], mb, &sm.full[s], kc * BK, tc.nt * NB);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, NB, false, false);
      bool ok = true;
      for (int kc = kc0, g = 0; kc < kc1; ++kc, ++g) {
        const int s = g % SK_STAGES;
        if (!(ok = mbar_wait(&sm.full[s], (g / SK_STAGES) & 1, status))) break;
        tc_fence_after();
        const uint32_t aa = smem_u32(sm.a[s]), bb = smem_u32(sm.b[s]);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16_ss(tmem, sdesc_sw128(aa + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 32, 16, 1024), idesc,
                       (kc > kc0 || kk > 0) ? 1u : 0u);
        umma_commit(&sm.empty[s]);
      }
      if (ok) umma_commit(&sm.acc_full);
    }
  } else if ((warp & 3) == 0) {
    // the epilogue warp of TMEM lanes 0..31: row `lane` of the tile
    const bool got = mbar_wait(&sm.acc_full, 0, status);
    tc_fence_after();
    if (rank != 0) {
      // stage this CTA's partial rows and send them to CTA 0
      uint8_t *stage = sm.part[0];
#pragma unroll 1
      for (int c = 0; c < NB / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + c * 32, v);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4 *>(stage + sk_off<NB>(lane, c * 8 + q)) =
              got ? make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t dst = mapa_shared(smem_u32(sm.part[rank - 1]), 0);
        bulk_copy_to_peer(dst, stage, Sm::PART, mapa_shared(smem_u32(&sm.recv), 0));
      }
    } else {
      const bool have = mbar_wait(&sm.recv, 0, status) && got;
      const GemmOut &o = P.g.prob[tc.prob];
      const int t = lane;  // row
      const bool row_ok = have && t < P.g.a_rows;
      uint16_t *orow = o.out + (t / o.rows_per_b) * o.sb + (t % o.rows_per_b) * o.st + o.off;
#pragma unroll 1
      for (int c = 0; c < NB / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + c * 32, v);
        for (int s2 = 0; s2 < sk - 1; ++s2) {
          const uint8_t *part = sm.part[s2];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 u = *reinterpret_cast<const float4 *>(part + sk_off<NB>(lane, c * 8 + q));
            v[4 * q] += u.x;
            v[4 * q + 1] += u.y;
            v[4 * q + 2] += u.z;
            v[4 * q + 3] += u.w;
          }
        }
        const int n0 = tc.nt * NB + c * 32;
        if (row_ok && n0 < o.N) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + n0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]), pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                                pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]), pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
        }
      }
    }
    tc_fence_before();
  }

  __syncwarp();
  // CTA 0 has received every partial before any CTA of the cluster leaves (a
  // CTA's shared memory must outlive the copies that read or write it)
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace gemm

namespace {

static_assert(gemm::SK_ROWS == kFewRowsMax && gemm::SK_MAX == kFewRowsSplitMax, "few-row plan and kernel agree");

// The few-row plan (launch_plan.h) measured at M = 32, K = 12288 on B200: W_o
// in 48 tiles of 256 split in two (96 CTAs) 68 us, in 64 of 192 split in two
// (128 CTAs) 66 us; the [Q | G | C] projection in 98 tiles of 256 112 us, in
// 131 of 192 106 us.  Three-CTA clusters (144 CTAs for W_o) measured 105 us,
// and splits that need a second wave were slower.

template <int NB>
int launch_few_rows(const CUtensorMap &tmA, const CUtensorMap *tmB, gemm::Params P, int sk, SmemSlot slot,
                    cudaStream_t stream) {
  using namespace gemm;
  auto kern = gemm_splitk_kernel<NB>;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(kern), (int)smem_bytes_sk<NB>(), slot)) return -1;
  P.n_tiles_total = 0;
  for (int i = 0; i < 3; ++i) {
    P.n_tiles[i] = i < P.g.n_problems ? (P.g.prob[i].N + NB - 1) / NB : 0;
    P.n_tiles_total += P.n_tiles[i];
  }
  P.total_tiles = P.m_tiles * P.n_tiles_total;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(P.total_tiles * sk));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem_bytes_sk<NB>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)sk;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap &b1 = P.g.n_problems > 1 ? tmB[1] : tmB[0];
  const CUtensorMap &b2 = P.g.n_problems > 2 ? tmB[2] : tmB[0];
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB[0], b1, b2, P, sk) == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_gemm(const GemmArgs &a, cudaStream_t stream) {
  using namespace gemm;
  Params P;
  P.g = a;
  P.m_tiles_per_b = (a.a_rows + BM - 1) / BM;
  P.m_tiles = P.m_tiles_per_b * a.a_batches;
  P.n_tiles_total = 0;
  for (int i = 0; i < 3; ++i) {
    P.n_tiles[i] = i < a.n_problems ? (a.prob[i].N + BN - 1) / BN : 0;
    P.n_tiles_total += P.n_tiles[i];
  }
  P.total_tiles = P.m_tiles * P.n_tiles_total;
  P.k_chunks = (a.K + BK - 1) / BK;
  if (P.total_tiles <= 0 || P.k_chunks <= 0) return 0;
  const int sms = num_sms();
  int Ns[3] = {0, 0, 0};
  for (int i = 0; i < a.n_problems; ++i) Ns[i] = a.prob[i].N;
  const FewRowsPlan few = few_rows_plan(a.a_rows, a.a_batches, Ns, a.n_problems, P.k_chunks, sms);
  // The A map: boxes of 128 rows, or of the 32 rows the few-row kernel uses
  // (the tile's other rows feed accumulator lanes nothing reads, so they are
  // not loaded at all rather than filled with zeros).
  CUtensorMap tmA;
  const unsigned bA[3] = {(unsigned)BK, (unsigned)(few.nb ? SK_ROWS : BM), 1};
  if (!make_tmap_bf16(&tmA, a.a, 3, a.a_dims, a.a_strides, bA)) return -1;
  // B maps (K, N_i), one box of the tile's width in N
  CUtensorMap tmB[3];
  for (int i = 0; i < a.n_problems; ++i) {
    const long long dB[2] = {a.K, a.prob[i].N}, sB[1] = {a.prob[i].w_ld};
    const unsigned bB[2] = {(unsigned)BK, (unsigned)(few.nb ? few.nb : BN)};
    if (!make_tmap_bf16(&tmB[i], a.prob[i].w, 2, dB, sB, bB)) return -1;
  }
  if (few.nb == 256) return launch_few_rows<256>(tmA, tmB, P, few.sk, kSmemGemmSK, stream);
  if (few.nb == 192) return launch_few_rows<192>(tmA, tmB, P, few.sk, kSmemGemmSK192, stream);

  if (!set_smem_limit_once(reinterpret_cast<const void *>(gemm_kernel), (int)kSmemBytes, kSmemGemm)) return -1;
  // Output maps: problem i is stored by TMA when its rows can be described as
  // a 3-D tiled map (16-byte aligned base and row / batch strides).
  CUtensorMap tmO[3];
  const long long rows_total = (long long)a.a_rows * a.a_batches;
  for (int i = 0; i < 3; ++i) {
    P.tma_out[i] = 0;
    if (i >= a.n_problems) continue;
    const GemmOut &o = a.prob[i];
    const uint16_t *base = o.out + o.off;
    const long long nb = (rows_total + o.rows_per_b - 1) / o.rows_per_b;
    const long long sb = nb > 1 ? o.sb : o.rows_per_b * o.st;
    const bool addressable = (reinterpret_cast<uintptr_t>(base) & 15) == 0 && o.st % 8 == 0 && sb % 8 == 0 &&
                             o.st >= o.N && sb >= o.rows_per_b * o.st && o.N > 0;
    if (!addressable) continue;
    const long long dims[3] = {o.N, o.rows_per_b, nb}, strides[2] = {o.st, sb};
    const unsigned box[3] = {OUT_COLS, OUT_ROWS, 1};
    P.tma_out[i] = make_tmap_bf16(&tmO[i], base, 3, dims, strides, box) ? 1 : 0;
  }
  for (int i = 0; i < 3; ++i)
    if (!P.tma_out[i]) tmO[i] = tmA;  // never read: the kernel stores problem i directly
  const int grid = P.total_tiles < sms ? P.total_tiles : sms;
  const CUtensorMap &b1 = a.n_problems > 1 ? tmB[1] : tmB[0];
  const CUtensorMap &b2 = a.n_problems > 2 ? tmB[2] : tmB[0];
  gemm_kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tmA, tmB[0], b1, b2, tmO[0], tmO[1], tmO[2], P);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

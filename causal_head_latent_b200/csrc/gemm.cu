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
//   warps 2..5  epilogue: TMEM -> registers -> bf16 -> global, one output
//               row per thread; two TMEM accumulators (2 x 256 columns) let
//               the epilogue of tile i overlap the main loop of tile i+1.
// The tile order walks groups of 16 m-tiles across all n-tiles so the CTAs
// resident at one time share A rows and B columns in L2.
#include "internal.h"
#include "ptx.cuh"

namespace gmla {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int NUM_THREADS = 192;
constexpr int GROUP_M = 16;

struct Smem {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
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
                const Params P) {
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
    int it = 0;
    for (int idx = blockIdx.x; idx < P.total_tiles; idx += gridDim.x, ++it) {
      const TileCoord tc = tile_coord(P, idx);
      const int ab = it & 1;
      if (!mbar_wait(&sm.acc_full[ab], (it >> 1) & 1, status)) break;
      tc_fence_after();
      const GemmOut &o = P.g.prob[tc.prob];
      const int bidx = tc.mt / P.m_tiles_per_b;
      const int t = (tc.mt % P.m_tiles_per_b) * BM + r;
      const bool row_ok = t < P.g.a_rows;
      const long long m = (long long)bidx * P.g.a_rows + t;
      uint16_t *orow = o.out + (m / o.rows_per_b) * o.sb + (m % o.rows_per_b) * o.st + o.off;
      const uint32_t tD = tmem + ab * BN + lane_off;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tD + c * 32, v);
        const int n0 = tc.nt * BN + c * 32;
        if (row_ok && n0 < o.N) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + n0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]), pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                                pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]), pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
    }
  }

  __syncwarp();  // lane 0 of the producer / MMA warps ran its loop alone
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gemm

int launch_gemm(const CUtensorMap &tmA, const CUtensorMap *tmB, const GemmArgs &a, cudaStream_t stream) {
  using namespace gemm;
  if (!set_smem_limit_once(reinterpret_cast<const void *>(gemm_kernel), (int)kSmemBytes, kSmemGemm)) return -1;
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
  const int grid = P.total_tiles < num_sms() ? P.total_tiles : num_sms();
  const CUtensorMap &b1 = a.n_problems > 1 ? tmB[1] : tmB[0];
  const CUtensorMap &b2 = a.n_problems > 2 ? tmB[2] : tmB[0];
  gemm_kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tmA, tmB[0], b1, b2, P);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gmla

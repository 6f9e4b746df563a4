// C-ABI entry points of libgmla.so (declared in include/gmla.h).
//
// Every entry point checks its arguments on the host, builds the TMA tensor
// maps it needs, and launches on the caller's stream.  Nothing is allocated
// per call: scratch lives in a caller workspace.  A device status word
// (one per device) collects in-kernel timeouts; gmla_get_device_status reads
// and clears it.
#include <math.h>
#include <mutex>

#include "../../include/gmla.h"
#include <vector>

#include "internal.h"
#include "ptx.cuh"
#include "ws_layout.h"

namespace gmla {

__device__ unsigned g_status_word;

static constexpr int kMaxDevices = 64;
static unsigned *g_status_ptr[kMaxDevices];
static int g_num_sms[kMaxDevices];
static std::mutex g_mu;

static int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

// Per-device set-up: the status word's device address and the SM count.
static bool device_setup(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status_ptr[dev]) return true;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return false;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  g_num_sms[dev] = sms;
  g_status_ptr[dev] = static_cast<unsigned *>(p);
  // Commit the scratch array of gmla_attend_decode_noalloc on this device now
  // (its lookup loads the device code that holds it), so that a caller's first
  // call of any entry point, not its first no-alloc decode, is the one that
  // takes that memory.  A failure here is reported by the no-alloc call itself.
  (void)latent_noalloc_scratch_address();
  return true;
}

int num_sms() {
  const int d = current_device();
  return (d >= 0 && d < kMaxDevices && g_num_sms[d] > 0) ? g_num_sms[d] : 148;
}

bool set_smem_limit_once(const void *kernel, int bytes, SmemSlot slot) {
  static bool done[kSmemSlots][kMaxDevices];
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices || slot < 0 || slot >= kSmemSlots) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (done[slot][d]) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done[slot][d] = true;
  return true;
}

static unsigned *status_ptr() {
  const int d = current_device();
  if (!device_setup(d)) return nullptr;
  return g_status_ptr[d];
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tiled map with 128-byte swizzle.  dims/strides in elements, dim 0 innermost (contiguous).
bool make_tmap_bf16(CUtensorMap *m, const void *base, int rank, const long long *dims, const long long *strides,
                     const unsigned *box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = (cuuint64_t)dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = (cuuint64_t)strides[i] * 2;  // bytes, dims 1..rank-1
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// One thread waits, with a short bounded limit, on an mbarrier that nothing
// arrives at: the wait runs out, records the timeout in the status word and the
// kernel returns normally.
__global__ void wait_timeout_kernel(unsigned *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_limit(&bar, 0, status, limit_ns);
  }
}

}  // namespace gmla

using namespace gmla;

extern "C" {

int gmla_version(void) { return 100; }

const char *gmla_status_string(gmla_status s) {
  switch (s) {
    case GMLA_OK: return "ok";
    case GMLA_ERR_ARG: return "invalid argument";
    case GMLA_ERR_UNSUPPORTED: return "unsupported size or option";
    case GMLA_ERR_CUDA: return "CUDA error";
    case GMLA_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    case GMLA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

gmla_status gmla_get_device_status(gmla_stream_t stream) {
  unsigned *sp = status_ptr();
  if (!sp) return GMLA_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GMLA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, sp, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return GMLA_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpy(sp, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return GMLA_ERR_CUDA;
  }
  if (v & kStatusTimeout) return GMLA_ERR_TIMEOUT;
  if (v) return GMLA_ERR_CUDA;
  return GMLA_OK;
}

gmla_status gmla_selftest_wait_timeout(unsigned milliseconds, gmla_stream_t stream) {
  if (milliseconds == 0 || milliseconds > 1000) return GMLA_ERR_ARG;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(st, 1000000ull * milliseconds);
  return cudaGetLastError() == cudaSuccess ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ projections

// [Q | G | C] = X [W_q; W_g; W_c]^T and [K | V] = C [W_k; W_v]^T for the heads
// [h0, h1) (rows 128*h0 .. 128*h1-1 of W_q, W_g, W_k, W_v; the latent is
// always full width).
static gmla_status latent_project_heads(const gmla_bf16 *X, int64_t B, int64_t T, int64_t d_model, int64_t h0,
                                        int64_t h1, const gmla_bf16 *W_q, const gmla_bf16 *W_g, const gmla_bf16 *W_c,
                                        int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v, gmla_bf16 *Q,
                                        gmla_bf16 *G, gmla_bf16 *C, int64_t cache_len_max, int64_t cache_pos,
                                        gmla_bf16 *K, gmla_bf16 *V, gmla_stream_t stream) {
  if (!X || B <= 0 || T <= 0 || d_model <= 0) return GMLA_ERR_ARG;
  if ((Q && !W_q) || (G && !W_g) || (C && !W_c) || (K && !W_k) || (V && !W_v)) return GMLA_ERR_ARG;
  if ((K || V) && !C) return GMLA_ERR_ARG;
  if (C && (d_c <= 0 || cache_pos < 0 || cache_len_max <= 0 || cache_pos + T > cache_len_max)) return GMLA_ERR_ARG;
  const void *ptrs[] = {X, W_q, W_g, W_c, W_k, W_v, Q, G, C, K, V};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (d_model % 128 != 0 || (C && d_c % 64 != 0)) return GMLA_ERR_UNSUPPORTED;
  if (h0 < 0 || h1 <= h0 || h1 > d_model / 128) return GMLA_ERR_ARG;
  if (B * T > 0x7fffffffLL || cache_len_max > 0x7fffffffLL || B > 65535) return GMLA_ERR_UNSUPPORTED;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long M = B * T;
  const long long w = 128 * (h1 - h0);  // output width of Q, G, K, V

  // [Q | G | C] = X [W_q; W_g; W_c]^T
  {
    GemmArgs ga{};
    ga.a = X;
    ga.a_dims[0] = d_model;
    ga.a_dims[1] = M;
    ga.a_dims[2] = 1;
    ga.a_strides[0] = d_model;
    ga.a_strides[1] = M * d_model;
    ga.a_rows = (int)M;
    ga.a_batches = 1;
    ga.a_row0 = 0;
    ga.K = (int)d_model;
    ga.status = st;
    int np = 0;
    const gmla_bf16 *Ws[3] = {W_q ? W_q + 128 * h0 * d_model : nullptr, W_g ? W_g + 128 * h0 * d_model : nullptr,
                              W_c};
    gmla_bf16 *Os[3] = {Q, G, C};
    for (int i = 0; i < 3; ++i) {
      if (!Os[i]) continue;
      const long long N = i == 2 ? d_c : w;
      GemmOut &o = ga.prob[np];
      o.w = Ws[i];
      o.w_ld = d_model;
      o.out = Os[i];
      o.N = (int)N;
      if (i == 2) {  // latent rows go to cache rows [cache_pos, cache_pos + T) of each batch
        o.rows_per_b = T;
        o.sb = cache_len_max * d_c;
        o.st = d_c;
        o.off = cache_pos * d_c;
      } else {
        o.rows_per_b = M;
        o.sb = 0;
        o.st = w;
        o.off = 0;
      }
      ++np;
    }
    ga.n_problems = np;
    if (np > 0 && launch_gemm(ga, s) != 0) return GMLA_ERR_CUDA;
  }
  // [K | V] = C [W_k; W_v]^T, reading the bf16 latents just written to the cache
  if (K || V) {
    GemmArgs ga{};
    ga.a = C;
    ga.a_dims[0] = d_c;
    ga.a_dims[1] = cache_pos + T;
    ga.a_dims[2] = B;
    ga.a_strides[0] = d_c;
    ga.a_strides[1] = cache_len_max * d_c;
    ga.a_rows = (int)T;
    ga.a_batches = (int)B;
    ga.a_row0 = (int)cache_pos;
    ga.K = (int)d_c;
    ga.status = st;
    int np = 0;
    const gmla_bf16 *Ws[2] = {W_k ? W_k + 128 * h0 * d_c : nullptr, W_v ? W_v + 128 * h0 * d_c : nullptr};
    gmla_bf16 *Os[2] = {K, V};
    for (int i = 0; i < 2; ++i) {
      if (!Os[i]) continue;
      GemmOut &o = ga.prob[np];
      o.w = Ws[i];
      o.w_ld = d_c;
      o.out = Os[i];
      o.N = (int)w;
      o.rows_per_b = M;
      o.sb = 0;
      o.st = w;
      o.off = 0;
      ++np;
    }
    ga.n_problems = np;
    if (launch_gemm(ga, s) != 0) return GMLA_ERR_CUDA;
  }
  return GMLA_OK;
}

gmla_status gmla_latent_project(const gmla_bf16 *X, int64_t B, int64_t T, int64_t d_model, const gmla_bf16 *W_q,
                                const gmla_bf16 *W_g, const gmla_bf16 *W_c, int64_t d_c, const gmla_bf16 *W_k,
                                const gmla_bf16 *W_v, gmla_bf16 *Q, gmla_bf16 *G, gmla_bf16 *C,
                                int64_t cache_len_max, int64_t cache_pos, gmla_bf16 *K, gmla_bf16 *V,
                                gmla_stream_t stream) {
  if (d_model <= 0) return GMLA_ERR_ARG;
  if (d_model % 128 != 0) return GMLA_ERR_UNSUPPORTED;
  return latent_project_heads(X, B, T, d_model, 0, d_model / 128, W_q, W_g, W_c, d_c, W_k, W_v, Q, G, C,
                              cache_len_max, cache_pos, K, V, stream);
}

gmla_status gmla_latent_project_heads(const gmla_bf16 *X, int64_t B, int64_t T, int64_t d_model, int64_t head_begin,
                                      int64_t head_end, const gmla_bf16 *W_q, const gmla_bf16 *W_g,
                                      const gmla_bf16 *W_c, int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v,
                                      gmla_bf16 *Q, gmla_bf16 *G, gmla_bf16 *C, int64_t cache_len_max,
                                      int64_t cache_pos, gmla_bf16 *K, gmla_bf16 *V, gmla_stream_t stream) {
  return latent_project_heads(X, B, T, d_model, head_begin, head_end, W_q, W_g, W_c, d_c, W_k, W_v, Q, G, C,
                              cache_len_max, cache_pos, K, V, stream);
}

// ------------------------------------------------------------------ K/V expansion of cached latents

gmla_status gmla_expand_kv(const gmla_bf16 *C, int64_t B, int64_t cache_len_max, int64_t row0, int64_t rows,
                           int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v, int64_t d_model, gmla_bf16 *K,
                           gmla_bf16 *V, gmla_stream_t stream) {
  if (!C || (!K && !V) || (K && !W_k) || (V && !W_v)) return GMLA_ERR_ARG;
  if (B <= 0 || rows <= 0 || row0 < 0 || d_c <= 0 || d_model <= 0 || cache_len_max <= 0 ||
      row0 + rows > cache_len_max)
    return GMLA_ERR_ARG;
  const void *ptrs[] = {C, W_k, W_v, K, V};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (d_model % 128 != 0 || d_c % 64 != 0) return GMLA_ERR_UNSUPPORTED;
  if (B * rows > 0x7fffffffLL || cache_len_max > 0x7fffffffLL || B > 65535) return GMLA_ERR_UNSUPPORTED;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  GemmArgs ga{};
  ga.a = C;
  ga.a_dims[0] = d_c;
  ga.a_dims[1] = row0 + rows;
  ga.a_dims[2] = B;
  ga.a_strides[0] = d_c;
  ga.a_strides[1] = cache_len_max * d_c;
  ga.a_rows = (int)rows;
  ga.a_batches = (int)B;
  ga.a_row0 = (int)row0;
  ga.K = (int)d_c;
  ga.status = st;
  int np = 0;
  const gmla_bf16 *Ws[2] = {W_k, W_v};
  gmla_bf16 *Os[2] = {K, V};
  for (int i = 0; i < 2; ++i) {
    if (!Os[i]) continue;
    GemmOut &o = ga.prob[np];
    o.w = Ws[i];
    o.w_ld = d_c;
    o.out = Os[i];
    o.N = (int)d_model;
    o.rows_per_b = B * rows;
    o.sb = 0;
    o.st = d_model;
    o.off = 0;
    ++np;
  }
  ga.n_problems = np;
  return launch_gemm(ga, static_cast<cudaStream_t>(stream)) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ attention over explicit Q, K, V

gmla_status gmla_attend_prefill(const gmla_bf16 *Q, const int64_t q_strides[3], const gmla_bf16 *K,
                                const int64_t k_strides[3], const gmla_bf16 *V, const int64_t v_strides[3],
                                int64_t B, int64_t H, int64_t Tq, int64_t Tk, int64_t D_h, int causal, float scale,
                                const gmla_bf16 *G, gmla_bf16 *O, const int64_t o_strides[3], float *lse,
                                float *weights, gmla_stream_t stream) {
  if (!Q || !K || !V || !O || !q_strides || !k_strides || !v_strides || !o_strides) return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || Tq < 0 || Tk <= 0 || Tq > Tk || D_h <= 0) return GMLA_ERR_ARG;
  if (causal != 0 && causal != 1) return GMLA_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (G && !aligned16(G))) return GMLA_ERR_ARG;
  for (int i = 0; i < 3; ++i) {
    if (q_strides[i] <= 0 || k_strides[i] <= 0 || v_strides[i] <= 0 || o_strides[i] <= 0) return GMLA_ERR_ARG;
    if (q_strides[i] % 8 || k_strides[i] % 8 || v_strides[i] % 8 || o_strides[i] % 8) return GMLA_ERR_ARG;
  }
  if (D_h != 128) return GMLA_ERR_UNSUPPORTED;
  if (B > 0xffff || H > 0xffff || Tk > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  if (Tq == 0) return GMLA_OK;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  if (Tq <= 4) {
    RowsArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.G = G; a.O = O;
    for (int i = 0; i < 3; ++i) {
      a.qs[i] = q_strides[i]; a.ks[i] = k_strides[i]; a.vs[i] = v_strides[i]; a.os[i] = o_strides[i];
    }
    a.lse = lse; a.weights = weights;
    a.B = (int)B; a.H = (int)H; a.Tq = (int)Tq; a.Tk = (int)Tk; a.causal = causal;
    a.scale = scale; a.status = st;
    return launch_attn_rows(a, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
  }

  CUtensorMap tq, tk, tv;
  const unsigned box[4] = {64, 128, 1, 1};
  {
    const long long d[4] = {128, Tq, H, B}, sd[3] = {q_strides[1], q_strides[2], q_strides[0]};
    if (!make_tmap_bf16(&tq, Q, 4, d, sd, box)) return GMLA_ERR_CUDA;
  }
  {
    const long long d[4] = {128, Tk, H, B}, sd[3] = {k_strides[1], k_strides[2], k_strides[0]};
    if (!make_tmap_bf16(&tk, K, 4, d, sd, box)) return GMLA_ERR_CUDA;
  }
  {
    const long long d[4] = {128, Tk, H, B}, sd[3] = {v_strides[1], v_strides[2], v_strides[0]};
    if (!make_tmap_bf16(&tv, V, 4, d, sd, box)) return GMLA_ERR_CUDA;
  }
  PrefillArgs a{};
  a.G = G; a.O = O;
  for (int i = 0; i < 3; ++i) a.o_strides[i] = o_strides[i];
  a.lse = lse; a.weights = weights;
  a.B = (int)B; a.H = (int)H; a.Tq = (int)Tq; a.Tk = (int)Tk; a.causal = causal;
  a.scale = scale; a.status = st;
  return launch_attn_prefill(tq, tk, tv, a, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ attention with per-sequence lengths

size_t gmla_attend_prefill_varlen_workspace_size(int64_t B) {
  if (B <= 0) return 0;
  return prefill_varlen_layout_bytes(B);
}

gmla_status gmla_attend_prefill_varlen(const gmla_bf16 *Q, const int64_t q_strides[3], const gmla_bf16 *K,
                                       const int64_t k_strides[3], const gmla_bf16 *V, const int64_t v_strides[3],
                                       int64_t B, int64_t H, int64_t Tq_max, int64_t Tk_max, int64_t D_h,
                                       const int64_t *q_lens, const int64_t *kv_lens, int causal, float scale,
                                       const gmla_bf16 *G, gmla_bf16 *O, const int64_t o_strides[3], float *lse,
                                       void *workspace, size_t workspace_bytes, gmla_stream_t stream) {
  if (!Q || !K || !V || !O || !q_strides || !k_strides || !v_strides || !o_strides || !q_lens || !kv_lens)
    return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || Tq_max <= 0 || Tk_max <= 0 || D_h <= 0) return GMLA_ERR_ARG;
  if (causal != 0 && causal != 1) return GMLA_ERR_ARG;
  for (int64_t b = 0; b < B; ++b)
    if (q_lens[b] < 0 || q_lens[b] > Tq_max || kv_lens[b] < 1 || kv_lens[b] > Tk_max || q_lens[b] > kv_lens[b])
      return GMLA_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (G && !aligned16(G))) return GMLA_ERR_ARG;
  for (int i = 0; i < 3; ++i) {
    if (q_strides[i] <= 0 || k_strides[i] <= 0 || v_strides[i] <= 0 || o_strides[i] <= 0) return GMLA_ERR_ARG;
    if (q_strides[i] % 8 || k_strides[i] % 8 || v_strides[i] % 8 || o_strides[i] % 8) return GMLA_ERR_ARG;
  }
  if (D_h != 128) return GMLA_ERR_UNSUPPORTED;
  if (B > 0xffff || H > 0xffff || Tk_max > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < gmla_attend_prefill_varlen_workspace_size(B)) return GMLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GMLA_ERR_ARG;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // per-sequence 3-D maps (D, length, H) and lengths, copied into the workspace
  // (the map region starts on a 256-byte boundary: TMA reads maps at 64-byte alignment)
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const PrefillVarlenLayout lay = prefill_varlen_layout(reinterpret_cast<uintptr_t>(ws), B);
  CUtensorMap *maps = reinterpret_cast<CUtensorMap *>(ws + lay.maps);
  int *lens = reinterpret_cast<int *>(ws + lay.lens);
  std::vector<CUtensorMap> hm(3 * (size_t)B);
  std::vector<int> hl(2 * (size_t)B);
  const unsigned box[3] = {64, 128, 1};
  for (int64_t b = 0; b < B; ++b) {
    const gmla_bf16 *base[3] = {Q + b * q_strides[0], K + b * k_strides[0], V + b * v_strides[0]};
    const int64_t *str[3] = {q_strides, k_strides, v_strides};
    const long long len[3] = {q_lens[b] > 0 ? q_lens[b] : 1, kv_lens[b], kv_lens[b]};
    for (int i = 0; i < 3; ++i) {
      const long long d[3] = {128, len[i], H}, sd[2] = {str[i][1], str[i][2]};
      if (!make_tmap_bf16(&hm[3 * b + i], base[i], 3, d, sd, box)) return GMLA_ERR_CUDA;
    }
    hl[b] = (int)q_lens[b];
    hl[B + b] = (int)kv_lens[b];
  }
  // pageable sources: the copies are staged before cudaMemcpyAsync returns
  if (cudaMemcpyAsync(maps, hm.data(), hm.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(lens, hl.data(), hl.size() * sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return GMLA_ERR_CUDA;
  CUtensorMap tq, tk, tv;  // unused by the kernel when maps are given; encoded for a valid parameter block
  const unsigned box4[4] = {64, 128, 1, 1};
  {
    const long long d[4] = {128, Tq_max, H, B}, sd[3] = {q_strides[1], q_strides[2], q_strides[0]};
    if (!make_tmap_bf16(&tq, Q, 4, d, sd, box4)) return GMLA_ERR_CUDA;
    const long long dk[4] = {128, Tk_max, H, B}, sk[3] = {k_strides[1], k_strides[2], k_strides[0]};
    if (!make_tmap_bf16(&tk, K, 4, dk, sk, box4)) return GMLA_ERR_CUDA;
    const long long sv[3] = {v_strides[1], v_strides[2], v_strides[0]};
    if (!make_tmap_bf16(&tv, V, 4, dk, sv, box4)) return GMLA_ERR_CUDA;
  }
  PrefillArgs a{};
  a.G = G; a.O = O;
  for (int i = 0; i < 3; ++i) a.o_strides[i] = o_strides[i];
  a.lse = lse; a.weights = nullptr;
  a.B = (int)B; a.H = (int)H; a.Tq = (int)Tq_max; a.Tk = (int)Tk_max; a.causal = causal;
  a.scale = scale; a.status = st;
  a.q_lens = lens; a.kv_lens = lens + B; a.maps = maps;
  return launch_attn_prefill(tq, tk, tv, a, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ decode over the latent cache

size_t gmla_attend_decode_workspace_size(int64_t B, int64_t L, int64_t H, int64_t d_c) {
  if (B <= 0 || L <= 0 || H <= 0 || d_c <= 0) return 0;
  return latent_workspace_bytes(B, L, H, d_c);
}

gmla_status gmla_attend_decode(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B, int64_t cache_len_max, int64_t L,
                               int64_t H, int64_t D_h, int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v,
                               float scale, const gmla_bf16 *G, gmla_bf16 *O, float *weights, void *workspace,
                               size_t workspace_bytes, gmla_stream_t stream) {
  if (!Q || !C || !W_k || !W_v || !O) return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || D_h <= 0 || d_c <= 0 || L < 1 || cache_len_max < L) return GMLA_ERR_ARG;
  const void *ptrs[] = {Q, C, W_k, W_v, G, O, workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (D_h != 128 || d_c % 64 != 0 || d_c > 512 || H > 96) return GMLA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || L > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  const size_t need = latent_workspace_bytes(B, L, H, d_c);
  if (!workspace || workspace_bytes < need) return GMLA_ERR_WORKSPACE;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  LatentArgs a{};
  a.Q = Q; a.C = C; a.Wk = W_k; a.Wv = W_v; a.G = G; a.O = O; a.weights = weights;
  a.cache_len_max = cache_len_max;
  a.B = (int)B; a.L = (int)L; a.H = (int)H; a.dc = (int)d_c;
  a.scale = scale; a.workspace = workspace; a.status = st;
  return launch_attend_latent(a, static_cast<cudaStream_t>(stream)) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ decode with per-sequence lengths

size_t gmla_attend_decode_varlen_workspace_size(int64_t B, int64_t cache_len_max, int64_t H, int64_t d_c) {
  if (B <= 0 || cache_len_max <= 0 || H <= 0 || d_c <= 0) return 0;
  return latent_varlen_workspace_bytes(B, cache_len_max, H, d_c);
}

gmla_status gmla_attend_decode_varlen(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B, int64_t cache_len_max,
                                      const int64_t *lens, int64_t H, int64_t D_h, int64_t d_c, const gmla_bf16 *W_k,
                                      const gmla_bf16 *W_v, float scale, const gmla_bf16 *G, gmla_bf16 *O,
                                      float *weights, void *workspace, size_t workspace_bytes, gmla_stream_t stream) {
  if (!Q || !C || !W_k || !W_v || !O || !lens) return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || D_h <= 0 || d_c <= 0 || cache_len_max < 1) return GMLA_ERR_ARG;
  for (int64_t b = 0; b < B; ++b)
    if (lens[b] < 1 || lens[b] > cache_len_max) return GMLA_ERR_ARG;
  const void *ptrs[] = {Q, C, W_k, W_v, G, O, workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (D_h != 128 || d_c % 64 != 0 || d_c > 512 || H > 96) return GMLA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || cache_len_max > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  const size_t need = latent_varlen_workspace_bytes(B, cache_len_max, H, d_c);
  if (!workspace || workspace_bytes < need) return GMLA_ERR_WORKSPACE;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  LatentArgs a{};
  a.Q = Q; a.C = C; a.Wk = W_k; a.Wv = W_v; a.G = G; a.O = O; a.weights = weights;
  a.cache_len_max = cache_len_max;
  a.B = (int)B; a.L = (int)cache_len_max; a.H = (int)H; a.dc = (int)d_c;
  a.scale = scale; a.workspace = workspace; a.status = st;
  a.lens = reinterpret_cast<const long long *>(lens);
  return launch_attend_latent(a, static_cast<cudaStream_t>(stream)) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ decode state over a key range, and its merge

size_t gmla_attend_decode_partial_workspace_size(int64_t B, int64_t k0, int64_t k1, int64_t H, int64_t d_c) {
  if (B <= 0 || k0 < 0 || k1 <= k0 || H <= 0 || d_c <= 0) return 0;
  return latent_workspace_bytes(B, k1 - k0, H, d_c);
}

gmla_status gmla_attend_decode_partial(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B, int64_t cache_len_max,
                                       int64_t k0, int64_t k1, int64_t H, int64_t D_h, int64_t d_c,
                                       const gmla_bf16 *W_k, float scale, float *lse, float *ctx, void *workspace,
                                       size_t workspace_bytes, gmla_stream_t stream) {
  if (!Q || !C || !W_k || !lse || !ctx) return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || D_h <= 0 || d_c <= 0 || k0 < 0 || k1 < k0 || k1 > cache_len_max) return GMLA_ERR_ARG;
  const void *ptrs[] = {Q, C, W_k, lse, ctx, workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (D_h != 128 || d_c % 64 != 0 || d_c > 512 || H > 96) return GMLA_ERR_UNSUPPORTED;
  if (B > 65535 || cache_len_max > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  if (k1 > k0 && (!workspace || workspace_bytes < latent_workspace_bytes(B, k1 - k0, H, d_c)))
    return GMLA_ERR_WORKSPACE;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k1 == k0) return launch_latent_empty_state(lse, ctx, B, H, d_c, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  LatentArgs a{};
  a.Q = Q; a.C = C; a.Wk = W_k; a.Wv = nullptr; a.G = nullptr; a.O = nullptr; a.weights = nullptr;
  a.cache_len_max = cache_len_max;
  a.B = (int)B; a.L = (int)k1; a.H = (int)H; a.dc = (int)d_c;
  a.scale = scale; a.workspace = workspace; a.status = st;
  a.k0 = k0; a.out_lse = lse; a.out_chat = ctx;
  return launch_attend_latent(a, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

gmla_status gmla_decode_combine(const float *lse, const float *ctx, int64_t n_parts, int64_t B, int64_t H,
                                int64_t D_h, int64_t d_c, const gmla_bf16 *W_v, const gmla_bf16 *G, gmla_bf16 *O,
                                gmla_stream_t stream) {
  if (!lse || !ctx || !W_v || !O) return GMLA_ERR_ARG;
  if (n_parts <= 0 || B <= 0 || H <= 0 || D_h <= 0 || d_c <= 0) return GMLA_ERR_ARG;
  const void *ptrs[] = {lse, ctx, W_v, G, O};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (D_h != 128 || d_c % 64 != 0 || d_c > 512 || n_parts > 1024) return GMLA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return GMLA_ERR_UNSUPPORTED;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  return launch_latent_combine(lse, ctx, (int)n_parts, (int)B, (int)H, (int)d_c, W_v, G, O,
                               static_cast<cudaStream_t>(stream)) == 0
             ? GMLA_OK
             : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ decode without a caller workspace

size_t gmla_attend_decode_noalloc_max_bytes(void) { return latent_noalloc_scratch_bytes(); }

gmla_status gmla_attend_decode_noalloc(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B, int64_t cache_len_max,
                                       int64_t L, int64_t H, int64_t D_h, int64_t d_c, const gmla_bf16 *W_k,
                                       const gmla_bf16 *W_v, float scale, const gmla_bf16 *G, gmla_bf16 *O,
                                       float *weights, gmla_stream_t stream) {
  if (!Q || !C || !W_k || !W_v || !O) return GMLA_ERR_ARG;
  if (B <= 0 || H <= 0 || D_h <= 0 || d_c <= 0 || L < 1 || cache_len_max < L) return GMLA_ERR_ARG;
  const void *ptrs[] = {Q, C, W_k, W_v, G, O};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GMLA_ERR_ARG;
  if (D_h != 128 || d_c % 64 != 0 || d_c > 512 || H > 96) return GMLA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || L > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D_h);
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  LatentArgs a{};
  a.Q = Q; a.C = C; a.Wk = W_k; a.Wv = W_v; a.G = G; a.O = O; a.weights = weights;
  a.cache_len_max = cache_len_max;
  a.B = (int)B; a.L = (int)L; a.H = (int)H; a.dc = (int)d_c;
  a.scale = scale; a.workspace = nullptr; a.status = st;
  const int rc = launch_attend_latent_noalloc(a, static_cast<cudaStream_t>(stream));
  if (rc == -3) return GMLA_ERR_WORKSPACE;
  return rc == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

// ------------------------------------------------------------------ output projection

size_t gmla_gate_out_workspace_size(int64_t M, int64_t d_model) {
  if (M <= 0 || d_model <= 0) return 0;
  return gate_out_layout_bytes(M, d_model);
}

// Y = (sigmoid(G) (.) O) W_o[:, 128*h0 .. 128*h1)^T with O, G [M, 128*(h1-h0)].
static gmla_status gate_out_heads(const gmla_bf16 *O, const gmla_bf16 *G, const gmla_bf16 *W_o, int64_t M,
                                  int64_t d_model, int64_t h0, int64_t h1, gmla_bf16 *Y, void *workspace,
                                  size_t workspace_bytes, gmla_stream_t stream) {
  if (!O || !W_o || !Y || M <= 0 || d_model <= 0) return GMLA_ERR_ARG;
  if (!aligned16(O) || !aligned16(W_o) || !aligned16(Y) || (G && !aligned16(G)) ||
      (workspace && !aligned16(workspace)))
    return GMLA_ERR_ARG;
  if (d_model % 128 != 0 || M > 0x7fffffffLL) return GMLA_ERR_UNSUPPORTED;
  if (h0 < 0 || h1 <= h0 || h1 > d_model / 128) return GMLA_ERR_ARG;
  const long long w = 128 * (h1 - h0);  // width of O and G
  if (G && (!workspace || workspace_bytes < gate_out_layout_bytes(M, w))) return GMLA_ERR_WORKSPACE;
  unsigned *st = status_ptr();
  if (!st) return GMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const gmla_bf16 *A = O;
  if (G) {  // the gated context, staged in the workspace
    gmla_bf16 *gated = reinterpret_cast<gmla_bf16 *>(static_cast<uint8_t *>(workspace) +
                                                     gate_out_layout_offset(reinterpret_cast<uintptr_t>(workspace)));
    if (launch_gate(O, G, gated, (size_t)M * w, s) != 0) return GMLA_ERR_CUDA;
    A = gated;
  }
  GemmArgs ga{};
  ga.a = A;
  ga.a_dims[0] = w;
  ga.a_dims[1] = M;
  ga.a_dims[2] = 1;
  ga.a_strides[0] = w;
  ga.a_strides[1] = M * w;
  // columns 128*h0 .. 128*h1-1 of every row of W_o: a strided sub-matrix
  ga.prob[0].w = W_o + 128 * h0;
  ga.prob[0].w_ld = d_model;
  ga.a_rows = (int)M;
  ga.a_batches = 1;
  ga.a_row0 = 0;
  ga.K = (int)w;
  ga.status = st;
  ga.n_problems = 1;
  ga.prob[0].out = Y;
  ga.prob[0].N = (int)d_model;
  ga.prob[0].rows_per_b = M;
  ga.prob[0].sb = 0;
  ga.prob[0].st = d_model;
  ga.prob[0].off = 0;
  return launch_gemm(ga, s) == 0 ? GMLA_OK : GMLA_ERR_CUDA;
}

gmla_status gmla_gate_out(const gmla_bf16 *O, const gmla_bf16 *G, const gmla_bf16 *W_o, int64_t M, int64_t d_model,
                          gmla_bf16 *Y, void *workspace, size_t workspace_bytes, gmla_stream_t stream) {
  if (d_model <= 0) return GMLA_ERR_ARG;
  if (d_model % 128 != 0) return GMLA_ERR_UNSUPPORTED;
  return gate_out_heads(O, G, W_o, M, d_model, 0, d_model / 128, Y, workspace, workspace_bytes, stream);
}

gmla_status gmla_gate_out_heads(const gmla_bf16 *O, const gmla_bf16 *G, const gmla_bf16 *W_o, int64_t M,
                                int64_t d_model, int64_t head_begin, int64_t head_end, gmla_bf16 *Y, void *workspace,
                                size_t workspace_bytes, gmla_stream_t stream) {
  return gate_out_heads(O, G, W_o, M, d_model, head_begin, head_end, Y, workspace, workspace_bytes, stream);
}

}  // extern "C"

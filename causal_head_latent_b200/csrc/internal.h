// Internal launch interfaces between the C-ABI layer (gmla_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gmla {

// Device status word bits (read back by gmla_get_device_status).
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadIndex = 2u;

// ---------------------------------------------------------------- prefill attention
struct PrefillArgs {
  const uint16_t *G;  // optional gate logits [B, Tq, H*128]
  uint16_t *O;
  long long o_strides[3];
  float *lse;
  float *weights;
  int B, H, Tq, Tk, causal;
  float scale;
  unsigned *status;
  // Optional per-sequence lengths (device arrays of B ints) and per-sequence
  // 3-D maps (D, length, H) of Q, K, V (device array of 3*B maps).
  const int *q_lens = nullptr, *kv_lens = nullptr;
  const CUtensorMap *maps = nullptr;
};
// tmQ/tmK/tmV: 4-D maps (D=128, T, H, B), bf16, box (64, 128, 1, 1), 128-byte swizzle.
int launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                        const PrefillArgs &a, cudaStream_t stream);
size_t attn_prefill_smem_bytes();

// ---------------------------------------------------------------- few-query attention (decode over explicit K/V)
struct RowsArgs {
  const uint16_t *Q, *K, *V, *G;
  long long qs[3], ks[3], vs[3], os[3];
  uint16_t *O;
  float *lse;
  float *weights;
  int B, H, Tq, Tk, causal;
  float scale;
  unsigned *status;
};
int launch_attn_rows(const RowsArgs &a, cudaStream_t stream);

// ---------------------------------------------------------------- tcgen05 GEMM  D = A B^T
// Output row mapping: global row m -> element offset
//   (m / rows_per_b) * sb + (m % rows_per_b) * st + off
struct GemmOut {
  uint16_t *out;
  long long rows_per_b, sb, st, off;
  int N;
  const uint16_t *w;  // the B operand: N rows of K elements, w_ld elements apart
  long long w_ld;
};
struct GemmArgs {
  const uint16_t *a;     // the A operand: a 3-D array (K, rows, batches) ...
  long long a_dims[3];   // ... of these extents (elements) ...
  long long a_strides[2];  // ... with these row and batch strides (elements)
  int a_rows;        // rows per batch of A (rows of the A map's dimension 1 that belong to the problem)
  int a_batches;     // batches (A map dimension 2)
  int a_row0;        // first row coordinate in the A map
  int K;
  int n_problems;    // 1..3, all share A
  GemmOut prob[3];
  unsigned *status;
};
// The tensor maps of A (K, rows, batches) and of each B (K, N_i) are built
// here, with boxes as tall and as wide as the tiles the launch uses.
int launch_gemm(const GemmArgs &a, cudaStream_t stream);

// ---------------------------------------------------------------- decode over the latent cache
struct LatentArgs {
  const uint16_t *Q, *C, *Wk, *Wv, *G;
  uint16_t *O;
  float *weights;
  long long cache_len_max;
  int B, L, H, dc;
  float scale;
  void *workspace;
  unsigned *status;
  // Optional per-sequence lengths (host array of B values in 1..cache_len_max);
  // when set, L is ignored and the split plan and workspace follow cache_len_max.
  const long long *lens = nullptr;
  // Partial form: keys [k0, L) only; the merged state goes to out_lse
  // (natural log, [B,H]) and out_chat ([B,H,dc]) instead of O (out_chat
  // non-null selects the partial form).
  long long k0 = 0;
  float *out_lse = nullptr, *out_chat = nullptr;
};
int launch_attend_latent(const LatentArgs &a, cudaStream_t stream);
// tcgen05 products around the latent decode (attn_latent_side.cu): q~ = scale*log2(e) W_k^(h)T q_h
// ([B,H,dc] bf16) and O = sigmoid(G) (.) W_v^(h) c^ ([B,H*128] bf16); d_c a multiple of 64, <= 512.
int launch_absorb_tc(const uint16_t *Q, const uint16_t *Wk, int B, int H, int dc, float sl2, uint16_t *qt,
                     unsigned *status, cudaStream_t stream);
int launch_wv_tc(const float *chat, const uint16_t *Wv, const uint16_t *G, uint16_t *O, int B, int H, int dc,
                 unsigned *status, cudaStream_t stream);
size_t latent_workspace_bytes(long long B, long long L, long long H, long long dc);
size_t latent_varlen_workspace_bytes(long long B, long long cache_len_max, long long H, long long dc);
// The state of an empty key range (lse = -inf, chat = 0).
int launch_latent_empty_state(float *lse, float *chat, long long B, long long H, long long dc, cudaStream_t stream);
// Merge n partial states (lse [n,B,H] natural log, chat [n,B,H,dc]), then W_v and the gate into O.
int launch_latent_combine(const float *lse, const float *chat, int n, int B, int H, int dc, const uint16_t *Wv,
                          const uint16_t *G, uint16_t *O, cudaStream_t stream);
// Same launches with the scratch in a fixed device array of this library
// (no workspace argument).  Returns 0, -1 (CUDA error) or -3 (too large).
int launch_attend_latent_noalloc(const LatentArgs &a, cudaStream_t stream);
size_t latent_noalloc_scratch_bytes();
// Device address of that array on the current device (looked up once per device).
void *latent_noalloc_scratch_address();

// out = sigmoid(G) (.) O over n bf16 elements (n a multiple of 8, 16-byte aligned pointers).
int launch_gate(const uint16_t *O, const uint16_t *G, uint16_t *out, size_t n, cudaStream_t stream);

int num_sms();
// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel slot, device): the attribute belongs to the
// device's context, so a process that drives several GPUs sets it on each.
enum SmemSlot { kSmemPrefill = 0, kSmemGemm = 1, kSmemLatentTc = 2, kSmemWv = 3, kSmemGemmSK = 4, kSmemRows = 5, kSmemAbsorbTc = 6, kSmemGemmSK192 = 7, kSmemSlots = 8 };
bool set_smem_limit_once(const void *kernel, int bytes, SmemSlot slot);

// bf16 TMA tensor map with 128-byte swizzle; dims/strides in elements, dim 0 contiguous.
bool make_tmap_bf16(CUtensorMap *m, const void *base, int rank, const long long *dims, const long long *strides,
                    const unsigned *box);

}  // namespace gmla

/*
 * gmla.h -- C ABI of the Gated MLA (gated multi-head latent attention) hot path
 * on NVIDIA B200 (sm_100a).
 *
 * The layer (the "Gated MLA" problem page, sections "Start from familiar
 * attention", "Split attention into heads" and "The channel-wise output
 * gate") is
 *
 *     C = X W_c^T,  Q = X W_q^T,  K = C W_k^T,  V = C W_v^T,
 *     per head h:  A_h = softmax(Q_h K_h^T / sqrt(D_h) + M),  O_h = A_h V_h,
 *     O = [O_1 | ... | O_H]                      (heads joined, not summed)
 *     Y = (sigmoid(X W_g^T) (.) O) W_o^T
 *
 * with the causal mask M[t,s] = 0 for s <= t and -inf for s > t ("Kimi K2 -
 * Construct causal mask"), the softmax taken over keys in float32 ("Kimi K3 -
 * Softmax over keys") and no positional encoding.  The latent C is the only
 * cached tensor.
 *
 * Entry points
 * ------------
 *  gmla_latent_project       projections [Q | G | C] = X [W_q; W_g; W_c]^T (C into
 *                            the cache rows) and optionally K, V of those rows
 *  gmla_latent_project_heads   the same for a range of heads (head-parallel prefill)
 *  gmla_expand_kv            K, V of any range of cached latent rows
 *  gmla_attend_prefill       causal (or full) attention over explicit Q, K, V
 *  gmla_attend_prefill_varlen  the same over a padded batch with per-sequence
 *                            query / key lengths
 *  gmla_attend_decode        one new query per sequence over the latent cache
 *  gmla_attend_decode_varlen   the same with per-sequence cache lengths
 *  gmla_attend_decode_partial  the softmax state of that query over a range of
 *                            cached rows (context-parallel decode) ...
 *  gmla_decode_combine       ... and the exact merge of such states into the output
 *  gmla_attend_decode_noalloc  gmla_attend_decode without a caller workspace
 *  gmla_gate_out             the gate and output projection Y = (sigmoid(G) (.) O) W_o^T
 *  gmla_gate_out_heads       its share for a range of heads (head-parallel prefill)
 *  gmla_get_device_status, gmla_selftest_wait_timeout, gmla_status_string,
 *  gmla_version, and a *_workspace_size query per call that needs scratch.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor is bfloat16 (gmla_bf16 holds the raw 16-bit pattern) unless
 *    stated otherwise; debug outputs are float32.
 *  - Every pointer is a DEVICE pointer on the current CUDA device, except where
 *    a comment says host.  The caller owns every buffer.  The library never
 *    allocates memory in a call; scratch comes from a caller workspace whose
 *    size the matching *_workspace_size function returns.
 *  - Inputs are never written.  The latent cache C is the one in/out buffer:
 *    gmla_latent_project writes only rows [cache_pos, cache_pos + T).
 *  - Weights use the nn.Linear orientation [out_features, in_features]:
 *    W_q, W_g, W_o [d_model, d_model]; W_c [d_c, d_model]; W_k, W_v [d_model, d_c].
 *  - Head h owns channels [h*D_h, (h+1)*D_h) of model width (D_h = d_model / H).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and return before the GPU work ends.  Only
 *    gmla_get_device_status synchronises.
 *  - Arguments are checked on the host before any launch; a bad argument
 *    returns GMLA_ERR_ARG and launches nothing.  Device pointers must be
 *    16-byte aligned and row strides multiples of 8 elements.
 *  - Supported sizes: D_h = 128 (the pages fix 96 heads of width 128), d_c a
 *    multiple of 64, d_model = 128 * H.  Other sizes return
 *    GMLA_ERR_UNSUPPORTED.
 *  - Every wait inside a kernel is bounded; a wait that runs out records
 *    GMLA_ERR_TIMEOUT in a device status word read by gmla_get_device_status.
 */
#ifndef GMLA_H
#define GMLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GMLA_API __attribute__((visibility("default")))
#else
#define GMLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GMLA_OK = 0,
    GMLA_ERR_ARG = 1,         /* invalid argument (null, shape, alignment, causal flag) */
    GMLA_ERR_UNSUPPORTED = 2, /* valid but outside the sizes this library implements */
    GMLA_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
    GMLA_ERR_TIMEOUT = 4,     /* a bounded in-kernel wait ran out (device status word) */
    GMLA_ERR_WORKSPACE = 5    /* workspace pointer null or smaller than required */
} gmla_status;

typedef uint16_t gmla_bf16; /* raw bfloat16 bits */
typedef void *gmla_stream_t; /* a cudaStream_t */

/*
 * gmla_latent_project -- the projections of the hidden states.
 * "Gated MLA" page, sections "Start from familiar attention" (C = X W_c^T,
 * K = C W_k^T, V = C W_v^T; queries come straight from the hidden states,
 * read as Q = X W_q^T) and "The channel-wise output gate" (gate logits
 * G = X W_g^T); implementation-order steps 1, 2 and the gate of step 6.
 *
 *  X       [B, T, d_model]                      hidden states (input)
 *  W_q, W_g [d_model, d_model]; W_c [d_c, d_model]; W_k, W_v [d_model, d_c]
 *  Q, G    [B, T, d_model]  outputs, may be NULL to skip (then the matching
 *                           weight may be NULL too)
 *  C       latent cache [B, cache_len_max, d_c]; row cache_pos + t of batch b
 *          receives the latent of token (b, t).  Prefill: cache_pos = 0;
 *          decode of one new token: T = 1, cache_pos = L - 1.
 *          cache_pos + T <= cache_len_max.  Required when K or V is requested.
 *  K, V    [B, T, d_model] outputs, may be NULL.  They are expanded from the
 *          bfloat16 latents just written to C.
 * d_c and the cache arguments matter only when C is given.  Needs no
 * scratch memory.
 * Returns GMLA_ERR_ARG for null required pointers, cache_pos + T >
 * cache_len_max or misalignment; GMLA_ERR_UNSUPPORTED when d_model is not a
 * multiple of 128 or d_c not a multiple of 64.
 */
GMLA_API gmla_status gmla_latent_project(const gmla_bf16 *X, int64_t B, int64_t T, int64_t d_model,
                                const gmla_bf16 *W_q, const gmla_bf16 *W_g, const gmla_bf16 *W_c,
                                int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v,
                                gmla_bf16 *Q, gmla_bf16 *G, gmla_bf16 *C, int64_t cache_len_max,
                                int64_t cache_pos, gmla_bf16 *K, gmla_bf16 *V, gmla_stream_t stream);

/*
 * gmla_latent_project_heads -- gmla_latent_project for the heads
 * [head_begin, head_end) only: the share of one GPU when the heads of a layer
 * are split over several GPUs.  Head h owns channels [128h, 128h + 128) of
 * Q, G, K and V ("Gated MLA" page, "Split attention into heads"), i.e. rows
 * 128h .. 128h+127 of W_q, W_g, W_k and W_v, so a head range needs only those
 * rows; the latent C is shared by all heads and is computed in full.
 *
 *  W_q, W_g, W_c, W_k, W_v   the FULL weights, as for gmla_latent_project
 *                            (only the rows of the range are read)
 *  Q, G, K, V  [B, T, 128 * (head_end - head_begin)] outputs for the range
 *  0 <= head_begin < head_end <= d_model / 128.  The other arguments, and the
 *  errors, are those of gmla_latent_project; the full range gives its result.
 */
GMLA_API gmla_status gmla_latent_project_heads(const gmla_bf16 *X, int64_t B, int64_t T, int64_t d_model,
                                              int64_t head_begin, int64_t head_end, const gmla_bf16 *W_q,
                                              const gmla_bf16 *W_g, const gmla_bf16 *W_c, int64_t d_c,
                                              const gmla_bf16 *W_k, const gmla_bf16 *W_v, gmla_bf16 *Q,
                                              gmla_bf16 *G, gmla_bf16 *C, int64_t cache_len_max,
                                              int64_t cache_pos, gmla_bf16 *K, gmla_bf16 *V,
                                              gmla_stream_t stream);

/*
 * gmla_expand_kv -- K = C W_k^T and V = C W_v^T for cached latent rows
 * [row0, row0 + rows) of every sequence ("Gated MLA" page, "Start from
 * familiar attention"; implementation-order step 2).  A prefill chunk that
 * continues a sequence already in the cache attends to all earlier rows too
 * (its queries sit at positions cache_pos + t, "Kimi K2 - Construct causal
 * mask" page), and the cache holds only latents, so those rows are expanded
 * again: gmla_latent_project(X_chunk, cache_pos = P) appends the chunk, then
 * gmla_expand_kv(row0 = 0, rows = P + T) gives the keys and values that
 * gmla_attend_prefill(Tq = T, Tk = P + T) needs.
 *
 *  C       latent cache [B, cache_len_max, d_c] (input)
 *  W_k, W_v [d_model, d_c]; either output may be NULL (then its weight too)
 *  K, V    [B, rows, d_model] outputs
 * Returns GMLA_ERR_ARG for null required pointers, row0 < 0, rows < 1,
 * row0 + rows > cache_len_max or misalignment; GMLA_ERR_UNSUPPORTED when
 * d_model is not a multiple of 128 or d_c not a multiple of 64.
 */
GMLA_API gmla_status gmla_expand_kv(const gmla_bf16 *C, int64_t B, int64_t cache_len_max, int64_t row0,
                                   int64_t rows, int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v,
                                   int64_t d_model, gmla_bf16 *K, gmla_bf16 *V, gmla_stream_t stream);

/*
 * gmla_attend_prefill -- per-head scaled dot-product attention over explicit
 * Q, K, V, with the causal mask and float32 softmax over keys, optionally
 * followed by the channel gate.  "Gated MLA" page, "Start from familiar
 * attention" (A = softmax(QK^T/sqrt(D_h) + M), context A V) and steps 3-5;
 * "Kimi K3 - Softmax over keys" (weights of visible keys sum to one, blocked
 * keys weigh zero, P cast to the input type before P V); "Kimi K2 - Construct
 * causal mask" (positions numbered from the cached length).
 *
 *  Q       [B, Tq, H, D_h] as addressed by q_strides; K, V [B, Tk, H, D_h].
 *          *_strides[0..2] are the element strides of batch, token and head;
 *          the D_h elements of one head are contiguous.  Both [B,T,H,D] and
 *          [B,H,T,D] layouts are expressible.
 *  Tq <= Tk: query t sits at absolute position Tk - Tq + t and, when causal,
 *          sees keys s <= Tk - Tq + t.  causal must be 0 or 1.
 *  scale   softmax scale; <= 0 selects 1/sqrt(D_h).
 *  G       optional gate logits [B, Tq, H*D_h] (contiguous); when given, O
 *          receives sigmoid(G) (.) O.
 *  O       output [B, Tq, H, D_h] as addressed by o_strides (bfloat16).
 *  lse     optional float32 [B, H, Tq]: natural log of sum_s exp(scale * q.k_s)
 *          over visible keys.
 *  weights optional float32 [B, H, Tq, Tk] debug softmax weights (before the
 *          bfloat16 cast), zero for blocked keys.  Slow; for checks only.
 */
GMLA_API gmla_status gmla_attend_prefill(const gmla_bf16 *Q, const int64_t q_strides[3],
                                const gmla_bf16 *K, const int64_t k_strides[3],
                                const gmla_bf16 *V, const int64_t v_strides[3], int64_t B, int64_t H,
                                int64_t Tq, int64_t Tk, int64_t D_h, int causal, float scale,
                                const gmla_bf16 *G, gmla_bf16 *O, const int64_t o_strides[3],
                                float *lse, float *weights, gmla_stream_t stream);

/*
 * gmla_attend_prefill_varlen -- gmla_attend_prefill over a padded batch whose
 * sequences have their own query and key counts: the two-dimensional padding
 * mask of the "Kimi K2 - Construct causal mask" page in length form, with the
 * causal mask applied per sequence at that page's positions (queries
 * continue after the sequence's past length).
 *
 *  Sequence b has q_lens[b] query rows (rows 0..q_lens[b]-1 of Q) and
 *  kv_lens[b] keys (rows 0..kv_lens[b]-1 of K and V); its query t sits at
 *  position kv_lens[b] - q_lens[b] + t.  Rows past a length are never read as
 *  data (they may hold anything, NaN included) and output rows t >= q_lens[b]
 *  of O and lse are left untouched.
 *  q_lens, kv_lens  HOST arrays of B lengths, 0 <= q_lens[b] <= kv_lens[b],
 *          q_lens[b] <= Tq_max, 1 <= kv_lens[b] <= Tk_max; read during the
 *          call only.
 *  Q, O    [B, Tq_max, H, D_h]; K, V [B, Tk_max, H, D_h]; G [B, Tq_max, H*D_h];
 *          lse [B, H, Tq_max] -- as for gmla_attend_prefill (strides in
 *          elements, last dimension contiguous).  No debug weights.
 *  workspace >= gmla_attend_prefill_varlen_workspace_size(B) bytes, 16-byte
 *          aligned; it receives three tensor maps and two lengths per
 *          sequence, copied from the host on `stream` before the launch.
 * Errors: GMLA_ERR_ARG for null pointers, lengths outside those bounds, bad
 * strides or alignment; GMLA_ERR_UNSUPPORTED for D_h != 128;
 * GMLA_ERR_WORKSPACE for a short workspace.
 */
GMLA_API gmla_status gmla_attend_prefill_varlen(const gmla_bf16 *Q, const int64_t q_strides[3],
                                               const gmla_bf16 *K, const int64_t k_strides[3],
                                               const gmla_bf16 *V, const int64_t v_strides[3], int64_t B,
                                               int64_t H, int64_t Tq_max, int64_t Tk_max, int64_t D_h,
                                               const int64_t *q_lens, const int64_t *kv_lens, int causal,
                                               float scale, const gmla_bf16 *G, gmla_bf16 *O,
                                               const int64_t o_strides[3], float *lse, void *workspace,
                                               size_t workspace_bytes, gmla_stream_t stream);
GMLA_API size_t gmla_attend_prefill_varlen_workspace_size(int64_t B);

/*
 * gmla_attend_decode -- one new query per sequence over the latent cache.
 * Same mathematics as gmla_attend_prefill with Tq = 1 over K = C W_k^T and
 * V = C W_v^T ("Gated MLA" page, "Start from familiar attention"), evaluated
 * without rebuilding K or V: by associativity q_h . (W_k^(h) c_s) =
 * (W_k^(h)T q_h) . c_s and sum_s a_s W_v^(h) c_s = W_v^(h) sum_s a_s c_s, so
 * the kernel streams only the d_c-wide latents, each read once for all heads.
 * The key range is split over thread blocks and the partial softmax states are
 * merged exactly (log-sum-exp).
 *
 *  Q       [B, H*D_h] queries of the new tokens (from gmla_latent_project, T=1)
 *  C       latent cache [B, cache_len_max, d_c]; rows 0..L-1 are visible (the
 *          new token's own latent at row L-1 included), 1 <= L <= cache_len_max.
 *  W_k, W_v [H*D_h, d_c]
 *  scale   <= 0 selects 1/sqrt(D_h)
 *  G       optional gate logits [B, H*D_h]; when given, O = sigmoid(G) (.) O
 *  O       output [B, H*D_h]
 *  weights optional float32 [B, H, L] debug softmax weights
 *  workspace >= gmla_attend_decode_workspace_size(B, L, H, d_c) bytes
 */
GMLA_API gmla_status gmla_attend_decode(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B,
                               int64_t cache_len_max, int64_t L, int64_t H, int64_t D_h, int64_t d_c,
                               const gmla_bf16 *W_k, const gmla_bf16 *W_v, float scale,
                               const gmla_bf16 *G, gmla_bf16 *O, float *weights, void *workspace,
                               size_t workspace_bytes, gmla_stream_t stream);
GMLA_API size_t gmla_attend_decode_workspace_size(int64_t B, int64_t L, int64_t H, int64_t d_c);

/*
 * gmla_attend_decode_varlen -- gmla_attend_decode over a batch whose sequences
 * hold different numbers of cached latents: the two-dimensional padding mask
 * of the "Kimi K2 - Construct causal mask" page (positions past a sequence's
 * length are padding, combined with the causal mask) in its length form.
 * Sequence b attends to
 * rows 0..lens[b]-1 of its cache, its new latent at row lens[b]-1 (the query
 * position is the cached length: that page's position ids start at the past
 * length).  Rows at or past lens[b] are never read as data: they may hold
 * anything, NaN included.
 *
 *  lens    HOST array of B lengths, 1 <= lens[b] <= cache_len_max; read
 *          during the call only.  The other arguments are those of
 *          gmla_attend_decode.
 *  weights optional float32 [B, H, cache_len_max]; columns at or past lens[b]
 *          are written as 0.
 *  workspace >= gmla_attend_decode_varlen_workspace_size(B, cache_len_max,
 *          H, d_c) bytes, 16-byte aligned; it also receives one tensor map,
 *          one length and one record offset per sequence and the list of work
 *          items (copied from the host on `stream` before the launches; the
 *          call places them on 256-byte boundaries inside the workspace, which
 *          the reported size allows for).  The rows of every sequence are cut
 *          into work items of at most kps keys, kps chosen from `lens` on the
 *          host, so that the thread blocks of one launch stream about equally
 *          many latents whatever the length mix; the size depends only on
 *          (B, cache_len_max, H, d_c).
 * Errors: GMLA_ERR_ARG for a null pointer or a length outside 1..cache_len_max,
 * the rest as gmla_attend_decode.
 */
GMLA_API gmla_status gmla_attend_decode_varlen(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B,
                                              int64_t cache_len_max, const int64_t *lens, int64_t H,
                                              int64_t D_h, int64_t d_c, const gmla_bf16 *W_k,
                                              const gmla_bf16 *W_v, float scale, const gmla_bf16 *G,
                                              gmla_bf16 *O, float *weights, void *workspace,
                                              size_t workspace_bytes, gmla_stream_t stream);
GMLA_API size_t gmla_attend_decode_varlen_workspace_size(int64_t B, int64_t cache_len_max, int64_t H,
                                                         int64_t d_c);

/*
 * gmla_attend_decode_partial -- the softmax state of one new query per
 * sequence over the cached latent rows [k0, k1) only.  Softmax over keys
 * ("Kimi K3 - Softmax over keys") restricted to a key subset, with its
 * log-sum-exp, so that states of disjoint subsets merge exactly
 * (gmla_decode_combine): the share of one GPU when the latent cache of a
 * long context is split over several GPUs along its length (the
 * "Le Transformer et l'attention" page's cost table: at 1M tokens the cache
 * is 128 times that of 8K).  Same absorbed evaluation as gmla_attend_decode.
 *
 *  Q, C, B, cache_len_max, H, D_h, d_c, W_k, scale: as gmla_attend_decode.
 *  0 <= k0 <= k1 <= cache_len_max; rows [k0, k1) of every sequence are read
 *          (the query's own latent belongs to whichever range holds row L-1).
 *  lse     float32 [B, H] output: natural log of sum_{s in [k0,k1)} exp(scale q_h.k_s)
 *  ctx     float32 [B, H, d_c] output: sum_{s in [k0,k1)} a_s c_s, with a_s the
 *          softmax weights normalised over [k0, k1) and c_s the latent rows
 *          (so the head context over the range is W_v^(h) ctx[b,h,:]).
 *          k0 == k1 gives lse = -inf and ctx = 0: an empty range.
 *  workspace >= gmla_attend_decode_partial_workspace_size(B, k0, k1, H, d_c)
 *          bytes (0 when k0 == k1; the pointer may then be NULL).
 * Errors as gmla_attend_decode; GMLA_ERR_ARG also for a bad range.
 */
GMLA_API gmla_status gmla_attend_decode_partial(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B,
                                               int64_t cache_len_max, int64_t k0, int64_t k1, int64_t H,
                                               int64_t D_h, int64_t d_c, const gmla_bf16 *W_k, float scale,
                                               float *lse, float *ctx, void *workspace, size_t workspace_bytes,
                                               gmla_stream_t stream);
GMLA_API size_t gmla_attend_decode_partial_workspace_size(int64_t B, int64_t k0, int64_t k1, int64_t H,
                                                          int64_t d_c);

/*
 * gmla_decode_combine -- merge n_parts decode states of disjoint key ranges
 * (gmla_attend_decode_partial) into the decode output: with m = max_i lse_i,
 * w_i = exp(lse_i - m) / sum_j exp(lse_j - m), c^ = sum_i w_i ctx_i (the
 * softmax over the union of the ranges, exact in real arithmetic), then
 * o_h = W_v^(h) c^_h and, when G is given, the gate sigmoid(G) (.) o
 * ("Gated MLA" page, "The channel-wise output gate").
 *
 *  lse     float32 [n_parts, B, H]; ctx float32 [n_parts, B, H, d_c]: the
 *          states stacked along a leading axis (what an all-gather of the
 *          per-GPU states produces); states with lse = -inf are skipped, and a
 *          sequence whose states are all empty gets O = 0.
 *  W_v     [H*D_h, d_c]; G optional gate logits [B, H*D_h]; O [B, H*D_h] output.
 *  1 <= n_parts <= 1024.  Needs no scratch memory.
 */
GMLA_API gmla_status gmla_decode_combine(const float *lse, const float *ctx, int64_t n_parts, int64_t B,
                                        int64_t H, int64_t D_h, int64_t d_c, const gmla_bf16 *W_v,
                                        const gmla_bf16 *G, gmla_bf16 *O, gmla_stream_t stream);

/*
 * gmla_attend_decode_noalloc -- gmla_attend_decode for callers that cannot
 * allocate device memory.  No page has a counterpart: it is a service of this
 * library, not a step of the method.
 *
 * Some callers cannot hand over a workspace: a serving runtime that reserved
 * all device memory for its own pool up front, or host code running where the
 * CUDA allocator must not be called (the allocator can synchronise the device
 * or wait on a lock the caller holds).  This entry point takes the same
 * arguments as gmla_attend_decode minus the workspace and computes the same
 * result (the key range may be split into fewer pieces, so float32 rounding
 * may differ slightly).  Its scratch (q~, the per-split softmax states and the
 * log-sum-exp) lives in one fixed device array of
 * gmla_attend_decode_noalloc_max_bytes() bytes (32 MiB) inside the library,
 * which every GPU that loads the library holds until the process exits.
 *
 *  - Allocates nothing and calls no allocating routine.
 *  - Problems whose scratch does not fit even with a single key split
 *    (about B*H*d_c*6 bytes > 32 MiB, e.g. B > 113 at H = 96, d_c = 512) return
 *    GMLA_ERR_WORKSPACE before any launch.
 *  - Every call shares the array and leaves its contents behind; each call
 *    rewrites all the scratch it reads, so nothing needs clearing.  Calls whose
 *    GPU work overlaps (different streams, or unordered host threads) race on
 *    the array: order them on one stream.
 *  - The array's device address is looked up once per device, with that
 *    device current, by the first call of ANY entry point of this library on
 *    that device (gmla_get_device_status included); that lookup loads the
 *    library's device code there and commits the 32 MiB.  A caller that
 *    reserves all free device memory for its own pool should therefore make
 *    one call (gmla_get_device_status suffices) before reserving it.
 */
GMLA_API gmla_status gmla_attend_decode_noalloc(const gmla_bf16 *Q, const gmla_bf16 *C, int64_t B,
                                               int64_t cache_len_max, int64_t L, int64_t H, int64_t D_h,
                                               int64_t d_c, const gmla_bf16 *W_k, const gmla_bf16 *W_v,
                                               float scale, const gmla_bf16 *G, gmla_bf16 *O, float *weights,
                                               gmla_stream_t stream);
GMLA_API size_t gmla_attend_decode_noalloc_max_bytes(void);

/*
 * gmla_gate_out -- the gate and the output projection over M = B*T rows:
 * Y = (sigmoid(G) (.) O) W_o^T ("Gated MLA" page, "The channel-wise output
 * gate": the gate acts channel by channel, before W_o; step 6).  The
 * attention calls already fuse the gate (gmla_attend_prefill and
 * gmla_attend_decode take G), so the usual call passes their gated output
 * with G = NULL; a caller holding an ungated context passes its gate logits.
 *
 *  O [M, d_model] context; G [M, d_model] gate logits or NULL;
 *  W_o [d_model, d_model]; Y [M, d_model] output.
 *  workspace: with G != NULL, >= gmla_gate_out_workspace_size(M, d_model)
 *          bytes, 16-byte aligned; it receives the gated context (bfloat16)
 *          that the projection then reads.  With G == NULL it is not used
 *          and may be NULL.
 * Errors: GMLA_ERR_ARG for null or misaligned pointers; GMLA_ERR_UNSUPPORTED
 * when d_model is not a multiple of 128; GMLA_ERR_WORKSPACE for a missing or
 * short workspace when G is given.
 */
GMLA_API gmla_status gmla_gate_out(const gmla_bf16 *O, const gmla_bf16 *G, const gmla_bf16 *W_o, int64_t M,
                          int64_t d_model, gmla_bf16 *Y, void *workspace, size_t workspace_bytes,
                          gmla_stream_t stream);
GMLA_API size_t gmla_gate_out_workspace_size(int64_t M, int64_t d_model);

/*
 * gmla_gate_out_heads -- the share of the heads [head_begin, head_end) in
 * gmla_gate_out: Y_part = (sigmoid(G) (.) O) W_o[:, c]^T with c the channels
 * 128*head_begin .. 128*head_end - 1.  The output projection mixes all
 * channels, so Y is the sum of the shares of any partition of the heads
 * (each GPU of a head-parallel layer computes its share; a reduction over
 * the GPUs gives Y).
 *
 *  O, G    [M, 128 * (head_end - head_begin)]: the context and gate logits of
 *          the range (G may be NULL)
 *  W_o     the FULL [d_model, d_model] weight (only the range's columns are read)
 *  Y       [M, d_model] output: this range's share
 *  workspace: with G != NULL, >= gmla_gate_out_workspace_size(M,
 *          128 * (head_end - head_begin)) bytes.
 *  0 <= head_begin < head_end <= d_model / 128; errors as gmla_gate_out.
 */
GMLA_API gmla_status gmla_gate_out_heads(const gmla_bf16 *O, const gmla_bf16 *G, const gmla_bf16 *W_o, int64_t M,
                                        int64_t d_model, int64_t head_begin, int64_t head_end, gmla_bf16 *Y,
                                        void *workspace, size_t workspace_bytes, gmla_stream_t stream);

/* Synchronise `stream`, then read and clear this device's status word.
 * Returns GMLA_OK, GMLA_ERR_TIMEOUT (a bounded wait ran out) or GMLA_ERR_CUDA. */
GMLA_API gmla_status gmla_get_device_status(gmla_stream_t stream);

/* Self-test of the bounded-wait machinery (no counterpart on the pages): launches
 * one thread that waits `milliseconds` (1..1000) on an mbarrier nothing arrives
 * at; the wait runs out, records GMLA_ERR_TIMEOUT in the status word and the
 * kernel returns.  A following gmla_get_device_status returns GMLA_ERR_TIMEOUT
 * (and clears it); the CUDA context stays usable. */
GMLA_API gmla_status gmla_selftest_wait_timeout(unsigned milliseconds, gmla_stream_t stream);

/* Static, NUL-terminated description of a status code (host memory, never freed). */
GMLA_API const char *gmla_status_string(gmla_status s);

/* Library version as major*10000 + minor*100 + patch. */
GMLA_API int gmla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GMLA_H */

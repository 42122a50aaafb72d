/*
 * hstu.h — C ABI of libhstu.so: the forward pass of an HSTU layer stack over
 * jagged (unpadded) user sequences, and M-FALCON candidate ranking, on one
 * NVIDIA B200 (sm_100a).
 *
 * Source of the operations: the page 'HSTUとGenerative Recommenders――行動履歴から
 * 1.5兆parameterの推薦モデルへ' (koktn.github.io, an explainer of Zhai et al.,
 * "Actions Speak Louder than Words", ICML 2024):
 *   - section 'HSTUはTransformerと何が違うのか', subsections
 *     '1. U、V、Q、Kは同じ入力を見る4つの役割' (f1 + SiLU, split U,V,Q,K),
 *     '2. QKᵀで「どの履歴を見るか」を決める' (score = Q_i.K_j + position bias +
 *     time bias, causal, pointwise SiLU weights without softmax),
 *     '3. Uでcontextをgateし、次のlayerへ渡す' (LayerNorm(context) * U, f2,
 *     residual connection);
 *   - section '長い履歴を現実の計算量へ収める4つの工夫', subsections
 *     '1. 長さの異なるsequenceをpaddingせず処理する' (ragged batches without
 *     padding) and '4. M-FALCONで候補間の履歴計算を共有する' (candidates in
 *     microbatches appended after the history, mask and relative bias
 *     adjusted, history K/V cache shared across microbatches).
 *
 * Per user b (rows i, j of that user, n_b rows) one layer computes
 *   G = SiLU(X W1^T + b1) = [U | V | Q | K]   (head-major inside each part)
 *   s_ij = Q_i.K_j + rab_pos[h][pb(i-j)] + rab_time[h][tb(max(0, t_i - t_j))],  j <= i
 *   O_i  = (1/n_b) sum_{j<=i} SiLU(s_ij) V_j
 *   Y_i  = X_i + (LayerNorm(O_i) * U_i) W2^T + b2
 * where pb/tb are log-linear buckets: x < 2^S -> x; otherwise, with
 * e = floor(log2 x), (e-S+1)*2^S + (x >> (e-S)) - 2^S; clamped to N-1.
 * LayerNorm runs over all h*d_v features of a row (biased variance, eps from
 * the descriptor), then gamma, beta.
 *
 * Conventions for every entry point
 *   Ownership   The caller owns every buffer.  The library never allocates,
 *               frees or synchronises device memory, except that
 *               hstu_read_status synchronises the given stream.
 *   Execution   Asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *               default stream).  Returning HSTU_OK means the work was
 *               enqueued; device-detected errors are read with hstu_read_status.
 *   Layout      Row-major.  Activations [rows, d_model]; weights in [out, in]
 *               layout: W1 [F, d_model] with F = 2*h*d_v + 2*h*d_qk in the
 *               column order U, V, Q, K; W2 [d_model, h*d_v]; b1 [F]; b2
 *               [d_model]; ln_gamma, ln_beta [h*d_v]; rab_pos [h, n_pos_buckets]
 *               and rab_time [h, n_time_buckets] always fp32.  Element type of
 *               everything else is the descriptor's dtype (bf16 or fp32).
 *               Every device pointer must be 16-byte aligned.  Inputs and
 *               outputs must not alias each other or the workspace.
 *   Offsets     int64 [B+1], offsets[0] = 0, non-decreasing, offsets[B] =
 *               total rows; every length <= max_len.
 *   Timestamps  int64 seconds, one per row; within one user every timestamp
 *               must lie within 2^30 s of that user's first one.
 *   Errors      Host-detectable argument errors return at once and enqueue
 *               nothing.  Device-detected errors (bad offsets or timestamps,
 *               a wait that timed out) set a status word in the workspace; the
 *               remaining kernels of the call then exit early.  No entry
 *               point traps or asserts on the device.
 *   Precision   dtype HSTU_BF16 (inputs, weights, outputs bf16): the tensor
 *               cores take fp16 operands with fp32 accumulation.  bf16 values
 *               within [2^-14, 65504] in magnitude convert to fp16 exactly;
 *               the f1 output, P, Z and the residual stream between layers
 *               are stored in fp16 (saturating at +-65504), the attention
 *               output O and the LayerNorm statistics stay fp32 (M-FALCON's
 *               candidate rows also keep an fp32 residual), and only the final
 *               output is rounded to bf16.  fp16 keeps 3 more mantissa bits than
 *               bf16 at the same tensor-core rate; inputs, weights and layer
 *               outputs must lie within fp16 range (|x| <= 65504).  Weights
 *               below 2^-14 in magnitude become fp16 subnormals (absolute
 *               error up to 2^-25 each): against activations of order one
 *               they stay within the bf16 bound (tested: W2 drawn from
 *               N(0, 1e-5)); against activations in the thousands the error
 *               they add grows with the activations and can exceed it (Q and
 *               K rows of W1 near 1e-5 against activations of 8192 gave
 *               2.3e-2).  dtype HSTU_FP32: fp32 throughout (CUDA-core FMA).
 *   Supported   bf16: d_qk = d_v in {64, 128}; d_model and h*d_v multiples
 *               of 64; bucket counts in [1, 4096].  fp32: d_qk, d_v <= 128
 *               and multiples of 4; d_model multiple of 4.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,   /* host: null/misaligned pointer, bad size */
  HSTU_ERR_UNSUPPORTED = 2,   /* host: a shape or dtype the library does not run */
  HSTU_ERR_WORKSPACE = 3,     /* host: workspace smaller than hstu_workspace_size */
  HSTU_ERR_CUDA = 4,          /* host: a CUDA runtime call failed */
  HSTU_ERR_BAD_OFFSETS = 5,   /* device: offsets not monotone, wrong total, length > max */
  HSTU_ERR_TIMEOUT = 6,       /* device: an in-kernel wait gave up */
  HSTU_ERR_BAD_TIMESTAMPS = 7, /* device: a user's timestamps span 2^30 s or more */
  HSTU_ERR_BAD_IDS = 8         /* device: a token id outside its embedding table */
} hstu_status;

typedef enum { HSTU_BF16 = 0, HSTU_FP32 = 1 } hstu_dtype;

/* Shape of one layer (all layers of a stack share it). */
typedef struct {
  int32_t d_model;         /* d */
  int32_t n_heads;         /* h */
  int32_t d_qk;            /* per-head query/key width */
  int32_t d_v;             /* per-head value/gate width */
  int32_t n_pos_buckets;   /* N_p: entries per head in rab_pos */
  int32_t n_time_buckets;  /* N_t: entries per head in rab_time */
  int32_t pos_sub_bits;    /* S_p of the position buckets, 0..20 */
  int32_t time_sub_bits;   /* S_t of the time-gap buckets, 0..20 */
  float ln_eps;            /* LayerNorm epsilon */
  int32_t dtype;           /* hstu_dtype of activations and dense weights */
} hstu_layer_desc;

/* Device pointers to one layer's parameters (layout above). */
typedef struct {
  const void* W1;
  const void* b1;
  const void* W2;
  const void* b2;
  const void* ln_gamma;
  const void* ln_beta;
  const float* rab_pos;
  const float* rab_time;
  /* Optional, bf16 layers only: fp16 copies of W1 and W2 (same layout),
   * e.g. made once with hstu_bf16_to_f16.  The tensor-core path multiplies
   * the fp16 residual stream and the fp16 gated Z by fp16 weights; when these
   * are null every call converts W1 (layers >= 1) and W2 into its workspace
   * first.  Must be 16-byte aligned when set; ignored for fp32 layers. */
  const void* W1_f16;
  const void* W2_f16;
} hstu_layer_weights;

/* Bytes of device workspace an entry point needs for these sizes.
 * For hstu_layer_fwd / hstu_stack_fwd pass total_cands = max_cands = 0 and
 * microbatch = 0.  Returns 0 if the arguments are invalid. */
size_t hstu_workspace_size(const hstu_layer_desc* desc, int32_t n_layers, int64_t B,
                           int64_t total_tokens, int64_t max_len, int64_t total_cands,
                           int64_t max_cands, int32_t microbatch);

/* One HSTU layer.  offsets: device int64 [B+1]; X: device [T, d]; weights:
 * host struct of device pointers; timestamps: device int64 [T]; out: device
 * [T, d] (must not alias X). */
hstu_status hstu_layer_fwd(const hstu_layer_desc* desc, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const hstu_layer_weights* weights, const int64_t* timestamps,
                           void* out, void* workspace, size_t workspace_bytes, void* stream);

/* n_layers layers, each layer's output the next one's input (section '3. U
 * でcontextをgateし、次のlayerへ渡す').  weights: host array [n_layers].  The
 * offsets are validated once and the tile schedule is shared by all layers. */
hstu_status hstu_stack_fwd(const hstu_layer_desc* desc, int32_t n_layers,
                           const hstu_layer_weights* weights, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const int64_t* timestamps, void* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* M-FALCON ranking (section '4. M-FALCONで候補間の履歴計算を共有する').
 * The histories run through n_layers layers once, keeping every layer's K/V;
 * then candidates, in microbatches of `microbatch` per user, run through the
 * layers attending to their user's whole history and to themselves only.
 * Every candidate sits at position n_b (distance n_b - j to history row j)
 * and at time request_ts[b] (NULL: the user's last history timestamp); its
 * normaliser is max(n_b, 1).  scores[c] = <y_c, head_vec> in fp32, where y_c
 * is candidate c's output of the last layer.
 * hist_offsets [B+1], history [T_hist, d], hist_timestamps [T_hist],
 * cand_offsets [B+1] (device), candidates [C, d], head_vec [d], scores fp32
 * [C].  Every user has at most max_cands candidates. */
hstu_status hstu_mfalcon_rank(const hstu_layer_desc* desc, int32_t n_layers,
                              const hstu_layer_weights* weights, int64_t B, int64_t total_hist,
                              int64_t max_len, const int64_t* hist_offsets, const void* history,
                              const int64_t* hist_timestamps, int64_t total_cands,
                              int64_t max_cands, const int64_t* cand_offsets,
                              const void* candidates, const int64_t* request_ts,
                              int32_t microbatch, const void* head_vec, float* scores,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch used by hstu_layer_fwd_noalloc. */
#define HSTU_NOALLOC_SCRATCH_BYTES (64u << 20)

/* hstu_layer_fwd without a workspace argument, for callers that cannot
 * allocate device memory (an allocator owned by another runtime, no
 * cudaMalloc allowed after start-up, a memory-capped sandbox).  It has no
 * counterpart on the pages: it is the same layer as hstu_layer_fwd, run in a
 * file-scope device array of HSTU_NOALLOC_SCRATCH_BYTES (64 MiB) that every
 * device loading this library holds until the process exits.  It allocates
 * nothing itself: no cudaMalloc, no cudaFree, no allocating library call.
 * The caller still passes the inputs and the output (as for hstu_layer_fwd).
 *   - Sizes whose workspace (hstu_workspace_size with n_layers = 1) exceeds
 *     HSTU_NOALLOC_SCRATCH_BYTES return HSTU_ERR_WORKSPACE and launch nothing;
 *     other argument errors are those of hstu_layer_fwd.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after a cudaDeviceReset (which releases the module's device
 *     memory) it is stale, so the function must not be called again in that
 *     process.
 *   - Every call shares the one array and leaves its contents behind; each
 *     call resets what must start at zero (the status word and counters).
 *     Calls whose execution overlaps on the GPU (other streams, other host
 *     threads) race on the array: serialise them.
 *   - The device status word lives in the array, so hstu_read_status cannot
 *     read it; check the output or use hstu_layer_fwd to diagnose. */
hstu_status hstu_layer_fwd_noalloc(const hstu_layer_desc* desc, int64_t B, int64_t total_tokens,
                                   int64_t max_len, const int64_t* offsets, const void* X,
                                   const hstu_layer_weights* weights, const int64_t* timestamps,
                                   void* out, void* stream);

/* Backward pass (gradients, for training) of hstu_layer_fwd / hstu_stack_fwd
 * ('HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか': the
 * forward layer whose chain rule this is; section 'Production評価の12.4%をどう
 * 読むか': training is where the pages report the largest gain).  Given the
 * layers' input X and the gradient dY of a loss with respect to the stack's
 * output, computes dX (the gradient with respect to X) and, per layer, the
 * gradients of every parameter.  The call runs the stack's forward itself
 * first, keeping each layer's input, f1 output and pre-activation and
 * attention output in the workspace (about 2 T (d + 2F + h d_v) bytes per
 * layer), so nothing of an earlier forward call has to be kept.
 * Derivatives, per user (n = n_b) and head, written out by the chain rule:
 *   dZ = dY W2;  dW2 = dY^T Z;  db2 = sum_rows dY
 *   dL = dZ * U; dU = dZ * L (L = LayerNorm(O) before the gate); dgamma =
 *   sum_rows dL * xhat; dbeta = sum_rows dL; dO = (dxh - mean(dxh) - xhat
 *   mean(dxh xhat)) / sd with dxh = dL * gamma
 *   dA_ij = (1/n) dO_i . V_j; dV_j = (1/n) sum_i SiLU(s_ij) dO_i;
 *   dS_ij = dA_ij SiLU'(s_ij); dQ_i = sum_j dS_ij K_j; dK_j = sum_i dS_ij Q_i;
 *   drab_pos[h][b] / drab_time[h][b] = sum of dS_ij over the pairs (i, j) of
 *   bucket b
 *   dP = [dU | dV | dQ | dK] * SiLU'(P), P = X W1^T + b1;  dW1 = dP^T X;
 *   db1 = sum_rows dP;  dX = dY + dP W1.
 * dtype HSTU_BF16 only (HSTU_ERR_UNSUPPORTED otherwise), with the forward's
 * shape limits and n_time_buckets <= 256.  X and dY are bf16 [T, d] (device);
 * dX is bf16 [T, d]; every gradient is fp32, in its parameter's layout, and
 * is overwritten (not accumulated into).  The tensor cores take fp16
 * operands with fp32 accumulation (as in the forward; the gradients flowing
 * into them must lie within fp16 range); the gradient stream between layers
 * is fp32.  Every result is deterministic: the bias-table gradients are summed
 * in 64-bit fixed point (units of 2^-32, each partial sum clamped to
 * +-2^30), whose additions do not depend on their order, then rounded to fp32.
 * grads: host array [n_layers] of device pointers.  Workspace:
 * hstu_bwd_workspace_size() bytes, 256-byte aligned.  Asynchronous on
 * `stream`; device-detected errors (bad offsets or timestamps, a wait that
 * gave up) set the workspace's status word (hstu_read_status). */
typedef struct {
  float* dW1;        /* [F, d_model] */
  float* db1;        /* [F] */
  float* dW2;        /* [d_model, h*d_v] */
  float* db2;        /* [d_model] */
  float* dln_gamma;  /* [h*d_v] */
  float* dln_beta;   /* [h*d_v] */
  float* drab_pos;   /* [h, n_pos_buckets] */
  float* drab_time;  /* [h, n_time_buckets] */
} hstu_layer_grads;
size_t hstu_bwd_workspace_size(const hstu_layer_desc* desc, int32_t n_layers, int64_t B,
                               int64_t total_tokens, int64_t max_len);
hstu_status hstu_layer_bwd(const hstu_layer_desc* desc, const hstu_layer_weights* weights,
                           int64_t B, int64_t total_tokens, int64_t max_len,
                           const int64_t* offsets, const void* X, const int64_t* timestamps,
                           const void* dY, void* dX, const hstu_layer_grads* grads,
                           void* workspace, size_t workspace_bytes, void* stream);
hstu_status hstu_stack_bwd(const hstu_layer_desc* desc, int32_t n_layers,
                           const hstu_layer_weights* weights, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const int64_t* timestamps, const void* dY, void* dX,
                           const hstu_layer_grads* grads, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Stochastic Length sampling and token embedding ('HSTUとGenerative
 * Recommenders', section '2. Stochastic Lengthで学習時の履歴を間引く': a long
 * history is shortened to a random subset of its positions; 4096 tokens keep
 * 776).  For each user b with a raw sequence of n_b tokens, keeps
 * k_b = min(n_b, floor(n_b^0.8)) (at least 1) positions: those whose keys are
 * smallest, the key of position p being output number b * 2^32 + p + 1 of the
 * SplitMix64 generator started from state `seed`, ties by position; the kept
 * tokens stay in their original order.  A kept token at an even original
 * position is a content item (row raw_ids[.] of content_table), at an odd
 * position an action (row of action_table).
 *   raw_offsets     device int64 [B+1], raw_offsets[0] = 0, [B] = raw_total,
 *                   each length at most max_raw_len (<= 32767)
 *   raw_ids         device int64 [raw_total] (row indices into the tables)
 *   raw_timestamps  device int64 [raw_total]
 *   content_table   device bf16 [n_content, d_model], 16-byte aligned
 *   action_table    device bf16 [n_action, d_model], 16-byte aligned
 *   out_offsets     device int64 [B+1]: the kept sequences' offsets
 *   out_X           device bf16 [sum k_b, d_model] (at most raw_total rows)
 *   out_timestamps  device int64 [sum k_b]
 *   workspace       hstu_sl_embed_workspace_size() bytes, 256-byte aligned
 *                   (holds the device status word)
 * d_model must be a multiple of 8.  Host-detectable errors return at once;
 * bad offsets or an id outside its table set the status word
 * (HSTU_ERR_BAD_OFFSETS: all out_offsets are 0; HSTU_ERR_BAD_IDS: that row is
 * zero), read back with hstu_read_status.  Asynchronous on `stream`. */
size_t hstu_sl_embed_workspace_size(void);
/* Full-catalog retrieval ('NetflixのGenRec解説――LLMを生成させず推薦rankerとして使う',
 * section '全体像：LLMは入力を読み、ranking headが作品を採点する'; the GenRec
 * explainer on techistory.net, s = E^T h): every one of n_items catalog
 * items is scored against every user vector, s[u, m] = <E_m, h_u>, in fp32
 * on the tensor cores, and the K highest scores per user are returned in
 * descending order, equal scores ordered by ascending item id.
 *   H             device bf16: the user vectors [n_users, d], or, when
 *                 user_offsets is given, the encoder output [total_rows, d]
 *                 whose row user_offsets[u+1]-1 is user u's vector (a user
 *                 without rows scores every item 0)
 *   user_offsets  device int64 [n_users+1] or null
 *   E             device bf16 [n_items, d] item embeddings
 *   out_scores    device fp32 [n_users, K]; out_ids device int64 [n_users, K]
 *   workspace     hstu_retrieval_workspace_size(...) bytes, 256-byte aligned
 *                 (from_rows = 1 when user_offsets will be given); it holds
 *                 the status word and the [n_users, n_items] score matrix
 * Requires d % 64 == 0, 1 <= K <= min(n_items, 1024), n_users <= 65535,
 * n_items < 2^31 - 256, H and E 16-byte aligned.  Offsets that are not
 * monotone or pass total_rows set HSTU_ERR_BAD_OFFSETS in the status word
 * (outputs then unspecified).  Asynchronous on `stream`. */
size_t hstu_retrieval_workspace_size(int64_t n_users, int64_t n_items, int32_t d, int32_t K,
                                     int32_t from_rows);
hstu_status hstu_retrieval_topk(int64_t n_users, int64_t n_items, int32_t d, const void* H,
                                const int64_t* user_offsets, int64_t total_rows, const void* E,
                                int32_t K, float* out_scores, int64_t* out_ids, void* workspace,
                                size_t workspace_bytes, void* stream);
/* Catalogs of 65,536 items or more are first scored on a 1-in-16 strided
 * sample to find a per-user score threshold, and the full pass keeps only
 * the items at or above it (the score matrix is never written); a user left
 * with fewer than K such items (or too many) makes the call fall back to
 * scoring and selecting over every item, with the same result.  After a call
 * (and a synchronisation of `stream`), *taken = 1 if that fallback ran. */
hstu_status hstu_retrieval_fallback_taken(const void* workspace, size_t workspace_bytes,
                                          int32_t* taken, void* stream);

/* Softmax-Transformer encoder layer: the comparator of the HSTU layer on the
 * same jagged batches ('HSTUとGenerative Recommenders', section 'Production評価の
 * 12.4%をどう読むか': HSTU against a FlashAttention-2 Transformer at 8,192
 * tokens, d = 512, 8 heads; attention as in the GenRec explainer on
 * techistory.net, softmax(QK^T / sqrt(d_k)) V).  Pre-LayerNorm, causal per
 * user:  A = LN1(X); [Q|K|V] = A W_qkv^T; ctx = per-head causal softmax
 * attention; X1 = X + ctx W_o^T; Y = X1 + SiLU(LN2(X1) W_1^T + b_1) W_2^T + b_2.
 * Dense weights are fp16 ([out, in] row-major: W_qkv [3d, d] with Q, K, V
 * row blocks, W_o [d, d], W_1 [d_ff, d], W_2 [d, d_ff]); LayerNorm gamma/beta
 * and the biases are bf16.  X and out are bf16 [T, d]; intermediates fp16.
 * Requires d % 256 == 0, d <= 1024, head dim d/h of 64 or 128, d_ff % 256 == 0;
 * every pointer 16-byte aligned.  Offsets are checked on the device
 * (HSTU_ERR_BAD_OFFSETS in the status word). */
typedef struct {
  const void* ln1_gamma;
  const void* ln1_beta;
  const void* W_qkv;
  const void* W_o;
  const void* ln2_gamma;
  const void* ln2_beta;
  const void* W_1;
  const void* b_1;
  const void* W_2;
  const void* b_2;
} hstu_transformer_weights;
size_t hstu_transformer_workspace_size(int32_t d_model, int32_t n_heads, int32_t d_ff, int64_t B,
                                       int64_t total_tokens);
hstu_status hstu_transformer_layer_fwd(int32_t d_model, int32_t n_heads, int32_t d_ff,
                                       float ln_eps, const hstu_transformer_weights* weights,
                                       int64_t B, int64_t total_tokens, int64_t max_len,
                                       const int64_t* offsets, const void* X, void* out,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* Round-to-nearest conversion of n bf16 values to fp16 (device to device,
 * asynchronous on `stream`), for the optional W1_f16 / W2_f16 weight copies.
 * n must be a multiple of 8 and both pointers 16-byte aligned. */
hstu_status hstu_bf16_to_f16(const void* src, void* dst, int64_t n, void* stream);

/* The keep count k(n) = min(n, floor(n^0.8)) (at least 1 for n >= 1) that
 * hstu_sl_embed applies to a raw stream of n tokens, computed on the host
 * with the same integer definition (the largest k with k^5 <= n^4), so a
 * caller can size the kept batch (sum and max of k) without reading the
 * device.  Returns -1 for n < 0 or n > 32767. */
int64_t hstu_sl_keep_count(int64_t n);
hstu_status hstu_sl_embed(int64_t B, int64_t raw_total, int64_t max_raw_len,
                          const int64_t* raw_offsets, const int64_t* raw_ids,
                          const int64_t* raw_timestamps, uint64_t seed,
                          const void* content_table, int64_t n_content,
                          const void* action_table, int64_t n_action, int32_t d_model,
                          int64_t* out_offsets, void* out_X, int64_t* out_timestamps,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then returns the device status word that the last
 * call using this workspace left (HSTU_OK if none of its checks failed). */
hstu_status hstu_read_status(const void* workspace, size_t workspace_bytes, void* stream);

/* Test hook: byte offsets inside the workspace where hstu_layer_fwd (and the
 * last layer of hstu_stack_fwd) leaves its intermediates: the f1 output
 * [T, F] (U|V|Q|K after SiLU), the pre-LayerNorm attention output O [T, h*d_v]
 * (already scaled by 1/n_b) and the gated Z [T, h*d_v].
 * dtype HSTU_FP32: O and Z are fp32.  dtype HSTU_BF16: the f1 output is fp16;
 * O is stored per (row, head) as its mean m and standard deviation s over
 * the head's d_v values and the normalised values (O - m) / s: the fp16
 * values [T, h*d_v] at o_offset, then, at the next multiple of 256 bytes,
 * the (m, s) pairs as fp32 [T, h, 2]; Z (fp16) is formed inside the output
 * projection and written at z_offset only while hstu_debug_keep_z(1) is in
 * effect. */
hstu_status hstu_debug_offsets(const hstu_layer_desc* desc, int64_t B, int64_t total_tokens,
                               int64_t max_len, size_t* f1_offset, size_t* o_offset,
                               size_t* z_offset);

/* Tracing.  hstu_trace_enable(n) records a CUDA event pair around each of
 * the next n kernel launches (n = 0 turns tracing off); hstu_trace_only(id)
 * restricts the recording to launches of one kernel id (-1, the default:
 * every kernel; HSTU_ERR_INVALID_ARG for an unknown id); hstu_trace_read
 * synchronises and returns, per traced launch, the kernel id and the device
 * time in ms.  hstu_kernel_name maps an id to a name.  hstu_launch_count
 * counts every kernel this library has launched in this process. */
hstu_status hstu_trace_enable(int32_t max_records);
hstu_status hstu_trace_only(int32_t kernel_id);
int32_t hstu_trace_read(int32_t* kernel_ids, float* ms, int32_t capacity);
const char* hstu_kernel_name(int32_t kernel_id);
int64_t hstu_launch_count(void);

/* Test hook: with on = 1, later layer calls on the tensor-core path also
 * write the gated Z = LayerNorm(O) * U into the workspace (at the z offset
 * of hstu_debug_offsets) when the output projection forms it in its shared
 * memory (see the "ln_fusion" option); with on = 0 (the default) Z is in the
 * workspace only when the separate LayerNorm * U kernel formed it.
 * Process-wide.  Returns HSTU_ERR_INVALID_ARG for other values. */
hstu_status hstu_debug_keep_z(int32_t on);

/* Test hook for the failure detection of the in-kernel waits.  Every wait
 * inside the attention kernel is bounded: after wait_limit_us microseconds
 * (default 1 s) it gives up, the call's status word becomes HSTU_ERR_TIMEOUT,
 * and the kernel winds down (loads in flight land, tensor memory is freed)
 * and returns, so the context stays usable and the next call on the same
 * workspace runs normally.  hstu_debug_wait_test sets, for the NEXT attention
 * launch only (of any call, on any stream), the wait bound (0 = the default)
 * and, with inject_stall = 1, makes that launch's first CTA stop handing out
 * work after two items without telling its other roles, which then wait
 * until the bound runs out.  It touches no memory and issues no load; the
 * launch after that one uses the defaults again.  Not a page operation: the
 * pages describe no failure handling.  Returns HSTU_ERR_INVALID_ARG for an
 * inject_stall other than 0 or 1. */
hstu_status hstu_debug_wait_test(uint32_t wait_limit_us, int32_t inject_stall);

/* Process-wide options.  "ln_fusion": 1 forms LayerNorm(O) * U inside the
 * output projection's operand stage (Z never reaches memory), 0 writes Z with
 * a separate kernel that f2 then reads, 2 (default) chooses per layer: inside
 * f2 when d_model <= 512 (f2 then has at most two 256-column output tiles,
 * each of which forms Z again), the separate kernel otherwise.  All give the
 * same layer within the bf16 bound.  "gemm_pair": where a projection (f1 with
 * SiLU, f2 with its 16-bit residual, a plain-bias product) takes 256-column
 * output tiles, 1 (default) runs it on clusters of two CTAs sharing each
 * 256 x 256 tile through the pair MMA when its inner dimension is at least
 * 1024, 2 does so at any inner dimension, 0 never; all give bitwise the same
 * result.  Returns HSTU_ERR_INVALID_ARG for
 * an unknown name or value. */
hstu_status hstu_set_option(const char* name, int64_t value);

/* After an entry point returned HSTU_ERR_CUDA: the failing CUDA runtime
 * call's error and the step it belonged to, as text (per host thread; ""
 * if none). */
const char* hstu_last_error(void);

const char* hstu_status_string(hstu_status s);
int32_t hstu_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */

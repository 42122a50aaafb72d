// hstu_internal.h — declarations shared by the library's translation units:
// kernel argument blocks, launchers, tracing ids and the workspace layout.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/hstu.h"

namespace hstu {

// Query-tile height of the attention kernels and of every M tile.
constexpr int kTile = 128;

// ---------------------------------------------------------------- tracing
enum KernelId : int32_t {
  K_SCHEDULE = 0,
  K_TIME_REL = 1,
  K_GEMM_F1 = 2,
  K_ATTN = 3,
  K_LN_GATE = 4,
  K_GEMM_F2 = 5,
  K_MB_PLAN = 6,
  K_MB_GATHER = 7,
  K_ATTN_CAND = 8,
  K_SCORE = 9,
  K_SIMT_GEMM_F1 = 10,
  K_SIMT_ATTN = 11,
  K_SIMT_GEMM_F2 = 12,
  K_SIMT_ATTN_CAND = 13,
  K_CONVERT = 14,
  K_TIME_BUCKETS = 15,
  K_SL_OFFSETS = 16,
  K_SL_SELECT = 17,
  K_SL_GATHER = 18,
  K_RET_GATHER = 19,
  K_GEMM_SCORES = 20,
  K_TOPK_CHUNK = 21,
  K_TOPK_MERGE = 22,
  K_TF_LN = 23,
  K_TF_QKV = 24,
  K_TF_ATTN = 25,
  K_TF_OPROJ = 26,
  K_TF_FFN1 = 27,
  K_TF_FFN2 = 28,
  K_GEMM_FILTER = 29,
  K_FILTER_MERGE = 30,
  K_ATTN_BWD_DKV = 31,
  K_ATTN_BWD_DQ = 32,
  K_GEMM_BWD = 33,
  K_LN_BWD = 34,
  K_SUM_ROWS = 35,
  K_F32_TO_F16 = 36,
  K_LN_COEF = 37,
  K_NUM_KERNELS = 38
};
const char* kernel_name(int id);

// Wraps one kernel launch: counts it and, when tracing is on, brackets it
// with a CUDA event pair on `stream`.
struct LaunchScope {
  LaunchScope(int kernel_id, cudaStream_t stream);
  ~LaunchScope();
  int id;
  cudaStream_t s;
  int slot;
};

// ---------------------------------------------------------------- device info
int num_sms();
// Raises `fn`'s dynamic shared-memory limit to at least `bytes` on the
// current device (again only when a larger limit is needed).
cudaError_t ensure_smem_limit(const void* fn, int bytes);
// Bound of an in-kernel wait unless a test asks for a shorter one.
constexpr uint32_t kDefaultWaitLimitUs = 1000u * 1000u;
// The wait bound and stall injection for the next attention launch
// (hstu_debug_wait_test), reset to the defaults once taken.
void take_wait_test(uint32_t* limit_us, int* inject_stall);
// Whether layer calls of the tensor-core path also write the gated Z into the
// workspace (hstu_debug_keep_z).
bool keep_z();
// Records a failed CUDA runtime call for hstu_last_error (per host thread).
void note_cuda_error(cudaError_t e, const char* where);
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).  Returns false if the driver call is unavailable/failed.
// 2-D map of a row-major matrix with an explicit element type and swizzle.
bool encode_tmap_2d_ex(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                       CUtensorMapDataType dtype, CUtensorMapSwizzle swizzle);
// 2-D map of a row-major 16-bit matrix (bf16, or fp16 if f16), 128-byte swizzle.
bool encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool f16);

// ---------------------------------------------------------------- workspace
struct Header {           // first 256 bytes of every workspace
  int32_t status;         // hstu_status of the device checks
  int32_t n_items;        // attention work items of the history pass
  int32_t n_cand_items;   // attention work items of the current microbatch
  int32_t n_tiles;        // time-bucket tiles of the history pass
  int64_t mb_rows;        // rows of the current candidate microbatch
  int32_t work_next;      // dynamic work counter of the running attention launch
  int32_t work_done;      // CTAs of that launch that have finished
};

struct Layout {
  size_t header, items, t_rel, ubase, tbuckets, f1, o, ostats, z;
  size_t lncoef, lncoef_c;  // tensor-core path: LayerNorm coefficients per (row, head)
  size_t xres, xh;          // residual stream: fp32 (fp32 path) / fp16, also the next f1's operand
  size_t w16;               // tensor-core path: fp16 copies of W1 (layers >= 1) and W2, per layer
  size_t f1_cache;          // M-FALCON: every layer's f1 output (its K/V) for the history
  size_t mb_off, c_items, t_req_rel, xres_c, xb_c, xh_c, f1c, oc, ostats_c, zc;  // candidate microbatch
  size_t total;
  int64_t item_cap, cand_item_cap, mb_cap, tile_cap;
};
bool make_layout(const hstu_layer_desc& d, int n_layers, int64_t B, int64_t T, int64_t max_len,
                 int64_t total_cands, int64_t max_cands, int microbatch, Layout* L);

// ---------------------------------------------------------------- kernels
// One attention work item: (user, 128-row query tile, head), the number of
// 128-row KV tiles it reads, (causal self-attention) the index of the
// time-bucket tile of (user, query tile, KV tile 0), and the row offsets the
// kernel needs, so that starting an item takes no dependent loads.
struct AttnItem {
  int32_t b;
  int16_t qt, head;
  int32_t nkv;
  int32_t tile0;
  int32_t q_row0;   // first query row of the tile
  int32_t kv_row0;  // first KV row of the user
  int32_t n_q;      // query rows of the user
  int32_t n_kv;     // KV rows of the user (history length for candidates)
};
// A time-bucket tile: the bucket of t_i - t_j for 128 query rows x 128 KV
// columns, one byte each, 4 consecutive columns per 32-bit word, stored
// word-column-major ([32][128] words) so that a warp's 32 rows read 128
// contiguous bytes.
constexpr int kBucketTileWords = 32 * 128;

// Validate offsets; build the causal work list (user, q-tile, head) grouped
// by (user, head), longest users first, q-tiles longest first inside a group;
// ubase[b] = first time-bucket tile of user b.
void launch_schedule(const int64_t* offsets, int64_t B, int64_t T, int64_t max_len, int n_heads,
                     AttnItem* items, int64_t item_cap, int64_t* ubase, int64_t tile_cap,
                     Header* hdr, cudaStream_t s);
// Time-bucket tiles of every causal (q-tile, kv-tile) pair of the batch.
void launch_time_buckets(const int64_t* offsets, int64_t B, int64_t max_len, const int32_t* t_rel,
                         const int64_t* ubase, int64_t tile_cap, int St, int Nt,
                         uint32_t* tbuckets, Header* hdr, cudaStream_t s);
// Per-row timestamp relative to the user's first one (int32), with checks.
void launch_time_rel(const int64_t* offsets, int64_t B, int64_t max_len, const int64_t* ts,
                     int64_t T, int32_t* t_rel, Header* hdr, cudaStream_t s);

// C[M, N] = A[M, K] * W[n_off + N, K]^T with fused epilogue, bf16 tcgen05.
enum Epilogue { EPI_SILU = 0, EPI_RESID = 1, EPI_SCORE = 2, EPI_BIAS = 3, EPI_FILTER = 4 };
enum ResidKind { RESID_BF16 = 0, RESID_F32 = 1, RESID_F16 = 2 };
struct GemmCall {
  const void* A;  int64_t lda;   // [M_cap, K] row stride in elements
  const void* W;  int64_t ldw;   // [N_total, K]
  int ab_f16;                    // tensor-core path: A and W are fp16 (else bf16)
  int64_t M_cap;                 // rows allocated in A / out
  const int64_t* M_dev;          // actual rows (device), or null = M_cap
  int N, K, n_off;
  const void* bias;              // [N_total] (bf16 on the tensor-core path)
  void* out; int64_t ldo;        // written at columns n_off + n; may be null for EPI_RESID
  int out_f16;                   // tensor-core path: `out` is fp16 (else bf16)
  void* out32;                   // tensor-core EPI_RESID: optional fp32 copy of the output
  const void* resid; int64_t ldr;
  int resid_kind;                // tensor-core EPI_RESID residual: RESID_BF16, RESID_F32, RESID_F16
  int epi;
  int* status;
  // Tensor-core EPI_RESID only: when ln_x is set, A is not read; the kernel
  // builds A = LayerNorm(O) * U itself from the attention output stored as
  // (O - m) / s in fp16 (ln_x, [M, K]) with each (row, head)'s (m, s)
  // (ln_stats, [M, ln_h] pairs), U (the first K columns of ln_u, row stride
  // ld_u), gamma and beta (bf16 [K]); K = ln_h * ln_dv.  ln_coef: scratch of
  // M * ln_h words for each (row, head)'s LayerNorm coefficients, which the
  // launcher computes first.  z_dbg (optional, fp16 [M, K]) receives Z.
  const void* ln_x;
  const float* ln_stats;
  uint32_t* ln_coef;
  const void* ln_u; int64_t ld_u;
  const void* ln_gamma; const void* ln_beta;
  float ln_eps;
  int ln_h, ln_dv;
  void* z_dbg;
  // EPI_SILU only: also store the pre-activation A W^T + b (16-bit like `out`,
  // same layout)
  void* out_pre;
};
cudaError_t launch_gemm_tc(const GemmCall& g, cudaStream_t s, int kernel_id);
// Products for the backward pass: out[s * split_rows + m, n] (fp32, row
// stride ldo) = sum over the K blocks of split s of A[m, k] W[n, k], 16-bit
// operands (fp16 if ab_f16).  a_mn: A is stored [K, M] row-major (else
// [M, K]); w_mn: W is stored [K, N] row-major (else [N, K]).  splits > 1 cuts
// K into that many ranges (the caller sums the partial products); M, N
// multiples of 64 are not required (ragged edges read zeros, stores clip);
// K rows past K_rows read zeros.  With resid (fp32, same layout as out; splits
// = 1 only) the output is out = resid + A W^T, and out16 (bf16, optional)
// receives a copy.
struct GradGemm {
  const void* A; int64_t lda; int a_mn;
  const void* W; int64_t ldw; int w_mn;
  int ab_f16;
  int64_t M, N, K;
  int splits; int64_t split_rows;
  float* out; int64_t ldo;
  const float* resid;
  void* out16;             // with resid: a 16-bit copy of out, bf16 (or fp16 with out16_f16)
  int out16_f16;
  const void* zero_bias;   // bf16 zeros, at least N (the residual epilogue adds a bias)
  int* status;
  int* splits_used;        // optional: receives the number of splits launched (<= splits)
};
cudaError_t launch_gemm_grad(const GradGemm& g, cudaStream_t s, int kernel_id);
// scores[M_cap, N] (fp32, row stride ldo) = A[M_cap, K] * W[N, K]^T, no bias;
// N may be ragged (the last 256-column tile is clipped); K % 64 == 0,
// ldo % 4 == 0, bf16 or fp16 operands (ab_f16).
cudaError_t launch_gemm_scores(const void* A, int64_t lda, const void* W, int64_t ldw, int ab_f16,
                               int64_t M_cap, int64_t N, int K, float* out, int64_t ldo,
                               int* status, cudaStream_t s, int kernel_id,
                               int64_t w_row_step = 1, const int* run_if = nullptr);
// Scores of the same product that reach a per-row threshold, appended to
// per-row candidate lists: row r keeps (key, column) for every score s with
// desc_key(s) <= desc_key(tau[r * tau_stride]) (i.e. s >= tau, -0 as +0), at
// most `cap` per row (cnt[r] counts all; beyond cap only *overflow is set).
cudaError_t launch_gemm_filter(const void* A, int64_t lda, const void* W, int64_t ldw, int ab_f16,
                               int64_t M_cap, int64_t N, int K, const float* tau, int tau_stride,
                               uint32_t* cand_key, int32_t* cand_id, int* cnt, int cap,
                               int* overflow, int* status, cudaStream_t s, int kernel_id);
cudaError_t launch_gemm_simt_f32(const GemmCall& g, cudaStream_t s, int kernel_id);

// Pointwise causal attention (SELF) or candidate-vs-history (CAND).
struct AttnCall {
  int mode;                        // 0 self, 1 candidate
  int64_t B;
  const AttnItem* items; const int32_t* n_items; int64_t item_cap;  // tensor-core path
  const int64_t* q_off;            // [B+1] query-row offsets (self: = kv_off)
  const int64_t* kv_off;           // [B+1]
  const int64_t* q_rows_dev;       // SIMT path: device count of query rows (null = cap)
  const void* q_buf; int64_t q_rows_cap;   // f1 output holding Q (and self K/V for CAND)
  const void* kv_buf; int64_t kv_rows_cap; // f1 output holding the history K and V
  int64_t ld_f1;                   // row stride (elements) of both f1 buffers = F
  int q_col, k_col, v_col;         // column where head 0 of Q, K, V starts
  const int32_t* t_rel;            // [T_kv] int32 relative timestamps
  const int32_t* t_req_rel;        // CAND: [B] request time relative to the user's first
  const uint32_t* tbuckets;        // SELF: time-bucket tiles
  int32_t* work_next; int32_t* work_done;  // dynamic scheduling counters (header)
  const float* rab_pos; const float* rab_time;
  int Np, Nt, Sp, St, h, dqk, dv;
  void* O; int64_t ldo;            // tensor-core path: normalised O, fp16; SIMT path: O, fp32
  float* ostats;                   // tensor-core path: [rows, h] (mean, deviation) of each head's O
  int* status;
};
cudaError_t launch_attn_tc(const AttnCall& a, cudaStream_t s);

// Backward pass of the causal pointwise attention (self mode): from dO
// ([rows, h*d_v] fp16, row stride ld_do) and the f1 output (U|V|Q|K fp16,
// [rows, F]) and its pre-activation (`pre`, same layout), writes the
// gradients of the pre-activation's V, K and Q columns into dP ([rows, F]
// fp16) and adds the bias-table gradients into drab_pos / drab_time (fp32;
// the caller zeroes them).  Uses the forward's work list.
struct AttnBwdCall {
  const AttnItem* items; const int32_t* n_items; int64_t item_cap;
  const void* f1; const void* pre; void* dP; int64_t ld_f1; int64_t rows;
  const void* dO; int64_t ld_do;
  int q_col, k_col, v_col;
  const int32_t* t_rel;
  const float* rab_pos; const float* rab_time;
  float* drab_pos; float* drab_time;   // written (not accumulated) from rab_acc
  unsigned long long* rab_acc;         // workspace, h * (Np + Nt) words
  int Np, Nt, Sp, St, h, dqk, dv;
  int32_t* work_next; int32_t* work_done;
  int* status;
};
cudaError_t launch_attn_bwd(const AttnBwdCall& c, cudaStream_t s);
cudaError_t launch_attn_simt_f32(const AttnCall& a, cudaStream_t s);

// Z = LayerNorm(O) * gamma + beta, then * U (per row over h*d_v features).
cudaError_t launch_ln_gate(int dtype, const void* O, const void* f1, int64_t ld_f1,
                           const void* gamma, const void* beta, float eps, void* Z, int hdv,
                           int64_t rows_cap, const int64_t* rows_dev, const int* status,
                           cudaStream_t s);

// Tensor-core path: Z = LayerNorm(O) * U from the attention's normalised O
// (fp16 [rows, hdv]) and its per-(row, head) (mean, deviation) pairs.
// hdv and d_v multiples of 8, h <= 32.
// Per (row, head) LayerNorm coefficients from the heads' (m, s): with the
// row's moments mu, rstd over all h*d_v features, (O - mu) rstd = a + b xn for
// the normalised O xn of that head, a = (m - mu) rstd, b = s rstd; written as
// fp16 pairs (a in the low half) into coef [rows, h].
cudaError_t launch_ln_coef(const float* stats, int h, float eps, uint32_t* coef, int64_t rows_cap,
                           const int64_t* rows_dev, const int* status, cudaStream_t s);
cudaError_t launch_ln_gate_norm(const void* xn, const float* stats, const void* f1, int64_t ld_f1,
                                const void* gamma, const void* beta, float eps, void* Z, int hdv,
                                int h, int dv, int64_t rows_cap, const int64_t* rows_dev,
                                const int* status, cudaStream_t s);
// Whether f2 forms LayerNorm * U in its operand stage (else a separate
// kernel writes Z first) for a layer of this width; hstu_set_option("ln_fusion", ...).
bool ln_fusion_for(int d_model);
// Whether products with 256-column tiles and inner dimension K (SiLU, plain
// bias, 16-bit residual) run on CTA pairs (the pair MMA);
// hstu_set_option("gemm_pair", ...).
bool gemm_pair_for(int K);

// bf16 -> fp16 (round to nearest, saturating at +-65504) of up to
// kMaxConvSegs segments in one launch; n elements each, multiples of 8.
constexpr int kMaxConvSegs = 32;
struct ConvSeg {
  const void* src;
  void* dst;
  int64_t n;
};
struct ConvBatch {
  ConvSeg seg[kMaxConvSegs];
  int n;
};
cudaError_t launch_bf16_to_f16(const ConvBatch& cb, cudaStream_t s);

// M-FALCON microbatch plumbing.
void launch_mb_plan(const int64_t* hist_off, const int64_t* cand_off, int64_t B, int64_t max_len,
                    int64_t max_cands, int k, int microbatch, int n_heads,
                    const int64_t* hist_ts, const int64_t* request_ts, int64_t* mb_off,
                    AttnItem* items, int64_t item_cap, int32_t* t_req_rel, Header* hdr,
                    cudaStream_t s);
cudaError_t launch_mb_gather(int dtype, const void* cands, int64_t d, const int64_t* cand_off,
                             const int64_t* mb_off, int64_t B, int k, int microbatch,
                             void* xc, int64_t rows_cap, const int64_t* rows_dev,
                             const int* status, cudaStream_t s);
cudaError_t launch_score(int dtype, const float* xc, int64_t d, const void* head_vec,
                         const int64_t* cand_off, const int64_t* mb_off, int64_t B, int k,
                         int microbatch, float* scores, int64_t rows_cap,
                         const int64_t* rows_dev, const int* status, cudaStream_t s);

}  // namespace hstu

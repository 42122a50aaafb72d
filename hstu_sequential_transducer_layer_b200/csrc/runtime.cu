// runtime.cu — host-side runtime of libhstu: launch counting and tracing,
// device queries, TMA descriptor encoding, and the workspace layout.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <map>
#include <utility>
#include <vector>

#include "hstu_internal.h"

namespace hstu {

// ---------------------------------------------------------------- tracing
namespace {
std::atomic<int64_t> g_launches{0};
std::mutex g_trace_mu;
int g_trace_cap = 0;
int g_trace_used = 0;
int g_trace_only = -1;  // trace only this kernel id (-1: every kernel)
std::vector<cudaEvent_t> g_ev0, g_ev1;
std::vector<int> g_ids;
}  // namespace

const char* kernel_name(int id) {
  static const char* names[K_NUM_KERNELS] = {
      "schedule",   "time_rel",   "gemm_f1_tc",      "attn_tc",
      "ln_gate",    "gemm_f2_tc", "mb_plan",         "mb_gather",
      "attn_cand_tc", "score",    "gemm_f1_simt_f32", "attn_simt_f32",
      "gemm_f2_simt_f32", "attn_cand_simt_f32", "bf16_to_f16", "time_buckets",
      "sl_offsets", "sl_select", "sl_gather", "ret_gather", "gemm_scores_tc", "topk_chunk",
      "topk_merge", "tf_ln", "tf_qkv_tc", "tf_softmax_attn_tc", "tf_oproj_tc", "tf_ffn1_tc",
      "tf_ffn2_tc", "gemm_filter_tc", "filter_merge", "attn_bwd_dkv_tc", "attn_bwd_dq_tc",
      "gemm_bwd_tc", "ln_bwd", "sum_rows", "f32_to_f16", "ln_coef"};
  return (id >= 0 && id < K_NUM_KERNELS) ? names[id] : "unknown";
}

LaunchScope::LaunchScope(int kernel_id, cudaStream_t stream) : id(kernel_id), s(stream), slot(-1) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (g_trace_used < g_trace_cap && (g_trace_only < 0 || g_trace_only == kernel_id)) {
    slot = g_trace_used++;
    g_ids[slot] = kernel_id;
    cudaEventRecord(g_ev0[slot], s);
  }
}
LaunchScope::~LaunchScope() {
  if (slot >= 0) cudaEventRecord(g_ev1[slot], s);
}

// ---------------------------------------------------------------- device
// The dynamic shared-memory limit is an attribute of a kernel on one device:
// it is raised per (kernel, device) pair, under a lock, whenever a launch
// needs more than was set before (so the first launch on a second GPU of the
// same process raises it there too, and a kernel whose shared memory depends
// on the shape gets the larger limit).
cudaError_t ensure_smem_limit(const void* fn, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> set_to;  // (kernel, device) -> limit
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(fn, dev);
  const auto it = set_to.find(key);
  if (it != set_to.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) set_to[key] = bytes;
  return e;
}

// ---------------------------------------------------------------- wait test hook
namespace {
std::mutex g_wait_mu;
uint32_t g_wait_limit_us = 0;  // 0: the default bound
int g_inject_stall = 0;
}  // namespace

namespace {
std::atomic<int> g_keep_z{0};
thread_local char g_last_error[256] = "";
}  // namespace

void note_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where ? where : "?",
           cudaGetErrorString(e), (int)e);
}

bool keep_z() { return g_keep_z.load(std::memory_order_relaxed) != 0; }

namespace {
std::atomic<int> g_ln_fusion{2};
std::atomic<int> g_gemm_pair{1};
}  // namespace

// 1 (automatic): on pairs when K >= 1024.  With shorter K the SiLU epilogue
// of a tile takes about as long as its MMAs, and the pair, whose MMAs wait
// for both CTAs' epilogues, is slower than single CTAs (measured at K = 512:
// f1 8 % slower; at K = 1024: f1 2-5 % faster, f2 15-20 %).
bool gemm_pair_for(int K) {
  const int m = g_gemm_pair.load(std::memory_order_relaxed);
  return m == 2 || (m == 1 && K >= 1024);
}

// 2 (automatic): inside f2 when f2 has at most two 256-column output tiles
// (d_model <= 512); with more, each A block would be formed once per tile and
// the separate kernel is faster (measured on the 8-layer d_model = 1024 stack).
bool ln_fusion_for(int d_model) {
  const int m = g_ln_fusion.load(std::memory_order_relaxed);
  return m == 1 || (m == 2 && d_model <= 512);
}

void take_wait_test(uint32_t* limit_us, int* inject_stall) {
  std::lock_guard<std::mutex> lk(g_wait_mu);
  *limit_us = g_wait_limit_us ? g_wait_limit_us : kDefaultWaitLimitUs;
  *inject_stall = g_inject_stall;
  g_wait_limit_us = 0;
  g_inject_stall = 0;
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_tmap_2d_ex(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                       CUtensorMapDataType dtype, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool f16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- workspace
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

bool make_layout(const hstu_layer_desc& d, int n_layers, int64_t B, int64_t T, int64_t max_len,
                 int64_t total_cands, int64_t max_cands, int microbatch, Layout* L) {
  if (B < 0 || T < 0 || n_layers < 1 || total_cands < 0 || max_cands < 0) return false;
  const bool bf16 = d.dtype == HSTU_BF16;
  const size_t es = bf16 ? 2 : 4;
  const size_t F = 2 * (size_t)d.n_heads * (d.d_v + d.d_qk);
  const size_t hdv = (size_t)d.n_heads * d.d_v;
  const size_t dm = (size_t)d.d_model;
  const bool mf = total_cands > 0 || microbatch > 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += up256(bytes);
    return o;
  };
  *L = Layout{};
  L->item_cap = ((T + kTile - 1) / kTile + B) * (int64_t)d.n_heads;
  L->header = take(256);
  L->items = take((size_t)L->item_cap * sizeof(AttnItem));
  L->t_rel = take((size_t)T * 4);
  // time-bucket tiles: sum over users of nq(nq+1)/2 <= (sum nq) * (max_q + 1) / 2
  const int64_t max_q = (max_len + kTile - 1) / kTile;
  L->tile_cap = bf16 ? ((T + kTile - 1) / kTile + B) * (max_q + 1) / 2 + 1 : 0;
  L->ubase = take((size_t)(B + 1) * 8);
  L->tbuckets = take((size_t)L->tile_cap * kBucketTileWords * 4);
  if (!mf) {
    L->f1 = take((size_t)T * F * es);
  } else {
    L->f1_cache = take((size_t)n_layers * T * F * es);
    L->f1 = L->f1_cache;
  }
  // attention output: fp32 O (fp32 path), or the normalised fp16 O followed
  // by each (row, head)'s (mean, deviation) (tensor-core path)
  L->o = take(bf16 ? up256((size_t)T * hdv * 2) + (size_t)T * d.n_heads * 8 : (size_t)T * hdv * 4);
  L->ostats = bf16 ? L->o + up256((size_t)T * hdv * 2) : 0;
  // LayerNorm coefficients per (row, head) for f2's operand stage
  L->lncoef = bf16 ? take((size_t)T * d.n_heads * 4) : 0;
  // Z: the fp32 path's LayerNorm * U output; on the tensor-core path Z is
  // formed in the output projection's shared memory and written here only
  // when a test asks for it (hstu_debug_keep_z)
  L->z = take((size_t)T * hdv * es);
  // residual stream between layers: fp16 on the tensor-core path, fp32 otherwise
  L->xres = bf16 ? 0 : take((size_t)T * dm * 4);
  L->xh = bf16 ? take((size_t)T * dm * 2) : L->xres;
  L->w16 = bf16 ? take((size_t)n_layers * (F * dm + dm * hdv) * 2) : 0;
  if (mf) {
    if (microbatch < 1) return false;
    int64_t cap = std::min<int64_t>(total_cands, B * (int64_t)microbatch);
    L->mb_cap = cap;
    L->cand_item_cap = ((cap + kTile - 1) / kTile + B) * (int64_t)d.n_heads;
    L->mb_off = take((size_t)(B + 1) * 8);
    L->c_items = take((size_t)L->cand_item_cap * sizeof(AttnItem));
    L->t_req_rel = take((size_t)B * 4);
    L->xres_c = take((size_t)cap * dm * 4);
    L->xb_c = bf16 ? take((size_t)cap * dm * 2) : L->xres_c;
    L->xh_c = bf16 ? take((size_t)cap * dm * 2) : L->xres_c;
    L->f1c = take((size_t)cap * F * es);
    L->oc = take(bf16 ? up256((size_t)cap * hdv * 2) + (size_t)cap * d.n_heads * 8
                      : (size_t)cap * hdv * 4);
    L->ostats_c = bf16 ? L->oc + up256((size_t)cap * hdv * 2) : 0;
    L->lncoef_c = bf16 ? take((size_t)cap * d.n_heads * 4) : 0;
    L->zc = take((size_t)cap * hdv * es);
  }
  (void)max_len;
  (void)max_cands;
  L->total = off;
  return true;
}

}  // namespace hstu

// ---------------------------------------------------------------- C ABI
extern "C" {

const char* hstu_last_error(void) { return hstu::g_last_error; }

hstu_status hstu_set_option(const char* name, int64_t value) {
  if (!name) return HSTU_ERR_INVALID_ARG;
  if (std::strcmp(name, "ln_fusion") == 0) {
    if (value < 0 || value > 2) return HSTU_ERR_INVALID_ARG;
    hstu::g_ln_fusion.store((int)value);
    return HSTU_OK;
  }
  if (std::strcmp(name, "gemm_pair") == 0) {
    if (value < 0 || value > 2) return HSTU_ERR_INVALID_ARG;
    hstu::g_gemm_pair.store((int)value);
    return HSTU_OK;
  }
  return HSTU_ERR_INVALID_ARG;
}

hstu_status hstu_debug_keep_z(int32_t on) {
  if (on != 0 && on != 1) return HSTU_ERR_INVALID_ARG;
  hstu::g_keep_z.store(on);
  return HSTU_OK;
}

hstu_status hstu_debug_wait_test(uint32_t wait_limit_us, int32_t inject_stall) {
  if (inject_stall != 0 && inject_stall != 1) return HSTU_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(hstu::g_wait_mu);
  hstu::g_wait_limit_us = wait_limit_us;
  hstu::g_inject_stall = inject_stall;
  return HSTU_OK;
}


hstu_status hstu_trace_enable(int32_t max_records) {
  using namespace hstu;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  for (auto e : g_ev0) cudaEventDestroy(e);
  for (auto e : g_ev1) cudaEventDestroy(e);
  g_ev0.clear();
  g_ev1.clear();
  g_ids.clear();
  g_trace_cap = 0;
  g_trace_used = 0;
  if (max_records <= 0) return HSTU_OK;
  g_ev0.resize(max_records);
  g_ev1.resize(max_records);
  g_ids.resize(max_records, -1);
  for (int i = 0; i < max_records; ++i) {
    if (cudaEventCreate(&g_ev0[i]) != cudaSuccess || cudaEventCreate(&g_ev1[i]) != cudaSuccess)
      return HSTU_ERR_CUDA;
  }
  g_trace_cap = max_records;
  return HSTU_OK;
}

hstu_status hstu_trace_only(int32_t kernel_id) {
  using namespace hstu;
  if (kernel_id < -1 || kernel_id >= K_NUM_KERNELS) return HSTU_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_only = kernel_id;
  return HSTU_OK;
}

int32_t hstu_trace_read(int32_t* kernel_ids, float* ms, int32_t capacity) {
  using namespace hstu;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  int n = std::min(g_trace_used, (int)capacity);
  for (int i = 0; i < n; ++i) {
    float t = -1.f;
    if (cudaEventSynchronize(g_ev1[i]) == cudaSuccess) cudaEventElapsedTime(&t, g_ev0[i], g_ev1[i]);
    if (kernel_ids) kernel_ids[i] = g_ids[i];
    if (ms) ms[i] = t;
  }
  return n;
}

const char* hstu_kernel_name(int32_t kernel_id) { return hstu::kernel_name(kernel_id); }

int64_t hstu_launch_count(void) { return hstu::g_launches.load(); }

}  // extern "C"

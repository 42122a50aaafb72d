// api.cu — the C ABI of libhstu (declared in include/hstu.h): host-side
// argument checks, workspace carving, and the launch sequence of a layer,
// a stack and M-FALCON ranking.  Everything is enqueued on the caller's
// stream; nothing here synchronises except hstu_read_status.
#include <cmath>
#include <cstring>

#include "hstu_internal.h"

using namespace hstu;

namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

hstu_status check_desc(const hstu_layer_desc* d) {
  if (!d) return HSTU_ERR_INVALID_ARG;
  if (d->dtype != HSTU_BF16 && d->dtype != HSTU_FP32) return HSTU_ERR_INVALID_ARG;
  if (d->d_model <= 0 || d->n_heads <= 0 || d->d_qk <= 0 || d->d_v <= 0) return HSTU_ERR_INVALID_ARG;
  if (d->n_pos_buckets < 1 || d->n_pos_buckets > 4096 || d->n_time_buckets < 1 ||
      d->n_time_buckets > 4096)
    return HSTU_ERR_INVALID_ARG;
  if (d->pos_sub_bits < 0 || d->pos_sub_bits > 20 || d->time_sub_bits < 0 || d->time_sub_bits > 20)
    return HSTU_ERR_INVALID_ARG;
  if (!(d->ln_eps >= 0.f) || !std::isfinite(d->ln_eps)) return HSTU_ERR_INVALID_ARG;
  const int64_t hdv = (int64_t)d->n_heads * d->d_v;
  if (hdv > 2048 || (int64_t)d->d_model > 65536) return HSTU_ERR_UNSUPPORTED;
  if (d->dtype == HSTU_BF16) {
    if (d->d_qk != d->d_v || (d->d_qk != 64 && d->d_qk != 128)) return HSTU_ERR_UNSUPPORTED;
    if (d->d_model % 64 != 0 || hdv % 64 != 0) return HSTU_ERR_UNSUPPORTED;
    if (d->n_time_buckets > 256) return HSTU_ERR_UNSUPPORTED;  // one byte per time bucket
  } else {
    if (d->d_qk > 128 || d->d_v > 128 || d->d_qk % 4 || d->d_v % 4 || d->d_model % 4)
      return HSTU_ERR_UNSUPPORTED;
  }
  return HSTU_OK;
}

hstu_status check_weights(const hstu_layer_weights* w) {
  if (!w) return HSTU_ERR_INVALID_ARG;
  const void* p[8] = {w->W1, w->b1, w->W2, w->b2, w->ln_gamma, w->ln_beta, w->rab_pos, w->rab_time};
  for (const void* q : p)
    if (!q || !al16(q)) return HSTU_ERR_INVALID_ARG;
  if ((w->W1_f16 && !al16(w->W1_f16)) || (w->W2_f16 && !al16(w->W2_f16)))
    return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status check_sizes(int64_t B, int64_t T, int64_t max_len) {
  if (B < 0 || T < 0 || max_len < 1 || max_len > (1ll << 30)) return HSTU_ERR_INVALID_ARG;
  if (T > (1ll << 31) - 1024 || B > (1ll << 30)) return HSTU_ERR_UNSUPPORTED;
  if (T > B * max_len) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

struct Ctx {
  hstu_layer_desc d;
  size_t es;
  int F, hdv, qcol, kcol, vcol;
  cudaStream_t s;
  Header* hdr;
  int* status;
  bool bf16;
};

Ctx make_ctx(const hstu_layer_desc& d, void* ws, void* stream) {
  Ctx c;
  c.d = d;
  c.bf16 = d.dtype == HSTU_BF16;
  c.es = c.bf16 ? 2 : 4;
  c.hdv = d.n_heads * d.d_v;
  c.F = 2 * c.hdv + 2 * d.n_heads * d.d_qk;
  c.vcol = c.hdv;
  c.qcol = 2 * c.hdv;
  c.kcol = 2 * c.hdv + d.n_heads * d.d_qk;
  c.s = static_cast<cudaStream_t>(stream);
  c.hdr = static_cast<Header*>(ws);
  c.status = &c.hdr->status;
  return c;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

cudaError_t gemm(const Ctx& c, const GemmCall& g, int kid_tc, int kid_simt) {
  return c.bf16 ? launch_gemm_tc(g, c.s, kid_tc) : launch_gemm_simt_f32(g, c.s, kid_simt);
}

// Operands of one f1 / f2 on the tensor-core path: fp16 copies of the
// weights live in the workspace (W1 of layers >= 1, every W2); layer 0's f1
// multiplies the caller's bf16 X by the caller's bf16 W1 directly.
struct LayerOps {
  const void* W1;
  int w1_f16;
  const void* W2;
};

LayerOps layer_ops(const Ctx& c, const hstu_layer_weights& w, const Layout& L, void* ws, int l,
                   int n_layers) {
  LayerOps o{w.W1, 0, w.W2};
  if (!c.bf16) return o;
  const size_t F = c.F, dm = c.d.d_model, hdv = c.hdv;
  uint8_t* base = at<uint8_t>(ws, L.w16) + (size_t)l * (F * dm + dm * hdv) * 2;
  if (l > 0) {
    o.W1 = w.W1_f16 ? w.W1_f16 : base;
    o.w1_f16 = 1;
  }
  o.W2 = w.W2_f16 ? w.W2_f16 : base + F * dm * 2;
  (void)n_layers;
  return o;
}

// fp16 copies of the weights the call needs (W1 of layers >= 1, every W2),
// batched kMaxConvSegs segments per launch.
cudaError_t convert_weights(const Ctx& c, const hstu_layer_weights* w, int n_layers,
                            const Layout& L, void* ws) {
  if (!c.bf16) return cudaSuccess;
  const int64_t F = c.F, dm = c.d.d_model, hdv = c.hdv;
  ConvBatch cb{};
  for (int l = 0; l < n_layers; ++l) {
    LayerOps o = layer_ops(c, w[l], L, ws, l, n_layers);
    if (l > 0 && !w[l].W1_f16) cb.seg[cb.n++] = ConvSeg{w[l].W1, const_cast<void*>(o.W1), F * dm};
    if (!w[l].W2_f16) cb.seg[cb.n++] = ConvSeg{w[l].W2, const_cast<void*>(o.W2), dm * hdv};
    if (cb.n > kMaxConvSegs - 2 || l == n_layers - 1) {
      cudaError_t e = launch_bf16_to_f16(cb, c.s);
      if (e != cudaSuccess) return e;
      cb.n = 0;
    }
  }
  return cudaSuccess;
}

// f1 (all columns, or only the V and K columns when kv_only); the output is
// fp16 on the tensor-core path.
cudaError_t run_f1(const Ctx& c, const hstu_layer_weights& w, const LayerOps& ops, const void* X,
                   int a_f16, int64_t rows_cap, const int64_t* rows_dev, void* f1, bool kv_only) {
  GemmCall g{};
  g.A = X;
  g.lda = c.d.d_model;
  g.W = ops.W1;
  g.ldw = c.d.d_model;
  g.ab_f16 = a_f16;
  g.M_cap = rows_cap;
  g.M_dev = rows_dev;
  g.K = c.d.d_model;
  g.bias = w.b1;
  g.out = f1;
  g.out_f16 = 1;
  g.ldo = c.F;
  g.epi = EPI_SILU;
  g.status = c.status;
  if (!kv_only) {
    g.N = c.F;
    g.n_off = 0;
    return gemm(c, g, K_GEMM_F1, K_SIMT_GEMM_F1);
  }
  g.N = c.hdv;  // V
  g.n_off = c.vcol;
  cudaError_t e = gemm(c, g, K_GEMM_F1, K_SIMT_GEMM_F1);
  if (e != cudaSuccess) return e;
  g.N = c.d.n_heads * c.d.d_qk;  // K
  g.n_off = c.kcol;
  return gemm(c, g, K_GEMM_F1, K_SIMT_GEMM_F1);
}

// f2 + bias + residual.  resid_kind (tensor-core path): the residual is the
// caller's bf16 rows, an fp32 stream or an fp16 stream; out16 (fp16 stream, or
// the caller's bf16 output when out16_bf16) and out32 (fp32 stream) may each
// be null.  Each output element is read (residual) before it is written, by
// the same warp, so a stream may be updated in place.
// With `ostats` (tensor-core path, LayerNorm * U fused): f2's A operand is
// LayerNorm(O) * U, built by the GEMM itself from the attention's normalised
// O (`Z`), its statistics (`ostats`) and U (the first h*d_v columns of `f1`);
// `z_dbg` takes an optional copy of Z.  Without: `Z` is LayerNorm * U itself.
cudaError_t run_f2(const Ctx& c, const hstu_layer_weights& w, const LayerOps& ops, const void* Z,
                   const float* ostats, uint32_t* coef, const void* f1, void* z_dbg,
                   const void* resid, int resid_kind, int64_t rows_cap, const int64_t* rows_dev,
                   void* out16, bool out16_bf16, float* out32) {
  GemmCall g{};
  g.A = Z;
  if (c.bf16 && ostats) {  // Z formed in f2's operand stage
    g.A = nullptr;
    g.ln_x = Z;
    g.ln_stats = ostats;
    g.ln_coef = coef;
    g.ln_u = f1;
    g.ld_u = c.F;
    g.ln_gamma = w.ln_gamma;
    g.ln_beta = w.ln_beta;
    g.ln_eps = c.d.ln_eps;
    g.ln_h = c.d.n_heads;
    g.ln_dv = c.d.d_v;
    g.z_dbg = z_dbg;
  }
  g.lda = c.hdv;
  g.W = ops.W2;
  g.ldw = c.hdv;
  g.ab_f16 = 1;
  g.M_cap = rows_cap;
  g.M_dev = rows_dev;
  g.N = c.d.d_model;
  g.K = c.hdv;
  g.n_off = 0;
  g.bias = w.b2;
  g.ldo = c.d.d_model;
  g.resid = resid;
  g.ldr = c.d.d_model;
  g.epi = EPI_RESID;
  g.status = c.status;
  if (c.bf16) {
    g.out = out16;
    g.out_f16 = out16_bf16 ? 0 : 1;
    g.out32 = out32;
    g.resid_kind = resid_kind;
  } else {  // fp32 layers: everything is already fp32; `out` is the fp32 destination
    g.out = out16 ? out16 : out32;
  }
  return gemm(c, g, K_GEMM_F2, K_SIMT_GEMM_F2);
}

AttnCall attn_common(const Ctx& c, const hstu_layer_weights& w, int64_t B) {
  AttnCall a{};
  a.B = B;
  a.ld_f1 = c.F;
  a.q_col = c.qcol;
  a.k_col = c.kcol;
  a.v_col = c.vcol;
  a.rab_pos = w.rab_pos;
  a.rab_time = w.rab_time;
  a.Np = c.d.n_pos_buckets;
  a.Nt = c.d.n_time_buckets;
  a.Sp = c.d.pos_sub_bits;
  a.St = c.d.time_sub_bits;
  a.h = c.d.n_heads;
  a.dqk = c.d.d_qk;
  a.dv = c.d.d_v;
  a.ldo = c.hdv;
  a.work_next = &c.hdr->work_next;
  a.work_done = &c.hdr->work_done;
  a.status = c.status;
  return a;
}

cudaError_t attn(const Ctx& c, const AttnCall& a) {
  return c.bf16 ? launch_attn_tc(a, c.s) : launch_attn_simt_f32(a, c.s);
}

// One causal layer over the jagged rows described by `off`: f1 reads `A`,
// f2 adds `resid` and writes out16 / out32 (see run_f2).
cudaError_t run_layer(const Ctx& c, const hstu_layer_weights& w, const LayerOps& ops, int64_t B,
                      int64_t T, const int64_t* off, const void* A, int a_f16, const void* resid,
                      int resid_kind, void* out16, bool out16_bf16, float* out32, void* f1,
                      const Layout& L, void* ws) {
  cudaError_t e = run_f1(c, w, ops, A, a_f16, T, nullptr, f1, false);
  if (e != cudaSuccess) return e;
  AttnCall a = attn_common(c, w, B);
  a.mode = 0;
  a.items = at<AttnItem>(ws, L.items);
  a.n_items = &c.hdr->n_items;
  a.item_cap = L.item_cap;
  a.q_off = off;
  a.kv_off = off;
  a.q_buf = f1;
  a.q_rows_cap = T;
  a.kv_buf = f1;
  a.kv_rows_cap = T;
  a.t_rel = at<int32_t>(ws, L.t_rel);
  a.tbuckets = at<uint32_t>(ws, L.tbuckets);
  a.O = at<void>(ws, L.o);
  a.ostats = c.bf16 ? at<float>(ws, L.ostats) : nullptr;
  e = attn(c, a);
  if (e != cudaSuccess) return e;
  if (c.bf16 && ln_fusion_for(c.d.d_model))  // LayerNorm * U inside f2's operand stage
    return run_f2(c, w, ops, at<void>(ws, L.o), at<float>(ws, L.ostats),
                  at<uint32_t>(ws, L.lncoef), f1, keep_z() ? at<void>(ws, L.z) : nullptr, resid,
                  resid_kind, T, nullptr, out16, out16_bf16, out32);
  if (c.bf16)  // LayerNorm * U from the normalised O, then f2 reads Z
    e = launch_ln_gate_norm(at<void>(ws, L.o), at<float>(ws, L.ostats), f1, c.F, w.ln_gamma,
                            w.ln_beta, c.d.ln_eps, at<void>(ws, L.z), c.hdv, c.d.n_heads,
                            c.d.d_v, T, nullptr, c.status, c.s);
  else
    e = launch_ln_gate(c.d.dtype, at<void>(ws, L.o), f1, c.F, w.ln_gamma, w.ln_beta, c.d.ln_eps,
                       at<void>(ws, L.z), c.hdv, T, nullptr, c.status, c.s);
  if (e != cudaSuccess) return e;
  return run_f2(c, w, ops, at<void>(ws, L.z), nullptr, nullptr, nullptr, nullptr, resid,
                resid_kind, T, nullptr, out16, out16_bf16, out32);
}

hstu_status finish(cudaError_t e) {
  if (e == cudaSuccess) e = cudaPeekAtLastError();
  if (e == cudaSuccess) return HSTU_OK;
  note_cuda_error(e, "forward");
  return HSTU_ERR_CUDA;
}

hstu_status stack_impl(const hstu_layer_desc* desc, int32_t n_layers,
                       const hstu_layer_weights* weights, int64_t B, int64_t T, int64_t max_len,
                       const int64_t* offsets, const void* X, const int64_t* timestamps,
                       void* out, void* ws, size_t ws_bytes, void* stream) {
  hstu_status st = check_desc(desc);
  if (st != HSTU_OK) return st;
  if (n_layers < 1 || !weights) return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if ((st = check_weights(&weights[l])) != HSTU_OK) return st;
  if ((st = check_sizes(B, T, max_len)) != HSTU_OK) return st;
  if (!offsets || !al16(offsets) || !ws || !al256(ws)) return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (!X || !out || !timestamps || !al16(X) || !al16(out) || !al16(timestamps)))
    return HSTU_ERR_INVALID_ARG;
  if (T > 0 && X == out) return HSTU_ERR_INVALID_ARG;
  Layout L;
  if (!make_layout(*desc, n_layers, B, T, max_len, 0, 0, 0, &L)) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return HSTU_ERR_WORKSPACE;
  Ctx c = make_ctx(*desc, ws, stream);
  launch_schedule(offsets, B, T, max_len, desc->n_heads, at<AttnItem>(ws, L.items), L.item_cap,
                  at<int64_t>(ws, L.ubase), L.tile_cap, c.hdr, c.s);
  if (T == 0) return finish(cudaSuccess);
  launch_time_rel(offsets, B, max_len, timestamps, T, at<int32_t>(ws, L.t_rel), c.hdr, c.s);
  if (c.bf16)  // time buckets: computed once, shared by every head and layer
    launch_time_buckets(offsets, B, max_len, at<int32_t>(ws, L.t_rel), at<int64_t>(ws, L.ubase),
                        L.tile_cap, desc->time_sub_bits, desc->n_time_buckets,
                        at<uint32_t>(ws, L.tbuckets), c.hdr, c.s);
  // Between layers the residual stream is fp16 on the tensor-core path (xh: the
  // next f1's operand, updated in place by f2) and fp32 on the fp32 path.
  float* xres = at<float>(ws, L.xres);
  void* xh = at<void>(ws, L.xh);
  cudaError_t e = convert_weights(c, weights, n_layers, L, ws);
  for (int l = 0; l < n_layers && e == cudaSuccess; ++l) {
    const bool first = l == 0, last = l == n_layers - 1;
    const LayerOps ops = layer_ops(c, weights[l], L, ws, l, n_layers);
    const void* A = first ? X : (c.bf16 ? xh : (const void*)xres);
    const void* resid = first ? X : (c.bf16 ? xh : (const void*)xres);
    void* o16 = last ? out : (c.bf16 ? xh : nullptr);
    float* o32 = (last || c.bf16) ? nullptr : xres;
    e = run_layer(c, weights[l], ops, B, T, offsets, A, first ? 0 : 1, resid,
                  first ? RESID_BF16 : RESID_F16, o16, last, o32, at<void>(ws, L.f1), L, ws);
  }
  return finish(e);
}

}  // namespace

extern "C" {

size_t hstu_workspace_size(const hstu_layer_desc* desc, int32_t n_layers, int64_t B,
                           int64_t total_tokens, int64_t max_len, int64_t total_cands,
                           int64_t max_cands, int32_t microbatch) {
  if (check_desc(desc) != HSTU_OK) return 0;
  if (check_sizes(B, total_tokens, max_len) != HSTU_OK) return 0;
  if (total_cands < 0 || max_cands < 0 || microbatch < 0) return 0;
  if (total_cands > 0 && microbatch < 1) return 0;
  Layout L;
  if (!make_layout(*desc, n_layers, B, total_tokens, max_len, total_cands, max_cands, microbatch,
                   &L))
    return 0;
  return L.total;
}

hstu_status hstu_layer_fwd(const hstu_layer_desc* desc, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const hstu_layer_weights* weights, const int64_t* timestamps,
                           void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return stack_impl(desc, 1, weights, B, total_tokens, max_len, offsets, X, timestamps, out,
                    workspace, workspace_bytes, stream);
}

hstu_status hstu_stack_fwd(const hstu_layer_desc* desc, int32_t n_layers,
                           const hstu_layer_weights* weights, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const int64_t* timestamps, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return stack_impl(desc, n_layers, weights, B, total_tokens, max_len, offsets, X, timestamps, out,
                    workspace, workspace_bytes, stream);
}

hstu_status hstu_mfalcon_rank(const hstu_layer_desc* desc, int32_t n_layers,
                              const hstu_layer_weights* weights, int64_t B, int64_t total_hist,
                              int64_t max_len, const int64_t* hist_offsets, const void* history,
                              const int64_t* hist_timestamps, int64_t total_cands,
                              int64_t max_cands, const int64_t* cand_offsets,
                              const void* candidates, const int64_t* request_ts,
                              int32_t microbatch, const void* head_vec, float* scores,
                              void* ws, size_t ws_bytes, void* stream) {
  hstu_status st = check_desc(desc);
  if (st != HSTU_OK) return st;
  if (n_layers < 1 || !weights) return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if ((st = check_weights(&weights[l])) != HSTU_OK) return st;
  const int64_t T = total_hist;
  if ((st = check_sizes(B, T, max_len)) != HSTU_OK) return st;
  if (total_cands < 0 || max_cands < 0 || microbatch < 1) return HSTU_ERR_INVALID_ARG;
  if (total_cands > B * max_cands) return HSTU_ERR_INVALID_ARG;
  if (total_cands > (1ll << 31) - 1024) return HSTU_ERR_UNSUPPORTED;
  if (!hist_offsets || !cand_offsets || !al16(hist_offsets) || !al16(cand_offsets) || !ws ||
      !al256(ws))
    return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (!history || !hist_timestamps || !al16(history) || !al16(hist_timestamps)))
    return HSTU_ERR_INVALID_ARG;
  if (total_cands > 0 && (!candidates || !scores || !head_vec || !al16(candidates) ||
                          !al16(scores) || !al16(head_vec)))
    return HSTU_ERR_INVALID_ARG;
  if (request_ts && !al16(request_ts)) return HSTU_ERR_INVALID_ARG;
  Layout L;
  if (!make_layout(*desc, n_layers, B, T, max_len, total_cands, max_cands, microbatch, &L))
    return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return HSTU_ERR_WORKSPACE;
  Ctx c = make_ctx(*desc, ws, stream);
  const size_t f1_bytes = (size_t)T * c.F * c.es;
  auto f1_of = [&](int l) { return at<void>(ws, L.f1_cache + (size_t)l * f1_bytes); };

  // ---- history pass: every layer's f1 output (and so its K/V) is kept
  launch_schedule(hist_offsets, B, T, max_len, desc->n_heads, at<AttnItem>(ws, L.items),
                  L.item_cap, at<int64_t>(ws, L.ubase), L.tile_cap, c.hdr, c.s);
  cudaError_t e = convert_weights(c, weights, n_layers, L, ws);
  float* xres = at<float>(ws, L.xres);
  void* xh = at<void>(ws, L.xh);
  if (T > 0 && e == cudaSuccess) {
    launch_time_rel(hist_offsets, B, max_len, hist_timestamps, T, at<int32_t>(ws, L.t_rel), c.hdr,
                    c.s);
    if (c.bf16 && n_layers > 1)
      launch_time_buckets(hist_offsets, B, max_len, at<int32_t>(ws, L.t_rel),
                          at<int64_t>(ws, L.ubase),
                          L.tile_cap, desc->time_sub_bits, desc->n_time_buckets,
                          at<uint32_t>(ws, L.tbuckets), c.hdr, c.s);
    for (int l = 0; l < n_layers && e == cudaSuccess; ++l) {
      const bool first = l == 0;
      const LayerOps ops = layer_ops(c, weights[l], L, ws, l, n_layers);
      const void* A = first ? history : (c.bf16 ? xh : (const void*)xres);
      if (l == n_layers - 1) {  // the last layer's history rows only serve as K and V
        e = run_f1(c, weights[l], ops, A, first ? 0 : 1, T, nullptr, f1_of(l), true);
        break;
      }
      e = run_layer(c, weights[l], ops, B, T, hist_offsets, A, first ? 0 : 1,
                    first ? history : (c.bf16 ? xh : (const void*)xres),
                    first ? RESID_BF16 : RESID_F16, c.bf16 ? xh : nullptr, false,
                    c.bf16 ? nullptr : xres, f1_of(l), L, ws);
    }
  }
  if (e != cudaSuccess || total_cands == 0) return finish(e);

  // ---- candidates, one microbatch of up to `microbatch` per user at a time
  const int64_t R = L.mb_cap;
  const int64_t* rows_dev = &c.hdr->mb_rows;
  int64_t* mb_off = at<int64_t>(ws, L.mb_off);
  AttnItem* citems = at<AttnItem>(ws, L.c_items);
  int32_t* t_req_rel = at<int32_t>(ws, L.t_req_rel);
  float* xres_c = at<float>(ws, L.xres_c);
  void* xb_c = at<void>(ws, L.xb_c);   // gathered candidate rows (caller dtype)
  void* xh_c = at<void>(ws, L.xh_c);   // fp16 copy of the stream (tensor-core path)
  void* f1c = at<void>(ws, L.f1c);
  void* oc = at<void>(ws, L.oc);
  void* zc = at<void>(ws, L.zc);
  const int n_mb = (int)((max_cands + microbatch - 1) / microbatch);
  for (int k = 0; k < n_mb && e == cudaSuccess; ++k) {
    launch_mb_plan(hist_offsets, cand_offsets, B, max_len, max_cands, k, microbatch,
                   desc->n_heads, hist_timestamps, request_ts, mb_off, citems, L.cand_item_cap,
                   t_req_rel, c.hdr, c.s);
    e = launch_mb_gather(desc->dtype, candidates, desc->d_model, cand_offsets, mb_off, B, k,
                         microbatch, xb_c, R, rows_dev, c.status, c.s);
    for (int l = 0; l < n_layers && e == cudaSuccess; ++l) {
      const bool first = l == 0, last = l == n_layers - 1;
      const LayerOps ops = layer_ops(c, weights[l], L, ws, l, n_layers);
      const void* A = first ? xb_c : (c.bf16 ? xh_c : (const void*)xres_c);
      e = run_f1(c, weights[l], ops, A, first ? 0 : 1, R, rows_dev, f1c, false);
      if (e != cudaSuccess) break;
      AttnCall a = attn_common(c, weights[l], B);
      a.mode = 1;
      a.items = citems;
      a.n_items = &c.hdr->n_cand_items;
      a.item_cap = L.cand_item_cap;
      a.q_off = mb_off;
      a.kv_off = hist_offsets;
      a.q_rows_dev = rows_dev;
      a.q_buf = f1c;
      a.q_rows_cap = R;
      a.kv_buf = f1_of(l);
      a.kv_rows_cap = T;
      a.t_rel = at<int32_t>(ws, L.t_rel);
      a.t_req_rel = t_req_rel;
      a.O = oc;
      a.ostats = c.bf16 ? at<float>(ws, L.ostats_c) : nullptr;
      e = attn(c, a);
      if (e != cudaSuccess) break;
      const void* resid = first ? xb_c : (const void*)xres_c;
      void* o16 = (c.bf16 && !last) ? xh_c : nullptr;
      if (c.bf16 && ln_fusion_for(c.d.d_model)) {  // LayerNorm * U inside f2's operand stage
        e = run_f2(c, weights[l], ops, oc, at<float>(ws, L.ostats_c),
                   at<uint32_t>(ws, L.lncoef_c), f1c, nullptr, resid,
                   first ? RESID_BF16 : RESID_F32, R, rows_dev, o16, false, xres_c);
        continue;
      }
      if (c.bf16)
        e = launch_ln_gate_norm(oc, at<float>(ws, L.ostats_c), f1c, c.F, weights[l].ln_gamma,
                                weights[l].ln_beta, desc->ln_eps, zc, c.hdv, desc->n_heads,
                                desc->d_v, R, rows_dev, c.status, c.s);
      else
        e = launch_ln_gate(desc->dtype, oc, f1c, c.F, weights[l].ln_gamma, weights[l].ln_beta,
                           desc->ln_eps, zc, c.hdv, R, rows_dev, c.status, c.s);
      if (e != cudaSuccess) break;
      e = run_f2(c, weights[l], ops, zc, nullptr, nullptr, nullptr, nullptr, resid,
                 first ? RESID_BF16 : RESID_F32, R, rows_dev, o16, false, xres_c);
    }
    if (e == cudaSuccess)
      e = launch_score(desc->dtype, xres_c, desc->d_model, head_vec, cand_offsets, mb_off, B, k,
                       microbatch, scores, R, rows_dev, c.status, c.s);
  }
  return finish(e);
}

hstu_status hstu_bf16_to_f16(const void* src, void* dst, int64_t n, void* stream) {
  if (n < 0 || n % 8 != 0) return HSTU_ERR_INVALID_ARG;
  if (n == 0) return HSTU_OK;
  if (!src || !dst || !al16(src) || !al16(dst)) return HSTU_ERR_INVALID_ARG;
  ConvBatch cb{};
  cb.seg[cb.n++] = ConvSeg{src, dst, n};
  return launch_bf16_to_f16(cb, static_cast<cudaStream_t>(stream)) == cudaSuccess ? HSTU_OK
                                                                                  : HSTU_ERR_CUDA;
}

hstu_status hstu_read_status(const void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < sizeof(Header)) return HSTU_ERR_INVALID_ARG;
  int32_t st = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
  return static_cast<hstu_status>(st);
}

hstu_status hstu_debug_offsets(const hstu_layer_desc* desc, int64_t B, int64_t total_tokens,
                               int64_t max_len, size_t* f1_offset, size_t* o_offset,
                               size_t* z_offset) {
  hstu_status st = check_desc(desc);
  if (st != HSTU_OK) return st;
  if ((st = check_sizes(B, total_tokens, max_len)) != HSTU_OK) return st;
  Layout L;
  if (!make_layout(*desc, 1, B, total_tokens, max_len, 0, 0, 0, &L)) return HSTU_ERR_INVALID_ARG;
  if (f1_offset) *f1_offset = L.f1;
  if (o_offset) *o_offset = L.o;
  if (z_offset) *z_offset = L.z;
  return HSTU_OK;
}

const char* hstu_status_string(hstu_status s) {
  switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARG: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case HSTU_ERR_WORKSPACE: return "workspace too small";
    case HSTU_ERR_CUDA: return "CUDA runtime error";
    case HSTU_ERR_BAD_OFFSETS: return "bad offsets (device check)";
    case HSTU_ERR_TIMEOUT: return "in-kernel wait timed out (device check)";
    case HSTU_ERR_BAD_TIMESTAMPS: return "timestamps span 2^30 s or more within a user (device check)";
    case HSTU_ERR_BAD_IDS: return "a token id outside its embedding table (device check)";
  }
  return "unknown status";
}

int32_t hstu_version(void) { return 1; }

}  // extern "C"

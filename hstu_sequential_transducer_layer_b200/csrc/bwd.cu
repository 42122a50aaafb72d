// bwd.cu — backward pass (gradients for training) of the HSTU layer stack:
// the row-wise LayerNorm * U backward, reductions, conversions, and the C ABI
// entry points hstu_layer_bwd / hstu_stack_bwd that sequence them with the
// tensor-core GEMMs (gemm_tc.cu) and the attention backward (attn_bwd.cu).
//
// 'HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか'
// defines the forward layer; its gradients are the chain rule through it in
// reverse order (section '長い履歴を現実の計算量へ収める4つの工夫' notes that
// training keeps only a few activations per layer; here the backward
// recomputes each layer's forward from the layer's input):
//   Y = X + Z W2^T + b2      dZ = dY W2, dW2 = dY^T Z, db2 = sum dY, dX = dY + ...
//   Z = L * U, L = LN(O) g + be
//                            dL = dZ * U, dU = dZ * L, dg = sum dL xhat, dbe = sum dL,
//                            dO = (dxh - mean dxh - xhat mean(dxh xhat)) / sd, dxh = dL g
//   O = (1/n) SiLU(S) V ...  (attn_bwd.cu)
//   G = SiLU(P), P = X W1^T + b1
//                            dP = dG * SiLU'(P), dW1 = dP^T X, db1 = sum dP, dX += dP W1
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>

#include "ptx.cuh"

namespace hstu {

namespace {
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
constexpr int kLnBwdMaxPairs = 32;   // h*d_v <= 2048: 64 features per lane
constexpr int kSumThreads = 256;
constexpr int kGradSplits = 8;       // split-K of the weight-gradient products
constexpr int kLnBwdBlocks = 1184;   // LayerNorm backward blocks (8 per SM)
}  // namespace

// ---------------------------------------------------------------- LayerNorm * U backward
// One warp per row.  O arrives as the attention kernel stores it, normalised
// per (row, head): O = m + s * xn.  Per row: mu, rstd over all h*d_v features;
// xhat = (O - mu) rstd; L = xhat g + be; Z = L U (stored for dW2);
// dL = dZ U; dU = dZ L, stored as dP_U = dU SiLU'(P_U) into the f1-shaped
// gradient; dxh = dL g; dO = (dxh - mean dxh - xhat mean(dxh xhat)) rstd.
// Column partial sums of dL xhat (dg) and dL (dbe) accumulate per warp in
// shared memory (each lane owns its features: no atomics, a fixed order) and
// are summed over the block's warps in warp order into one row per block.
__global__ void __launch_bounds__(256)
    k_ln_bwd(const float* __restrict__ dZ, const __half* __restrict__ xn,
             const float2* __restrict__ stats, const __half* __restrict__ f1,
             const __half* __restrict__ pre, int64_t ld_f1, const __nv_bfloat16* __restrict__ gamma,
             const __nv_bfloat16* __restrict__ beta, float eps, int hdv, int h, int dv,
             int64_t rows, int64_t rows_per_block, __half* __restrict__ Z,
             __half* __restrict__ dO, __half* __restrict__ dP, float* __restrict__ part,
             const int* __restrict__ status) {
  extern __shared__ float s_acc_all[];  // [warps][2][hdv]: dg, dbe partials per warp
  if (status && *status != HSTU_OK) return;
  for (int i = threadIdx.x; i < 2 * hdv * (int)(blockDim.x / 32); i += blockDim.x) s_acc_all[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float* s_acc = s_acc_all + (size_t)wid * 2 * hdv;
  const int npair = hdv / 64;  // feature pairs per lane: features 2 lane + 64 j
  const int64_t r_begin = blockIdx.x * rows_per_block;
  const int64_t r_end = min(rows, r_begin + rows_per_block);
  for (int64_t row = r_begin + wid; row < r_end; row += blockDim.x / 32) {
    const float2* st = stats + row * h;
    // row moments from the heads' (m, s): mu = mean m, var = mean (s^2 + (m - mu)^2)
    float sm = 0.f;
    for (int hh = lane; hh < h; hh += 32) sm += st[hh].x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
    const float mu = sm / (float)h;
    float sv = 0.f;
    for (int hh = lane; hh < h; hh += 32) {
      const float2 v = st[hh];
      const float dm = v.x - mu;
      sv = fmaf(v.y, v.y, fmaf(dm, dm, sv));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
    const float rstd = rsqrtf(sv / (float)h + eps);
    float xh[2 * kLnBwdMaxPairs], dx[2 * kLnBwdMaxPairs];
    float s_dx = 0.f, s_dxx = 0.f;
#pragma unroll
    for (int j = 0; j < kLnBwdMaxPairs; ++j) {
      if (j < npair) {
        const int k = 2 * lane + 64 * j;
        const float2 hs = st[k / dv];
        const __half2 xv = *reinterpret_cast<const __half2*>(xn + row * hdv + k);
        const __half2 uv = *reinterpret_cast<const __half2*>(f1 + row * ld_f1 + k);
        const __half2 pv = *reinterpret_cast<const __half2*>(pre + row * ld_f1 + k);
        const float2 dz = *reinterpret_cast<const float2*>(dZ + row * hdv + k);
        const __nv_bfloat162 gv = *reinterpret_cast<const __nv_bfloat162*>(gamma + k);
        const __nv_bfloat162 bv = *reinterpret_cast<const __nv_bfloat162*>(beta + k);
        const float x0 = (hs.x + hs.y * __low2float(xv) - mu) * rstd;
        const float x1 = (hs.x + hs.y * __high2float(xv) - mu) * rstd;
        const float g0 = __low2float(gv), g1 = __high2float(gv);
        const float l0 = fmaf(x0, g0, __low2float(bv)), l1 = fmaf(x1, g1, __high2float(bv));
        const float u0 = __low2float(uv), u1 = __high2float(uv);
        *reinterpret_cast<__half2*>(Z + row * hdv + k) = __floats2half2_rn(l0 * u0, l1 * u1);
        const float dl0 = dz.x * u0, dl1 = dz.y * u1;
        // dP_U = dU * SiLU'(P_U), dU = dZ * L
        const float p0 = __low2float(pv), p1 = __high2float(pv);
        const float sg0 = __fdividef(1.0f, 1.0f + __expf(-p0));
        const float sg1 = __fdividef(1.0f, 1.0f + __expf(-p1));
        const float dp0 = dz.x * l0 * sg0 * fmaf(p0, 1.0f - sg0, 1.0f);
        const float dp1 = dz.y * l1 * sg1 * fmaf(p1, 1.0f - sg1, 1.0f);
        *reinterpret_cast<uint32_t*>(dP + row * ld_f1 + k) = pack_f16x2_sat(dp0, dp1);
        s_acc[k] += dl0 * x0;
        s_acc[k + 1] += dl1 * x1;
        s_acc[hdv + k] += dl0;
        s_acc[hdv + k + 1] += dl1;
        xh[2 * j] = x0;
        xh[2 * j + 1] = x1;
        dx[2 * j] = dl0 * g0;
        dx[2 * j + 1] = dl1 * g1;
        s_dx += dx[2 * j] + dx[2 * j + 1];
        s_dxx += dx[2 * j] * x0 + dx[2 * j + 1] * x1;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s_dx += __shfl_xor_sync(0xffffffffu, s_dx, o);
      s_dxx += __shfl_xor_sync(0xffffffffu, s_dxx, o);
    }
    const float m_dx = s_dx / (float)hdv, m_dxx = s_dxx / (float)hdv;
#pragma unroll
    for (int j = 0; j < kLnBwdMaxPairs; ++j) {
      if (j < npair) {
        const int k = 2 * lane + 64 * j;
        const float o0 = (dx[2 * j] - m_dx - xh[2 * j] * m_dxx) * rstd;
        const float o1 = (dx[2 * j + 1] - m_dx - xh[2 * j + 1] * m_dxx) * rstd;
        *reinterpret_cast<uint32_t*>(dO + row * hdv + k) = pack_f16x2_sat(o0, o1);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * hdv; i += blockDim.x) {
    float acc = 0.f;
    for (int wv = 0; wv < (int)(blockDim.x / 32); ++wv) acc += s_acc_all[(size_t)wv * 2 * hdv + i];
    part[blockIdx.x * (int64_t)2 * hdv + i] = acc;
  }
}

// ---------------------------------------------------------------- reductions
// part[blockIdx.y, n] = sum over rows [y * rows_per_block, ...) of in[r, n]
// (fp32 or fp16 input, row stride ld).
template <typename T>
__global__ void __launch_bounds__(kSumThreads)
    k_sum_rows(const T* __restrict__ in, int64_t rows, int64_t N, int64_t ld,
               int64_t rows_per_block, float* __restrict__ part, const int* __restrict__ status) {
  if (status && *status != HSTU_OK) return;
  const int64_t n = blockIdx.x * (int64_t)kSumThreads + threadIdx.x;
  if (n >= N) return;
  const int64_t r0 = blockIdx.y * rows_per_block;
  const int64_t r1 = min(rows, r0 + rows_per_block);
  float acc = 0.f;
  for (int64_t r = r0; r < r1; ++r) acc += (float)in[r * ld + n];
  part[blockIdx.y * N + n] = acc;
}

// out[x] = sum_{s < S} in[s * stride + x], x < L.
__global__ void __launch_bounds__(kSumThreads)
    k_sum_slices(const float* __restrict__ in, int S, int64_t stride, int64_t L,
                 float* __restrict__ out, const int* __restrict__ status) {
  if (status && *status != HSTU_OK) return;
  for (int64_t x = blockIdx.x * (int64_t)kSumThreads + threadIdx.x; x < L;
       x += (int64_t)gridDim.x * kSumThreads) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += in[s * stride + x];
    out[x] = acc;
  }
}

// dst = src converted: fp32 or bf16 source (src_bf16), fp32 and/or fp16
// destinations (either may be null).  n elements, a multiple of 4.
__global__ void k_convert(const void* __restrict__ src, int src_bf16, float* __restrict__ d32,
                          __half* __restrict__ d16, int64_t n, const int* __restrict__ status) {
  if (status && *status != HSTU_OK) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n / 4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v[4];
    if (src_bf16) {
      const uint2 w = reinterpret_cast<const uint2*>(src)[i];
      v[0] = bf16lo(w.x);
      v[1] = bf16hi(w.x);
      v[2] = bf16lo(w.y);
      v[3] = bf16hi(w.y);
    } else {
      const float4 w = reinterpret_cast<const float4*>(src)[i];
      v[0] = w.x;
      v[1] = w.y;
      v[2] = w.z;
      v[3] = w.w;
    }
    if (d32) reinterpret_cast<float4*>(d32)[i] = make_float4(v[0], v[1], v[2], v[3]);
    if (d16)
      reinterpret_cast<uint2*>(d16)[i] = make_uint2(pack_f16x2_sat(v[0], v[1]), pack_f16x2_sat(v[2], v[3]));
  }
}

namespace {

int grid_for(int64_t n, int per) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((n + per - 1) / per, 4 * num_sms()));
}

cudaError_t convert(const void* src, int src_bf16, float* d32, __half* d16, int64_t n,
                    const int* status, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  LaunchScope ls(K_F32_TO_F16, s);
  k_convert<<<grid_for(n / 4, 256), 256, 0, s>>>(src, src_bf16, d32, d16, n, status);
  return cudaGetLastError();
}

// out[n] = sum over rows of in[r, n] (rows x N, row stride ld), via per-block
// partials in `part` (at least 256 * N floats).
template <typename T>
cudaError_t sum_rows(const T* in, int64_t rows, int64_t N, int64_t ld, float* part, float* out,
                     const int* status, cudaStream_t s) {
  const int nb = (int)std::max<int64_t>(1, std::min<int64_t>(256, (rows + 127) / 128));
  const int64_t rpb = (rows + nb - 1) / nb;
  {
    LaunchScope ls(K_SUM_ROWS, s);
    k_sum_rows<T><<<dim3((unsigned)((N + kSumThreads - 1) / kSumThreads), nb), kSumThreads, 0, s>>>(
        in, rows, N, ld, rpb, part, status);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  LaunchScope ls(K_SUM_ROWS, s);
  k_sum_slices<<<grid_for(N, kSumThreads), kSumThreads, 0, s>>>(part, nb, N, N, out, status);
  return cudaGetLastError();
}

struct BwdLayout {
  size_t header, items, t_rel, ubase, tbuckets;
  size_t xs;        // the layers' inputs, fp16, [n_layers][T, d]
  size_t g, pre;    // f1 output and pre-activation, fp16 [T, F]
  size_t o;         // normalised attention output fp16 [T, hdv] + (m, s) [T, h]
  size_t z, dz, dO, dP;
  size_t gy0, gy1;  // fp32 gradient streams [T, d]
  size_t gyh;       // fp16 copy of the current one
  size_t w16;       // fp16 copies of W1 and W2, per layer
  size_t part;      // partial sums
  size_t zbias;     // bf16 zeros
  size_t total;
  int64_t item_cap, tile_cap, part_floats;
};

bool make_bwd_layout(const hstu_layer_desc& d, int L, int64_t B, int64_t T, int64_t max_len,
                     BwdLayout* o) {
  if (B < 0 || T < 0 || L < 1) return false;
  const size_t F = 2 * (size_t)d.n_heads * (d.d_v + d.d_qk);
  const size_t hdv = (size_t)d.n_heads * d.d_v, dm = (size_t)d.d_model;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t r = off;
    off += up256(bytes);
    return r;
  };
  *o = BwdLayout{};
  o->item_cap = ((T + kTile - 1) / kTile + B) * (int64_t)d.n_heads;
  const int64_t max_q = (max_len + kTile - 1) / kTile;
  o->tile_cap = ((T + kTile - 1) / kTile + B) * (max_q + 1) / 2 + 1;
  o->header = take(256);
  o->items = take((size_t)o->item_cap * sizeof(AttnItem));
  o->t_rel = take((size_t)T * 4);
  o->ubase = take((size_t)(B + 1) * 8);
  o->tbuckets = take((size_t)o->tile_cap * kBucketTileWords * 4);
  o->xs = take((size_t)L * T * dm * 2);
  o->g = take((size_t)T * F * 2);
  o->pre = take((size_t)T * F * 2);
  o->o = take(up256((size_t)T * hdv * 2) + (size_t)T * d.n_heads * 8);
  o->z = take((size_t)T * hdv * 2);
  o->dz = take((size_t)T * hdv * 4);
  o->dO = take((size_t)T * hdv * 2);
  o->dP = take((size_t)T * F * 2);
  o->gy0 = take((size_t)T * dm * 4);
  o->gy1 = take((size_t)T * dm * 4);
  o->gyh = take((size_t)T * dm * 2);
  o->w16 = take((size_t)L * (F * dm + dm * hdv) * 2);
  const size_t F_pad = (F + 127) / 128 * 128, d_pad = (dm + 127) / 128 * 128;
  const size_t part = std::max<size_t>({(size_t)kGradSplits * std::max(F_pad * dm, d_pad * hdv),
                                        (size_t)kLnBwdBlocks * 2 * hdv,
                                        (size_t)256 * std::max({F, hdv, dm})});
  o->part_floats = (int64_t)part;
  o->part = take(part * 4);
  o->zbias = take(std::max({F, hdv, dm}) * 2 + 1024);
  o->total = off;
  return true;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hstu_status check_bwd_desc(const hstu_layer_desc* d) {
  if (!d) return HSTU_ERR_INVALID_ARG;
  if (d->dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (d->d_model <= 0 || d->n_heads <= 0 || d->d_qk != d->d_v) return HSTU_ERR_UNSUPPORTED;
  if (d->d_qk != 64 && d->d_qk != 128) return HSTU_ERR_UNSUPPORTED;
  if (d->d_model % 64 != 0 || (int64_t)d->n_heads * d->d_v > 2048) return HSTU_ERR_UNSUPPORTED;
  if (d->n_pos_buckets < 1 || d->n_pos_buckets > 4096 || d->n_time_buckets < 1 ||
      d->n_time_buckets > 256)
    return HSTU_ERR_UNSUPPORTED;
  if (d->pos_sub_bits < 0 || d->pos_sub_bits > 20 || d->time_sub_bits < 0 || d->time_sub_bits > 20)
    return HSTU_ERR_INVALID_ARG;
  if (!(d->ln_eps >= 0.f) || !std::isfinite(d->ln_eps)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status stack_bwd_impl(const hstu_layer_desc* desc, int32_t L, const hstu_layer_weights* W,
                           int64_t B, int64_t T, int64_t max_len, const int64_t* offsets,
                           const void* X, const int64_t* timestamps, const void* dY, void* dX,
                           const hstu_layer_grads* grads, void* ws, size_t ws_bytes,
                           void* stream) {
  hstu_status st = check_bwd_desc(desc);
  if (st != HSTU_OK) return st;
  if (L < 1 || !W || !grads) return HSTU_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || max_len < 1 || max_len > (1ll << 30) || T > B * max_len)
    return HSTU_ERR_INVALID_ARG;
  if (T > (1ll << 31) - 1024) return HSTU_ERR_UNSUPPORTED;
  if (!offsets || !al16(offsets) || !ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (!X || !dY || !dX || !timestamps || !al16(X) || !al16(dY) || !al16(dX) ||
                !al16(timestamps)))
    return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    const hstu_layer_weights& w = W[l];
    const void* p[8] = {w.W1, w.b1, w.W2, w.b2, w.ln_gamma, w.ln_beta, w.rab_pos, w.rab_time};
    for (const void* q : p)
      if (!q || !al16(q)) return HSTU_ERR_INVALID_ARG;
    const hstu_layer_grads& g = grads[l];
    const void* gp[8] = {g.dW1, g.db1, g.dW2, g.db2, g.dln_gamma, g.dln_beta, g.drab_pos,
                         g.drab_time};
    for (const void* q : gp)
      if (!q || !al16(q)) return HSTU_ERR_INVALID_ARG;
  }
  BwdLayout Lo;
  if (!make_bwd_layout(*desc, L, B, T, max_len, &Lo)) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < Lo.total) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const hstu_layer_desc& d = *desc;
  const int h = d.n_heads, dm = d.d_model;
  const int hdv = h * d.d_v, F = 2 * hdv + 2 * h * d.d_qk;
  const int vcol = hdv, qcol = 2 * hdv, kcol = 2 * hdv + h * d.d_qk;
  Header* hdr = at<Header>(ws, Lo.header);
  int* status = &hdr->status;
  float* part = at<float>(ws, Lo.part);
  cudaError_t e = cudaSuccess;
  const char* where = "setup";   // the step that failed, for hstu_last_error
  auto ok = [&]() { return e == cudaSuccess; };
  // gradients of tables and sums start at zero (the attention backward adds)
  for (int l = 0; l < L && ok(); ++l) {
    e = cudaMemsetAsync(grads[l].drab_pos, 0, (size_t)h * d.n_pos_buckets * 4, s);
    if (ok()) e = cudaMemsetAsync(grads[l].drab_time, 0, (size_t)h * d.n_time_buckets * 4, s);
  }
  if (ok()) e = cudaMemsetAsync(at<void>(ws, Lo.zbias), 0, std::max({F, hdv, dm}) * 2 + 1024, s);
  if (!ok()) {
    note_cuda_error(e, where);
    return HSTU_ERR_CUDA;
  }
  launch_schedule(offsets, B, T, max_len, h, at<AttnItem>(ws, Lo.items), Lo.item_cap,
                  at<int64_t>(ws, Lo.ubase), Lo.tile_cap, hdr, s);
  if (T == 0) {
    // no rows: every weight gradient is zero
    for (int l = 0; l < L && ok(); ++l) {
      const hstu_layer_grads& g = grads[l];
      e = cudaMemsetAsync(g.dW1, 0, (size_t)F * dm * 4, s);
      if (ok()) e = cudaMemsetAsync(g.db1, 0, (size_t)F * 4, s);
      if (ok()) e = cudaMemsetAsync(g.dW2, 0, (size_t)dm * hdv * 4, s);
      if (ok()) e = cudaMemsetAsync(g.db2, 0, (size_t)dm * 4, s);
      if (ok()) e = cudaMemsetAsync(g.dln_gamma, 0, (size_t)hdv * 4, s);
      if (ok()) e = cudaMemsetAsync(g.dln_beta, 0, (size_t)hdv * 4, s);
    }
    if (!ok()) note_cuda_error(e, "zero gradients");
    return ok() ? HSTU_OK : HSTU_ERR_CUDA;
  }
  launch_time_rel(offsets, B, timestamps, T, at<int32_t>(ws, Lo.t_rel), hdr, s);
  launch_time_buckets(offsets, B, at<int32_t>(ws, Lo.t_rel), at<int64_t>(ws, Lo.ubase),
                      Lo.tile_cap, d.time_sub_bits, d.n_time_buckets, at<uint32_t>(ws, Lo.tbuckets),
                      hdr, s);
  // fp16 copies of every layer's W1 and W2
  {
    ConvBatch cb{};
    for (int l = 0; l < L && ok(); ++l) {
      uint8_t* base = at<uint8_t>(ws, Lo.w16) + (size_t)l * ((size_t)F * dm + (size_t)dm * hdv) * 2;
      cb.seg[cb.n++] = ConvSeg{W[l].W1, base, (int64_t)F * dm};
      cb.seg[cb.n++] = ConvSeg{W[l].W2, base + (size_t)F * dm * 2, (int64_t)dm * hdv};
      if (cb.n > kMaxConvSegs - 2 || l == L - 1) {
        e = launch_bf16_to_f16(cb, s);
        cb.n = 0;
      }
    }
  }
  auto w1h = [&](int l) {
    return at<__half>(ws, Lo.w16) + (size_t)l * ((size_t)F * dm + (size_t)dm * hdv);
  };
  auto w2h = [&](int l) { return w1h(l) + (size_t)F * dm; };
  auto xs = [&](int l) { return at<__half>(ws, Lo.xs) + (size_t)l * T * dm; };
  void* g_buf = at<void>(ws, Lo.g);
  void* pre_buf = at<void>(ws, Lo.pre);
  void* o_buf = at<void>(ws, Lo.o);
  float* ostats = at<float>(ws, Lo.o + up256((size_t)T * hdv * 2));

  // f1 (with its pre-activation) and the attention of layer l, from xs(l)
  auto forward_parts = [&](int l) {
    GemmCall gc{};
    gc.A = xs(l);
    gc.lda = dm;
    gc.W = w1h(l);
    gc.ldw = dm;
    gc.ab_f16 = 1;
    gc.M_cap = T;
    gc.N = F;
    gc.K = dm;
    gc.bias = W[l].b1;
    gc.out = g_buf;
    gc.out_f16 = 1;
    gc.out_pre = pre_buf;
    gc.ldo = F;
    gc.epi = EPI_SILU;
    gc.status = status;
    where = "f1 recompute";
    e = launch_gemm_tc(gc, s, K_GEMM_F1);
    if (!ok()) return;
    AttnCall ac{};
    ac.mode = 0;
    ac.B = B;
    ac.items = at<AttnItem>(ws, Lo.items);
    ac.n_items = &hdr->n_items;
    ac.item_cap = Lo.item_cap;
    ac.q_off = offsets;
    ac.kv_off = offsets;
    ac.q_buf = g_buf;
    ac.q_rows_cap = T;
    ac.kv_buf = g_buf;
    ac.kv_rows_cap = T;
    ac.ld_f1 = F;
    ac.q_col = qcol;
    ac.k_col = kcol;
    ac.v_col = vcol;
    ac.t_rel = at<int32_t>(ws, Lo.t_rel);
    ac.tbuckets = at<uint32_t>(ws, Lo.tbuckets);
    ac.work_next = &hdr->work_next;
    ac.work_done = &hdr->work_done;
    ac.rab_pos = W[l].rab_pos;
    ac.rab_time = W[l].rab_time;
    ac.Np = d.n_pos_buckets;
    ac.Nt = d.n_time_buckets;
    ac.Sp = d.pos_sub_bits;
    ac.St = d.time_sub_bits;
    ac.h = h;
    ac.dqk = d.d_qk;
    ac.dv = d.d_v;
    ac.O = o_buf;
    ac.ldo = hdv;
    ac.ostats = ostats;
    ac.status = status;
    where = "attention recompute";
    e = launch_attn_tc(ac, s);
  };

  // ---- forward through layers 0..L-2, keeping every layer's input (fp16)
  e = convert(X, 1, nullptr, xs(0), (int64_t)T * dm, status, s);
  for (int l = 0; l + 1 < L && ok(); ++l) {
    forward_parts(l);
    if (!ok()) break;
    GemmCall gc{};
    if (ln_fusion()) {  // LayerNorm * U inside f2's operand stage
      gc.A = nullptr;
      gc.ln_x = o_buf;
      gc.ln_stats = ostats;
      gc.ln_u = g_buf;
      gc.ld_u = F;
      gc.ln_gamma = W[l].ln_gamma;
      gc.ln_beta = W[l].ln_beta;
      gc.ln_eps = d.ln_eps;
      gc.ln_h = h;
      gc.ln_dv = d.d_v;
    } else {
      where = "LayerNorm * U (forward of the stack)";
      e = launch_ln_gate_norm(o_buf, ostats, g_buf, F, W[l].ln_gamma, W[l].ln_beta, d.ln_eps,
                              at<void>(ws, Lo.z), hdv, h, d.d_v, T, nullptr, status, s);
      if (!ok()) break;
      gc.A = at<void>(ws, Lo.z);
    }
    gc.lda = hdv;
    gc.W = w2h(l);
    gc.ldw = hdv;
    gc.ab_f16 = 1;
    gc.M_cap = T;
    gc.N = dm;
    gc.K = hdv;
    gc.bias = W[l].b2;
    gc.ldo = dm;
    gc.resid = xs(l);
    gc.ldr = dm;
    gc.resid_kind = RESID_F16;
    gc.out = xs(l + 1);
    gc.out_f16 = 1;
    gc.epi = EPI_RESID;
    gc.status = status;
    where = "f2 (forward of the stack)";
    e = launch_gemm_tc(gc, s, K_GEMM_F2);
  }

  // ---- backward, last layer first; gy = gradient of the current layer's output
  float* gy = at<float>(ws, Lo.gy0);
  float* gx = at<float>(ws, Lo.gy1);
  __half* gyh = at<__half>(ws, Lo.gyh);
  if (ok()) e = convert(dY, 1, gy, gyh, (int64_t)T * dm, status, s);
  const int64_t F_pad = (F + 127) / 128 * 128, d_pad = (dm + 127) / 128 * 128;
  for (int l = L - 1; l >= 0 && ok(); --l) {
    const hstu_layer_grads& gr = grads[l];
    forward_parts(l);
    if (!ok()) break;
    if (l < L - 1) e = convert(gy, 0, nullptr, gyh, (int64_t)T * dm, status, s);
    // dZ = dY W2
    GradGemm gg{};
    gg.A = gyh;
    gg.lda = dm;
    gg.W = w2h(l);
    gg.ldw = hdv;
    gg.w_mn = 1;
    gg.ab_f16 = 1;
    gg.M = T;
    gg.N = hdv;
    gg.K = dm;
    gg.splits = 1;
    gg.out = at<float>(ws, Lo.dz);
    gg.ldo = hdv;
    gg.status = status;
    where = "dZ = dY W2";
    if (ok()) e = launch_gemm_grad(gg, s, K_GEMM_BWD);
    // LayerNorm * U backward: Z, dO, dP_U, and the dg / dbe partials
    if (ok()) {
      // many short row ranges: each warp has few rows, so more loads are in flight
      const int nb = (int)std::max<int64_t>(1, std::min<int64_t>(kLnBwdBlocks, (T + 31) / 32));
      const int64_t rpb = (T + nb - 1) / nb;
      where = "LayerNorm backward";
      LaunchScope ls(K_LN_BWD, s);
      const int ln_smem = 8 * 2 * hdv * 4;  // 8 warps x (dg, dbe) partials
      e = ensure_smem_limit(reinterpret_cast<const void*>(k_ln_bwd), ln_smem);
      if (!ok()) break;
      k_ln_bwd<<<nb, 256, ln_smem, s>>>(
          at<float>(ws, Lo.dz), static_cast<const __half*>(o_buf),
          reinterpret_cast<const float2*>(ostats), static_cast<const __half*>(g_buf),
          static_cast<const __half*>(pre_buf), F, static_cast<const __nv_bfloat16*>(W[l].ln_gamma),
          static_cast<const __nv_bfloat16*>(W[l].ln_beta), d.ln_eps, hdv, h, d.d_v, T, rpb,
          at<__half>(ws, Lo.z), at<__half>(ws, Lo.dO), at<__half>(ws, Lo.dP), part, status);
      e = cudaGetLastError();
      if (ok()) {
        LaunchScope ls2(K_SUM_ROWS, s);
        k_sum_slices<<<grid_for(hdv, kSumThreads), kSumThreads, 0, s>>>(part, nb, 2 * hdv, hdv,
                                                                         gr.dln_gamma, status);
        k_sum_slices<<<grid_for(hdv, kSumThreads), kSumThreads, 0, s>>>(part + hdv, nb, 2 * hdv,
                                                                         hdv, gr.dln_beta, status);
        e = cudaGetLastError();
      }
    }
    // dW2 = dY^T Z (split over the rows), db2 = sum of dY
    if (ok()) {
      GradGemm gw{};
      gw.A = gyh;
      gw.lda = dm;
      gw.a_mn = 1;
      where = "dW2";
      gw.W = at<void>(ws, Lo.z);
      gw.ldw = hdv;
      gw.w_mn = 1;
      gw.ab_f16 = 1;
      gw.M = dm;
      gw.N = hdv;
      gw.K = T;
      gw.splits = kGradSplits;
      gw.split_rows = d_pad;
      gw.out = part;
      gw.ldo = hdv;
      gw.status = status;
      int used = 1;
      gw.splits_used = &used;
      e = launch_gemm_grad(gw, s, K_GEMM_BWD);
      if (ok()) {
        LaunchScope ls(K_SUM_ROWS, s);
        k_sum_slices<<<grid_for((int64_t)dm * hdv, kSumThreads), kSumThreads, 0, s>>>(
            part, used, d_pad * hdv, (int64_t)dm * hdv, gr.dW2, status);
        e = cudaGetLastError();
      }
    }
    if (ok()) e = sum_rows<float>(gy, T, dm, dm, part, gr.db2, status, s);
    // attention backward: dP of the V, K and Q columns, and the bias tables
    if (ok()) {
      AttnBwdCall bc{};
      bc.items = at<AttnItem>(ws, Lo.items);
      bc.n_items = &hdr->n_items;
      bc.item_cap = Lo.item_cap;
      bc.f1 = g_buf;
      bc.pre = pre_buf;
      bc.dP = at<void>(ws, Lo.dP);
      bc.ld_f1 = F;
      bc.rows = T;
      bc.dO = at<void>(ws, Lo.dO);
      bc.ld_do = hdv;
      bc.q_col = qcol;
      bc.k_col = kcol;
      bc.v_col = vcol;
      bc.t_rel = at<int32_t>(ws, Lo.t_rel);
      bc.rab_pos = W[l].rab_pos;
      bc.rab_time = W[l].rab_time;
      bc.drab_pos = gr.drab_pos;
      bc.drab_time = gr.drab_time;
      bc.Np = d.n_pos_buckets;
      bc.Nt = d.n_time_buckets;
      bc.Sp = d.pos_sub_bits;
      bc.St = d.time_sub_bits;
      bc.h = h;
      bc.dqk = d.d_qk;
      bc.dv = d.d_v;
      bc.work_next = &hdr->work_next;
      bc.work_done = &hdr->work_done;
      bc.status = status;
      where = "attention backward";
      e = launch_attn_bwd(bc, s);
    }
    // dW1 = dP^T X (split over the rows), db1 = sum of dP
    if (ok()) {
      GradGemm gw{};
      gw.A = at<void>(ws, Lo.dP);
      gw.lda = F;
      gw.a_mn = 1;
      where = "dW1";
      gw.W = xs(l);
      gw.ldw = dm;
      gw.w_mn = 1;
      gw.ab_f16 = 1;
      gw.M = F;
      gw.N = dm;
      gw.K = T;
      gw.splits = kGradSplits;
      gw.split_rows = F_pad;
      gw.out = part;
      gw.ldo = dm;
      gw.status = status;
      int used = 1;
      gw.splits_used = &used;
      e = launch_gemm_grad(gw, s, K_GEMM_BWD);
      if (ok()) {
        LaunchScope ls(K_SUM_ROWS, s);
        k_sum_slices<<<grid_for((int64_t)F * dm, kSumThreads), kSumThreads, 0, s>>>(
            part, used, F_pad * dm, (int64_t)F * dm, gr.dW1, status);
        e = cudaGetLastError();
      }
    }
    if (ok()) e = sum_rows<__half>(at<__half>(ws, Lo.dP), T, F, F, part, gr.db1, status, s);
    // dX = dY + dP W1 (fp32 stream; the caller's bf16 dX at layer 0)
    if (ok()) {
      GradGemm gx_{};
      gx_.A = at<void>(ws, Lo.dP);
      gx_.lda = F;
      gx_.W = w1h(l);
      gx_.ldw = dm;
      gx_.w_mn = 1;
      gx_.ab_f16 = 1;
      gx_.M = T;
      gx_.N = dm;
      gx_.K = F;
      gx_.splits = 1;
      where = "dX";
      gx_.out = gx;
      gx_.ldo = dm;
      gx_.resid = gy;
      gx_.out16 = l == 0 ? dX : nullptr;
      gx_.zero_bias = at<void>(ws, Lo.zbias);
      gx_.status = status;
      e = launch_gemm_grad(gx_, s, K_GEMM_BWD);
    }
    std::swap(gy, gx);
  }
  if (ok()) e = cudaPeekAtLastError();
  if (!ok()) {
    note_cuda_error(e, where);
    return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

}  // namespace
}  // namespace hstu

using namespace hstu;

extern "C" {

size_t hstu_bwd_workspace_size(const hstu_layer_desc* desc, int32_t n_layers, int64_t B,
                               int64_t total_tokens, int64_t max_len) {
  if (check_bwd_desc(desc) != HSTU_OK || n_layers < 1) return 0;
  if (B < 0 || total_tokens < 0 || max_len < 1 || total_tokens > B * max_len) return 0;
  BwdLayout L;
  if (!make_bwd_layout(*desc, n_layers, B, total_tokens, max_len, &L)) return 0;
  return L.total;
}

hstu_status hstu_layer_bwd(const hstu_layer_desc* desc, const hstu_layer_weights* weights,
                           int64_t B, int64_t total_tokens, int64_t max_len,
                           const int64_t* offsets, const void* X, const int64_t* timestamps,
                           const void* dY, void* dX, const hstu_layer_grads* grads,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return stack_bwd_impl(desc, 1, weights, B, total_tokens, max_len, offsets, X, timestamps, dY,
                        dX, grads, workspace, workspace_bytes, stream);
}

hstu_status hstu_stack_bwd(const hstu_layer_desc* desc, int32_t n_layers,
                           const hstu_layer_weights* weights, int64_t B, int64_t total_tokens,
                           int64_t max_len, const int64_t* offsets, const void* X,
                           const int64_t* timestamps, const void* dY, void* dX,
                           const hstu_layer_grads* grads, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return stack_bwd_impl(desc, n_layers, weights, B, total_tokens, max_len, offsets, X, timestamps,
                        dY, dX, grads, workspace, workspace_bytes, stream);
}

}  // extern "C"

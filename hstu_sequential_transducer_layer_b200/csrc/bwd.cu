// bwd.cu — backward pass (gradients for training) of the HSTU layer stack:
// the row-wise LayerNorm * U backward, reductions, conversions, and the C ABI
// entry points hstu_layer_bwd / hstu_stack_bwd that sequence them with the
// tensor-core GEMMs (gemm_tc.cu) and the attention backward (attn_bwd.cu).
//
// 'HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか'
// defines the forward layer; its gradients are the chain rule through it in
// reverse order (section '長い履歴を現実の計算量へ収める4つの工夫' notes that
// training keeps only a few activations per layer; here the call runs the
// stack's forward once, keeping each layer's input, f1 output, f1
// pre-activation and attention output in the workspace, then goes backward):
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
constexpr int kSumThreads = 256;
constexpr int kGradSplits = 8;       // split-K of the weight-gradient products
constexpr int kLnBwdGroups = 2368;   // LayerNorm backward row groups (partial rows of dg, dbe)
constexpr int kLnSumSplit = 32;      // first-stage sums of those partial rows
constexpr int kSumBlocks = 1184;     // row ranges of a column sum (8 blocks per SM)
constexpr int kSumSplit = 32;        // first-stage sums of their partial rows
}  // namespace

// ---------------------------------------------------------------- LayerNorm * U backward
// A group of G threads (G = 32, 64 or 128: one to four warps) per row, each
// thread owning NV vectors of 8 consecutive features (vector gt + v G of the
// row).  O arrives as the attention kernel stores it, normalised per (row,
// head): O = m + s * xn.  Per row: mu, rstd over all h*d_v features;
// xhat = (O - mu) rstd; L = xhat g + be; Z = L U (stored for dW2);
// dL = dZ U; dU = dZ L, stored as dP_U = dU SiLU'(P_U) into the f1-shaped
// gradient; dxh = dL g; dO = (dxh - mean dxh - xhat mean(dxh xhat)) rstd.
// The two row sums meet across the group's warps in shared memory (double-
// buffered by row parity, one named barrier per row).  Column partial sums of
// dL xhat (dg) and dL (dbe) stay in each thread's registers over all the rows
// of its group (a fixed order) and are written as one partial row per group.
// Four blocks per SM (64 registers, a few spilled to L1): more rows in flight
// matter more for this memory-bound kernel than the spills.
template <int NV>
__global__ void __launch_bounds__(256, 4)
    k_ln_bwd(const float* __restrict__ dZ, const __half* __restrict__ xn,
             const float2* __restrict__ stats, const __half* __restrict__ f1,
             const __half* __restrict__ pre, int64_t ld_f1, const __nv_bfloat16* __restrict__ gamma,
             const __nv_bfloat16* __restrict__ beta, float eps, int hdv, int h, int dv,
             int64_t rows, int G, __half* __restrict__ Z, __half* __restrict__ dO,
             __half* __restrict__ dP, float* __restrict__ part, const int* __restrict__ status) {
  __shared__ float2 red[2][8];  // [row parity][warp]: partial (sum dxh, sum dxh xhat)
  if (status && *status != HSTU_OK) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gpb = 256 / G;              // groups per block
  const int grp = tid / G, gt = tid - grp * G;
  const int W = G / 32, w0 = grp * W;   // warps of this group: w0 .. w0+W-1
  const int64_t gid = (int64_t)blockIdx.x * gpb + grp;
  const int64_t ngrp = (int64_t)gridDim.x * gpb;
  const int nvec = hdv / 8;
  const float inv_h = 1.0f / (float)h, inv_f = 1.0f / (float)hdv;
  float ag[NV][8], ab[NV][8];
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int k = 0; k < 8; ++k) ag[v][k] = ab[v][k] = 0.f;
  int it = 0;
  for (int64_t row = gid; row < rows; row += ngrp, ++it) {
    // row moments from the heads' (m, s): mu = mean m, var = mean (s^2 + (m - mu)^2)
    const float2 mine = lane < h ? stats[row * h + lane] : make_float2(0.f, 0.f);
    float sm = mine.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
    const float mu = sm * inv_h;
    float sv = lane < h ? fmaf(mine.y, mine.y, (mine.x - mu) * (mine.x - mu)) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
    const float rstd = rsqrtf(sv * inv_h + eps);
    float xh[NV][8], dx[NV][8];
    float s_dx = 0.f, s_dxx = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int vec = gt + v * G;
      const int k = vec * 8;
      const int head = min(k / dv, h - 1);
      const float hm = __shfl_sync(0xffffffffu, mine.x, head);
      const float hs = __shfl_sync(0xffffffffu, mine.y, head);
      if (vec < nvec) {
        const float a = (hm - mu) * rstd, b = hs * rstd;  // xhat = xn b + a
        const uint4 xv = *reinterpret_cast<const uint4*>(xn + row * hdv + k);
        const uint4 uv = *reinterpret_cast<const uint4*>(f1 + row * ld_f1 + k);
        const uint4 pv = *reinterpret_cast<const uint4*>(pre + row * ld_f1 + k);
        const float4 z0 = *reinterpret_cast<const float4*>(dZ + row * hdv + k);
        const float4 z1 = *reinterpret_cast<const float4*>(dZ + row * hdv + k + 4);
        const uint4 gv = *reinterpret_cast<const uint4*>(gamma + k);
        const uint4 bv = *reinterpret_cast<const uint4*>(beta + k);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
        const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
        const float dz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
        uint32_t zo[4], po[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float zz[2], pp[2];
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int e = 2 * e2 + hi;
            const float x = fmaf(hi ? f16hi(xw[e2]) : f16lo(xw[e2]), b, a);
            const float g = hi ? bf16hi(gw[e2]) : bf16lo(gw[e2]);
            const float l = fmaf(x, g, hi ? bf16hi(bw[e2]) : bf16lo(bw[e2]));
            const float u = hi ? f16hi(uw[e2]) : f16lo(uw[e2]);
            const float p = hi ? f16hi(pw[e2]) : f16lo(pw[e2]);
            zz[hi] = l * u;
            const float dl = dz[e] * u;
            // dP_U = dU * SiLU'(P_U), dU = dZ * L
            const float sg = __fdividef(1.0f, 1.0f + __expf(-p));
            pp[hi] = dz[e] * l * sg * fmaf(p, 1.0f - sg, 1.0f);
            ag[v][e] = fmaf(dl, x, ag[v][e]);
            ab[v][e] += dl;
            xh[v][e] = x;
            dx[v][e] = dl * g;
            s_dx += dx[v][e];
            s_dxx = fmaf(dx[v][e], x, s_dxx);
          }
          zo[e2] = pack_f16x2_sat(zz[0], zz[1]);
          po[e2] = pack_f16x2_sat(pp[0], pp[1]);
        }
        *reinterpret_cast<uint4*>(Z + row * hdv + k) = make_uint4(zo[0], zo[1], zo[2], zo[3]);
        *reinterpret_cast<uint4*>(dP + row * ld_f1 + k) = make_uint4(po[0], po[1], po[2], po[3]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s_dx += __shfl_xor_sync(0xffffffffu, s_dx, o);
      s_dxx += __shfl_xor_sync(0xffffffffu, s_dxx, o);
    }
    if (W > 1) {
      if (lane == 0) red[it & 1][warp] = make_float2(s_dx, s_dxx);
      asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(G) : "memory");
      s_dx = s_dxx = 0.f;
      for (int ww = 0; ww < W; ++ww) {  // every thread sums in the same order
        const float2 r2 = red[it & 1][w0 + ww];
        s_dx += r2.x;
        s_dxx += r2.y;
      }
    }
    const float m_dx = s_dx * inv_f, m_dxx = s_dxx * inv_f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int vec = gt + v * G;
      if (vec < nvec) {
        uint32_t oo[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)
          oo[e2] = pack_f16x2_sat((dx[v][2 * e2] - m_dx - xh[v][2 * e2] * m_dxx) * rstd,
                                  (dx[v][2 * e2 + 1] - m_dx - xh[v][2 * e2 + 1] * m_dxx) * rstd);
        *reinterpret_cast<uint4*>(dO + row * hdv + vec * 8) = make_uint4(oo[0], oo[1], oo[2], oo[3]);
      }
    }
  }
  // this group's column partials: part[gid][0][.] = dg, part[gid][1][.] = dbe
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int vec = gt + v * G;
    if (vec < nvec) {
      float* pg = part + gid * 2 * hdv + vec * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pg[e] = ag[v][e];
        pg[hdv + e] = ab[v][e];
      }
    }
  }
}

// Threads per row of the LayerNorm backward for h*d_v features: one 8-feature
// vector per thread up to four warps.
static int ln_bwd_group(int hdv) { return std::min(128, std::max(32, (hdv / 8 + 31) / 32 * 32)); }

// ---------------------------------------------------------------- reductions
// part[blockIdx.x, n] = sum over rows [x * rows_per_block, ...) of in[r, n],
// n < N (a multiple of 8; fp32 or fp16 input, row stride ld, 16-byte aligned
// rows).  A thread sums 8 consecutive columns with 16-byte loads; when a row
// has fewer than 256 such vectors the block's threads also split the rows
// (row phase t / nvec) and the phases are added in a fixed order at the end.
DEVI void load8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
DEVI void load8(const __half* p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = f16lo(w[k]);
    v[2 * k + 1] = f16hi(w[k]);
  }
}
template <typename T>
__global__ void __launch_bounds__(kSumThreads)
    k_sum_rows(const T* __restrict__ in, int64_t rows, int N, int64_t ld, int64_t rows_per_block,
               float* __restrict__ part, const int* __restrict__ status) {
  __shared__ float red[kSumThreads * 8];
  if (status && *status != HSTU_OK) return;
  const int nvec = N / 8, t = threadIdx.x;
  const int64_t r0 = blockIdx.x * rows_per_block;
  const int64_t r1 = min(rows, r0 + rows_per_block);
  float* out = part + (int64_t)blockIdx.x * N;
  if (nvec >= kSumThreads) {
    for (int v = t; v < nvec; v += kSumThreads) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int64_t r = r0; r < r1; ++r) {
        float x[8];
        load8(in + r * ld + v * 8, x);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += x[k];
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) out[v * 8 + k] = acc[k];
    }
    return;
  }
  const int RS = kSumThreads / nvec;  // row phases
  const int v = t % nvec, rp = t / nvec;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (rp < RS) {
#pragma unroll 4
    for (int64_t r = r0 + rp; r < r1; r += RS) {
      float x[8];
      load8(in + r * ld + v * 8, x);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += x[k];
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[t * 8 + k] = acc[k];
  __syncthreads();
  if (t < nvec) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float sum = 0.f;
      for (int q = 0; q < RS; ++q) sum += red[(q * nvec + t) * 8 + k];
      out[t * 8 + k] = sum;
    }
  }
}

// out[y * out_stride + x] = sum over slices s in [y * chunk, min(S, (y + 1) * chunk))
// of in[s * stride + x], x < L, in slice order (gridDim.y = 1, chunk = S: one sum).
__global__ void __launch_bounds__(kSumThreads)
    k_sum_slices(const float* __restrict__ in, int S, int64_t stride, int64_t L,
                 float* __restrict__ out, const int* __restrict__ status, int chunk = 1 << 30,
                 int64_t out_stride = 0) {
  if (status && *status != HSTU_OK) return;
  const int s0 = blockIdx.y * chunk, s1 = min(S, s0 + chunk);
  for (int64_t x = blockIdx.x * (int64_t)kSumThreads + threadIdx.x; x < L;
       x += (int64_t)gridDim.x * kSumThreads) {
    float acc = 0.f;
    for (int s = s0; s < s1; ++s) acc += in[s * stride + x];
    out[blockIdx.y * out_stride + x] = acc;
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
// out[n] = sum over all rows of in[r, n] in a fixed order: kSumBlocks row
// ranges (k_sum_rows), then kSumSplit sums of consecutive partial rows, then
// their sum.  part holds (kSumBlocks + kSumSplit) * N floats.
template <typename T>
cudaError_t sum_rows(const T* in, int64_t rows, int64_t N, int64_t ld, float* part, float* out,
                     const int* status, cudaStream_t s) {
  const int nb = (int)std::max<int64_t>(1, std::min<int64_t>(kSumBlocks, (rows + 15) / 16));
  const int64_t rpb = (rows + nb - 1) / nb;
  LaunchScope ls(K_SUM_ROWS, s);
  k_sum_rows<T><<<nb, kSumThreads, 0, s>>>(in, rows, (int)N, ld, rpb, part, status);
  float* tmp = part + (int64_t)nb * N;
  const int chunk = (nb + kSumSplit - 1) / kSumSplit;
  k_sum_slices<<<dim3((unsigned)grid_for(N, kSumThreads), kSumSplit), kSumThreads, 0, s>>>(
      part, nb, N, N, tmp, status, chunk, N);
  k_sum_slices<<<grid_for(N, kSumThreads), kSumThreads, 0, s>>>(tmp, kSumSplit, N, N, out, status);
  return cudaGetLastError();
}

struct BwdLayout {
  size_t header, items, t_rel, ubase, tbuckets;
  size_t xs;        // the layers' inputs, fp16, [n_layers][T, d]
  size_t g, pre;    // f1 output and pre-activation, fp16 [n_layers][T, F]
  size_t o;         // normalised attention output fp16 [T, hdv] + (m, s) [T, h], per layer
  size_t o_stride;  // bytes from one layer's o segment to the next
  size_t z, dz, dO, dP;
  size_t gy0, gy1;  // fp32 gradient streams [T, d]
  size_t gyh;       // fp16 copy of the current one
  size_t w16;       // fp16 copies of W1 and W2, per layer
  size_t part;      // partial sums
  size_t zbias;     // bf16 zeros
  size_t rab_acc;   // fixed-point bias-table gradient sums [h][Np + Nt] (int64)
  size_t lncoef;    // LayerNorm coefficients per (row, head) (fused f2 of the forward)
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
  o->g = take((size_t)L * T * F * 2);
  o->pre = take((size_t)L * T * F * 2);
  o->o_stride = up256(up256((size_t)T * hdv * 2) + (size_t)T * d.n_heads * 8);
  o->o = take((size_t)L * o->o_stride);
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
                                        (size_t)(kLnBwdGroups + kLnSumSplit) * 2 * hdv,
                                        (size_t)(kSumBlocks + kSumSplit) * std::max({F, hdv, dm})});
  o->part_floats = (int64_t)part;
  o->part = take(part * 4);
  o->zbias = take(std::max({F, hdv, dm}) * 2 + 1024);
  o->rab_acc = take((size_t)d.n_heads * (d.n_pos_buckets + d.n_time_buckets) * 8);
  o->lncoef = take((size_t)T * d.n_heads * 4);
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
  launch_time_rel(offsets, B, max_len, timestamps, T, at<int32_t>(ws, Lo.t_rel), hdr, s);
  launch_time_buckets(offsets, B, max_len, at<int32_t>(ws, Lo.t_rel), at<int64_t>(ws, Lo.ubase),
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
  // every layer's f1 output, pre-activation and attention output are kept
  // from the forward pass for its backward (no recomputation)
  auto g_of = [&](int l) { return at<__half>(ws, Lo.g) + (size_t)l * T * F; };
  auto pre_of = [&](int l) { return at<__half>(ws, Lo.pre) + (size_t)l * T * F; };
  auto o_of = [&](int l) { return at<__half>(ws, Lo.o + (size_t)l * Lo.o_stride); };
  auto ostats_of = [&](int l) {
    return at<float>(ws, Lo.o + (size_t)l * Lo.o_stride + up256((size_t)T * hdv * 2));
  };

  // f1 (with its pre-activation) and the attention of layer l, from xs(l)
  auto forward_parts = [&](int l) {
    void* g_buf = g_of(l);
    void* pre_buf = pre_of(l);
    void* o_buf = o_of(l);
    float* ostats = ostats_of(l);
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
    where = "f1 (forward of the stack)";
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
    where = "attention (forward of the stack)";
    e = launch_attn_tc(ac, s);
  };

  // ---- forward through every layer, keeping each layer's input (fp16) and
  // f1 / attention outputs; the last layer's f2 output is not needed
  e = convert(X, 1, nullptr, xs(0), (int64_t)T * dm, status, s);
  for (int l = 0; l < L && ok(); ++l) {
    forward_parts(l);
    if (!ok() || l == L - 1) break;
    void* g_buf = g_of(l);
    void* o_buf = o_of(l);
    float* ostats = ostats_of(l);
    GemmCall gc{};
    if (ln_fusion_for(dm)) {  // LayerNorm * U inside f2's operand stage
      gc.A = nullptr;
      gc.ln_x = o_buf;
      gc.ln_stats = ostats;
      gc.ln_coef = at<uint32_t>(ws, Lo.lncoef);
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
    void* g_buf = g_of(l);
    void* pre_buf = pre_of(l);
    void* o_buf = o_of(l);
    float* ostats = ostats_of(l);
    // (gyh, the fp16 copy of gy, was written by the layer above's dX product)
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
      // G threads per row, 256 / G rows at a time per block, at most
      // kLnBwdGroups row groups (each leaves one partial row of dg, dbe)
      const int G = ln_bwd_group(hdv), gpb = 256 / G;
      const int nb = (int)std::max<int64_t>(
          1, std::min<int64_t>(kLnBwdGroups / gpb, (T + gpb - 1) / gpb));
      const int ngrp = nb * gpb;
      where = "LayerNorm backward";
      LaunchScope ls(K_LN_BWD, s);
      const bool two = hdv / 8 > G;  // two 8-feature vectors per thread (h*d_v > 1024)
      auto kfn = two ? k_ln_bwd<2> : k_ln_bwd<1>;
      kfn<<<nb, 256, 0, s>>>(
          at<float>(ws, Lo.dz), static_cast<const __half*>(o_buf),
          reinterpret_cast<const float2*>(ostats), static_cast<const __half*>(g_buf),
          static_cast<const __half*>(pre_buf), F, static_cast<const __nv_bfloat16*>(W[l].ln_gamma),
          static_cast<const __nv_bfloat16*>(W[l].ln_beta), d.ln_eps, hdv, h, d.d_v, T, G,
          at<__half>(ws, Lo.z), at<__half>(ws, Lo.dO), at<__half>(ws, Lo.dP), part, status);
      e = cudaGetLastError();
      if (ok()) {
        // the ngrp partial rows [dg | dbe] in two stages (kLnSumSplit sums of
        // consecutive partial rows, then their sum), each in a fixed order
        LaunchScope ls2(K_SUM_ROWS, s);
        float* tmp = part + (int64_t)ngrp * 2 * hdv;
        const int chunk = (ngrp + kLnSumSplit - 1) / kLnSumSplit;
        k_sum_slices<<<dim3((unsigned)grid_for(2 * hdv, kSumThreads), kLnSumSplit), kSumThreads, 0,
                       s>>>(part, ngrp, 2 * hdv, 2 * hdv, tmp, status, chunk, 2 * hdv);
        k_sum_slices<<<grid_for(hdv, kSumThreads), kSumThreads, 0, s>>>(tmp, kLnSumSplit, 2 * hdv,
                                                                         hdv, gr.dln_gamma, status);
        k_sum_slices<<<grid_for(hdv, kSumThreads), kSumThreads, 0, s>>>(
            tmp + hdv, kLnSumSplit, 2 * hdv, hdv, gr.dln_beta, status);
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
      bc.rab_acc = at<unsigned long long>(ws, Lo.rab_acc);
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
      // the caller's bf16 dX at layer 0; above it, the fp16 copy of this
      // gradient stream that the next layer's products read
      gx_.out16 = l == 0 ? dX : static_cast<void*>(gyh);
      gx_.out16_f16 = l == 0 ? 0 : 1;
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

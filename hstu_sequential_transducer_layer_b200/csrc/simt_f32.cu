// simt_f32.cu — the fp32 path: the same layer computed with FP32 FMA on the
// CUDA cores.  TF32 tensor-core math would round the operands to 10 mantissa
// bits, which cannot meet a 1e-4 relative error, so fp32 layers run here.
// ('HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか':
// f1 + SiLU + split, pointwise attention with relative bias, LayerNorm * U,
// f2 + residual.)
#include <climits>

#include "ptx.cuh"

namespace hstu {

// ---------------------------------------------------------------- GEMM
// C[M, N] = A[M, K] W[n_off + N, K]^T; 64 x 64 tiles, 256 threads, 4 x 4 each.
constexpr int kSG = 64, kSK = 16;

template <int EPI>
__global__ void __launch_bounds__(256)
    k_gemm_simt_f32(const float* __restrict__ A, int64_t lda, const float* __restrict__ W,
                    int64_t ldw, int64_t M_cap, const int64_t* M_dev, int N, int K, int n_off,
                    const float* __restrict__ bias, float* __restrict__ out, int64_t ldo,
                    const float* __restrict__ resid, int64_t ldr, const int* status) {
  if (status && *status != HSTU_OK) return;
  int64_t M = M_cap;
  if (M_dev) M = min(M, *M_dev);
  const int64_t m0 = (int64_t)blockIdx.y * kSG;
  const int n0 = blockIdx.x * kSG;
  if (m0 >= M) return;
  __shared__ float As[kSK][kSG + 1];
  __shared__ float Ws[kSK][kSG + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kSK) {
    for (int i = threadIdx.x; i < kSG * kSK; i += 256) {
      const int r = i / kSK, kk = i % kSK;
      const int64_t gm = m0 + r;
      const int gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? A[gm * lda + gk] : 0.f;
      const int gn = n0 + r;
      Ws[kk][r] = (gn < N && gk < K) ? W[(int64_t)(n_off + gn) * ldw + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        w[i] = Ws[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      const int col = n_off + gn;
      float v = acc[i][j] + bias[col];
      if (EPI == EPI_SILU) v = v / (1.0f + expf(-v));
      else v += resid[gm * ldr + col];
      out[gm * ldo + col] = v;
    }
  }
}

cudaError_t launch_gemm_simt_f32(const GemmCall& c, cudaStream_t s, int kernel_id) {
  if (c.M_cap <= 0 || c.N <= 0) return cudaSuccess;
  LaunchScope ls(kernel_id, s);
  dim3 grid((c.N + kSG - 1) / kSG, (unsigned)((c.M_cap + kSG - 1) / kSG));
  if (c.epi == EPI_SILU)
    k_gemm_simt_f32<EPI_SILU><<<grid, 256, 0, s>>>(
        (const float*)c.A, c.lda, (const float*)c.W, c.ldw, c.M_cap, c.M_dev, c.N, c.K, c.n_off,
        (const float*)c.bias, (float*)c.out, c.ldo, (const float*)c.resid, c.ldr, c.status);
  else
    k_gemm_simt_f32<EPI_RESID><<<grid, 256, 0, s>>>(
        (const float*)c.A, c.lda, (const float*)c.W, c.ldw, c.M_cap, c.M_dev, c.N, c.K, c.n_off,
        (const float*)c.bias, (float*)c.out, c.ldo, (const float*)c.resid, c.ldr, c.status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- attention
// One warp per (query row, head).  Lanes split the q.k dot product and the
// d_v outputs; the score and SiLU weight are warp-uniform.
__device__ __forceinline__ int64_t find_row_user(const int64_t* off, int64_t B, int64_t row) {
  int64_t lo = 0, hi = B;
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (off[mid] <= row) lo = mid;
    else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float silu_f32(float x) { return x / (1.0f + expf(-x)); }

template <int MODE>
__global__ void __launch_bounds__(256)
    k_attn_simt_f32(const int64_t* __restrict__ q_off, const int64_t* __restrict__ kv_off,
                    int64_t B, int64_t q_rows_cap, const int64_t* q_rows_dev,
                    const float* __restrict__ qbuf, const float* __restrict__ kvbuf, int64_t ld,
                    int q_col, int k_col, int v_col, const int32_t* __restrict__ t_rel,
                    const int32_t* __restrict__ t_req_rel, const float* __restrict__ rab_pos,
                    const float* __restrict__ rab_time, int Np, int Nt, int Sp, int St, int h,
                    int dqk, int dv, float* __restrict__ O, int64_t ldo, const int* status) {
  if (status && *status != HSTU_OK) return;
  int64_t rows = q_rows_cap;
  if (q_rows_dev) rows = min(rows, *q_rows_dev);
  const int lane = threadIdx.x & 31;
  const int64_t gw = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (gw >= rows * h) return;
  const int64_t row = gw / h;
  const int head = (int)(gw - row * h);
  const int64_t b = find_row_user(q_off, B, row);
  const int64_t kv0 = kv_off[b];
  const int n = (int)(kv_off[b + 1] - kv0);
  const float* Rp = rab_pos + (size_t)head * Np;
  const float* Rt = rab_time + (size_t)head * Nt;
  const float* qrow = qbuf + row * ld + q_col + head * dqk;
  float qv[4], o[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    qv[u] = c < dqk ? qrow[c] : 0.f;
    o[u] = 0.f;
  }
  int i_loc, jmax, t_i;
  if (MODE == 0) {
    i_loc = (int)(row - q_off[b]);
    jmax = i_loc;            // causal: j <= i
    t_i = t_rel[row];
  } else {
    i_loc = n;               // every candidate sits at position n
    jmax = n - 1;            // the whole history
    t_i = t_req_rel[b];
  }
  for (int j = 0; j <= jmax; ++j) {
    const float* krow = kvbuf + (kv0 + j) * ld + k_col + head * dqk;
    float part = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dqk) part = fmaf(qv[u], krow[c], part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const int gap = max(t_i - t_rel[kv0 + j], 0);
    const float sc = part + Rp[log_bucket(i_loc - j, Sp, Np)] + Rt[log_bucket(gap, St, Nt)];
    const float w = silu_f32(sc);
    const float* vrow = kvbuf + (kv0 + j) * ld + v_col + head * dv;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dv) o[u] = fmaf(w, vrow[c], o[u]);
    }
  }
  if (MODE == 1) {  // self term at distance 0, gap 0
    const float* krow = qbuf + row * ld + k_col + head * dqk;
    float part = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dqk) part = fmaf(qv[u], krow[c], part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float w = silu_f32(part + Rp[0] + Rt[0]);
    const float* vrow = qbuf + row * ld + v_col + head * dv;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dv) o[u] = fmaf(w, vrow[c], o[u]);
    }
  }
  const float inv_n = 1.0f / (float)max(n, 1);
  float* orow = O + row * ldo + head * dv;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    if (c < dv) orow[c] = o[u] * inv_n;
  }
}

cudaError_t launch_attn_simt_f32(const AttnCall& c, cudaStream_t s) {
  if (c.q_rows_cap <= 0) return cudaSuccess;
  if (c.dqk > 128 || c.dv > 128) return cudaErrorInvalidValue;
  LaunchScope ls(c.mode == 0 ? K_SIMT_ATTN : K_SIMT_ATTN_CAND, s);
  const int64_t warps = c.q_rows_cap * c.h;
  const int grid = (int)((warps + 7) / 8);
  if (c.mode == 0)
    k_attn_simt_f32<0><<<grid, 256, 0, s>>>(
        c.q_off, c.kv_off, c.B, c.q_rows_cap, c.q_rows_dev, (const float*)c.q_buf,
        (const float*)c.kv_buf, c.ld_f1, c.q_col, c.k_col, c.v_col, c.t_rel, c.t_req_rel,
        c.rab_pos, c.rab_time, c.Np, c.Nt, c.Sp, c.St, c.h, c.dqk, c.dv, (float*)c.O, c.ldo,
        c.status);
  else
    k_attn_simt_f32<1><<<grid, 256, 0, s>>>(
        c.q_off, c.kv_off, c.B, c.q_rows_cap, c.q_rows_dev, (const float*)c.q_buf,
        (const float*)c.kv_buf, c.ld_f1, c.q_col, c.k_col, c.v_col, c.t_rel, c.t_req_rel,
        c.rab_pos, c.rab_time, c.Np, c.Nt, c.Sp, c.St, c.h, c.dqk, c.dv, (float*)c.O, c.ldo,
        c.status);
  return cudaGetLastError();
}

}  // namespace hstu

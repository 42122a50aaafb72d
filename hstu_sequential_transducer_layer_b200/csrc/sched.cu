// sched.cu — the jagged tile scheduler and the small memory-bound kernels
// around the tensor-core ones:
//   * k_schedule: validates the offsets and lists the attention work items
//     (user, query tile, head) with the number of KV tiles each needs, longest
//     first ('HSTUとGenerative Recommenders', section '長い履歴を現実の計算量へ
//     収める4つの工夫', subsection '1. 長さの異なるsequenceをpaddingせず処理する':
//     ragged sequences without padding); fully masked causal tiles never appear.
//   * k_time_rel: per-row timestamp relative to the user's first one (int32).
//   * k_ln_gate: Z = LayerNorm(O) * gamma + beta, times U (subsection
//     '3. Uでcontextをgateし、次のlayerへ渡す').
//   * M-FALCON microbatch plan / gather / score (subsection '4. M-FALCONで
//     候補間の履歴計算を共有する').
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "ptx.cuh"

namespace hstu {

constexpr int kSchedThreads = 1024;

__device__ __forceinline__ void set_status(int* st, int code) { atomicCAS(st, 0, code); }

// ---------------------------------------------------------------- schedule
// Block-wide exclusive scan over users of v(b); writes out[0..B] (out[B] =
// total) and returns the total.  All threads of the block must call it.
template <typename F>
__device__ long long block_scan_users(int64_t B, F v, int64_t* out, long long* s_part,
                                      long long* s_carry) {
  if (threadIdx.x == 0) *s_carry = 0;
  __syncthreads();
  for (int64_t b0 = 0; b0 <= B; b0 += blockDim.x) {
    const int64_t b = b0 + threadIdx.x;
    const long long x = b < B ? v(b) : 0;
    s_part[threadIdx.x] = x;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
      const long long y = threadIdx.x >= (unsigned)o ? s_part[threadIdx.x - o] : 0;
      __syncthreads();
      s_part[threadIdx.x] += y;
      __syncthreads();
    }
    if (b <= B) out[b] = *s_carry + s_part[threadIdx.x] - x;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) *s_carry += s_part[threadIdx.x];
    __syncthreads();
  }
  return *s_carry;
}

constexpr int kMaxLevels = 4096;  // q-tiles per user handled by the parallel path

__global__ void __launch_bounds__(kSchedThreads)
    k_schedule(const int64_t* __restrict__ off, int64_t B, int64_t T, int64_t max_len, int h,
               AttnItem* __restrict__ items, int64_t item_cap, int64_t* __restrict__ ubase,
               int64_t tile_cap, Header* hdr) {
  __shared__ int s_bad, s_nqmax;
  __shared__ long long s_part[kSchedThreads];
  __shared__ long long s_carry;
  __shared__ int s_hist[kMaxLevels + 1];     // users per q-tile count
  __shared__ int s_cursor[kMaxLevels + 1];   // next item position per q-tile count
  if (threadIdx.x == 0) {
    hdr->status = HSTU_OK;
    hdr->n_items = 0;
    hdr->n_tiles = 0;
    hdr->work_next = 0;
    hdr->work_done = 0;
    s_bad = 0;
    s_nqmax = 0;
    if (off[0] != 0 || off[B] != T) s_bad = 1;
  }
  for (int i = threadIdx.x; i <= kMaxLevels; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t n = off[b + 1] - off[b];
    if (n < 0 || n > max_len) s_bad = 1;
    else atomicMax(&s_nqmax, (int)((n + kTile - 1) / kTile));
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) hdr->status = HSTU_ERR_BAD_OFFSETS;
    return;
  }
  auto nq_of = [&](int64_t b) { return (int)((off[b + 1] - off[b] + kTile - 1) / kTile); };
  // first time-bucket tile of every user: prefix of nq (nq + 1) / 2
  const long long tiles = block_scan_users(
      B, [&](int64_t b) { const long long q = nq_of(b); return q * (q + 1) / 2; }, ubase, s_part,
      &s_carry);
  // Items grouped by (user, head): users with more q-tiles first, then heads,
  // then q-tiles longest first; neighbouring items read the same K/V.  The
  // order of users with equal q-tile counts is immaterial (each item writes
  // only its own rows).
  const int nqmax = s_nqmax;
  long long total = 0;
  if (nqmax <= kMaxLevels) {
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
      const int c = nq_of(b);
      if (c > 0) atomicAdd(&s_hist[c], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long long acc = 0;
      for (int c = nqmax; c >= 1; --c) {
        s_cursor[c] = (int)(acc < (1ll << 30) ? acc : (1ll << 30));
        acc += (long long)s_hist[c] * c * h;
      }
      s_carry = acc;
    }
    __syncthreads();
    total = s_carry;
    // one warp per user (its lanes write the user's c * h items: head-major,
    // q-tiles longest first), so a few long users do not serialise the writes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
    for (int64_t b = warp; b < B; b += n_warps) {
      const int c = nq_of(b);
      if (c == 0) continue;
      long long pos = 0;
      if (lane == 0) pos = atomicAdd(&s_cursor[c], c * h);
      pos = __shfl_sync(0xffffffffu, pos, 0);
      const int64_t o0 = off[b];
      const int32_t n_b = (int32_t)(off[b + 1] - o0);
      const long long ub = ubase[b];
      for (int k = lane; k < c * h; k += 32) {
        const int hh = k / c, qt = c - 1 - (k - hh * c);
        if (pos + k < item_cap)
          items[pos + k] = AttnItem{(int32_t)b, (int16_t)qt, (int16_t)hh, qt + 1,
                                    (int32_t)(ub + (long long)qt * (qt + 1) / 2),
                                    (int32_t)(o0 + (int64_t)qt * kTile), (int32_t)o0, n_b, n_b};
      }
    }
  } else if (threadIdx.x == 0) {  // users over kMaxLevels * 128 tokens: one thread walks them
    long long pos = 0;
    for (int c = nqmax; c >= 1; --c)
      for (int64_t b = 0; b < B; ++b) {
        if (nq_of(b) != c) continue;
        for (int hh = 0; hh < h; ++hh)
          for (int qt = c - 1; qt >= 0; --qt, ++pos)
            if (pos < item_cap)
              items[pos] = AttnItem{(int32_t)b, (int16_t)qt, (int16_t)hh, qt + 1,
                                    (int32_t)(ubase[b] + (long long)qt * (qt + 1) / 2),
                                    (int32_t)(off[b] + (int64_t)qt * kTile), (int32_t)off[b],
                                    (int32_t)(off[b + 1] - off[b]),
                                    (int32_t)(off[b + 1] - off[b])};
      }
    total = pos;
  }
  if (threadIdx.x == 0) {
    hdr->n_items = (int32_t)(total < item_cap ? total : item_cap);
    hdr->n_tiles = (int32_t)(tiles < tile_cap ? tiles : tile_cap);
  }
}

void launch_schedule(const int64_t* offsets, int64_t B, int64_t T, int64_t max_len, int n_heads,
                     AttnItem* items, int64_t item_cap, int64_t* ubase, int64_t tile_cap,
                     Header* hdr, cudaStream_t s) {
  LaunchScope ls(K_SCHEDULE, s);
  k_schedule<<<1, kSchedThreads, 0, s>>>(offsets, B, T, max_len, n_heads, items, item_cap, ubase,
                                         tile_cap, hdr);
}

// ---------------------------------------------------------------- timestamps
__device__ __forceinline__ int64_t find_user(const int64_t* off, int64_t B, int64_t row) {
  int64_t lo = 0, hi = B;  // off[lo] <= row < off[hi]
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (off[mid] <= row) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Users along the grid's y dimension, each user's rows along x: no search for
// the user of a row.
__global__ void k_time_rel(const int64_t* __restrict__ off, int64_t B,
                           const int64_t* __restrict__ ts, int32_t* __restrict__ t_rel,
                           Header* hdr) {
  if (hdr->status != HSTU_OK) return;
  for (int64_t b = blockIdx.y; b < B; b += gridDim.y) {
    const int64_t s0 = off[b], s1 = off[b + 1];
    if (s1 <= s0) continue;
    const int64_t t0 = ts[s0];
    for (int64_t i = s0 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < s1;
         i += (int64_t)gridDim.x * blockDim.x) {
      const int64_t d = ts[i] - t0;
      if (d >= (1ll << 30) || d <= -(1ll << 30)) {
        set_status(&hdr->status, HSTU_ERR_BAD_TIMESTAMPS);
        t_rel[i] = 0;
      } else {
        t_rel[i] = (int32_t)d;
      }
    }
  }
}

void launch_time_rel(const int64_t* offsets, int64_t B, int64_t max_len, const int64_t* ts,
                     int64_t T, int32_t* t_rel, Header* hdr, cudaStream_t s) {
  if (T <= 0 || B <= 0) return;
  LaunchScope ls(K_TIME_REL, s);
  const dim3 grid((unsigned)std::max<int64_t>(1, std::min<int64_t>((max_len + 255) / 256, 32)),
                  (unsigned)std::min<int64_t>(B, 65535));
  k_time_rel<<<grid, 256, 0, s>>>(offsets, B, ts, t_rel, hdr);
}

// ---------------------------------------------------------------- time buckets
// One block per tile (grid-stride over every tile of the batch, so the work is
// even across blocks): tile t of user b is local index qt (qt + 1) / 2 + j
// (j <= qt), b found by binary search over the users' first tiles, which each
// block first copies into shared memory (up to kBucketUsersSmem users; beyond,
// the search reads them from global memory).  Word (c4, r) packs the buckets
// of row qt*128 + r against columns j*128 + 4*c4 .. +3; entries outside the
// causal triangle or the sequence are 0 (they are masked or unused).
constexpr int kBucketUsersSmem = 4096;

__global__ void __launch_bounds__(256)
    k_time_buckets(const int64_t* __restrict__ off, int64_t B, const int32_t* __restrict__ t_rel,
                   const int64_t* __restrict__ ubase, int St, int Nt,
                   uint32_t* __restrict__ tb, const Header* hdr) {
  __shared__ __align__(16) int s_tj[kTile];
  __shared__ int s_ub[kBucketUsersSmem + 1];  // first tile of each user (fits int: tiles < 2^31)
  if (hdr->status != HSTU_OK) return;
  const int n_tiles = hdr->n_tiles;
  const bool ub_smem = B < kBucketUsersSmem;
  if (ub_smem)
    for (int64_t i = threadIdx.x; i <= B; i += blockDim.x) s_ub[i] = (int)ubase[i];
  __syncthreads();
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    // the user of tile t: ubase[b] <= t < ubase[b + 1]
    int64_t lo = 0, hi = B;
    while (hi - lo > 1) {
      const int64_t mid = (lo + hi) >> 1;
      const int64_t u = ub_smem ? (int64_t)s_ub[mid] : ubase[mid];
      if (u <= t) lo = mid;
      else hi = mid;
    }
    const int64_t b = lo;
    const int64_t local = t - (ub_smem ? (int64_t)s_ub[b] : ubase[b]);
    int qt = (int)((sqrt(8.0 * (double)local + 1.0) - 1.0) * 0.5);
    while ((int64_t)qt * (qt + 1) / 2 > local) --qt;
    while ((int64_t)(qt + 1) * (qt + 2) / 2 <= local) ++qt;
    const int j = (int)(local - (int64_t)qt * (qt + 1) / 2);
    const int64_t kv0 = off[b];
    const int n = (int)(off[b + 1] - kv0);
    const int r = threadIdx.x & 127;
    const int i = qt * kTile + r;
    const bool row_ok = i < n;
    const int ti = row_ok ? t_rel[kv0 + i] : 0;
    // the tile's 128 column timestamps, read once into shared memory
    __syncthreads();  // the previous tile's columns are no longer read
    if (threadIdx.x < kTile) {
      const int jj = j * kTile + threadIdx.x;
      s_tj[threadIdx.x] = jj < n ? t_rel[kv0 + jj] : 0;
    }
    __syncthreads();
    uint32_t* dst = tb + (size_t)t * kBucketTileWords;
    // four buckets packed into a word by byte permutes (bucket k in byte k)
    auto pack4 = [](uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
      return __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u);
    };
    if (j < qt && row_ok) {
      // below the diagonal every column of a valid row is in the past: no mask
#pragma unroll 4
      for (int u = 0; u < 16; ++u) {
        const int c4 = (threadIdx.x >> 7) + 2 * u;
        const int4 tj = *reinterpret_cast<const int4*>(s_tj + 4 * c4);
        dst[c4 * 128 + r] = pack4(log_bucket_nb(max(ti - tj.x, 0), St, Nt),
                                  log_bucket_nb(max(ti - tj.y, 0), St, Nt),
                                  log_bucket_nb(max(ti - tj.z, 0), St, Nt),
                                  log_bucket_nb(max(ti - tj.w, 0), St, Nt));
      }
      continue;
    }
#pragma unroll 4
    for (int u = 0; u < 16; ++u) {
      const int c4 = (threadIdx.x >> 7) + 2 * u;
      const int4 tj = *reinterpret_cast<const int4*>(s_tj + 4 * c4);
      const int tjk[4] = {tj.x, tj.y, tj.z, tj.w};
      uint32_t bk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int jj = j * kTile + 4 * c4 + k;
        bk[k] = row_ok && jj <= i ? log_bucket_nb(max(ti - tjk[k], 0), St, Nt) : 0u;
      }
      dst[c4 * 128 + r] = pack4(bk[0], bk[1], bk[2], bk[3]);
    }
  }
}

void launch_time_buckets(const int64_t* offsets, int64_t B, int64_t max_len, const int32_t* t_rel,
                         const int64_t* ubase, int64_t tile_cap, int St, int Nt,
                         uint32_t* tbuckets, Header* hdr, cudaStream_t s) {
  (void)max_len;
  if (tile_cap <= 0 || B <= 0) return;
  LaunchScope ls(K_TIME_BUCKETS, s);
  const int grid = (int)std::min<int64_t>(tile_cap, 8 * num_sms());
  k_time_buckets<<<grid, 256, 0, s>>>(offsets, B, t_rel, ubase, St, Nt, tbuckets, hdr);
}

// ---------------------------------------------------------------- LayerNorm * U
template <typename Tv>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16(v); }
};
template <>
struct Elem<__half> {
  static __device__ __forceinline__ float ld(const __half* p) { return __half2float(*p); }
  static __device__ __forceinline__ void st(__half* p, float v) {
    *p = __float2half_rn(fminf(fmaxf(v, -65504.f), 65504.f));
  }
};
template <>
struct Elem<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};

// One warp per row; O is fp32, U / gamma / beta / Z are the layer dtype.
// Vectorised path for bf16 rows of a multiple of 256 features (8 per lane per
// step, up to 2048 features); otherwise strided scalar accesses.
constexpr int kLnMaxPerLane = 64;

template <typename Tu, typename Tg, bool VEC>
__global__ void __launch_bounds__(256)
    k_ln_gate(const float* __restrict__ O, const Tu* __restrict__ f1, int64_t ld_f1,
              const Tg* __restrict__ gamma, const Tg* __restrict__ beta, float eps,
              Tu* __restrict__ Z, int hdv, int64_t rows_cap, const int64_t* rows_dev,
              const int* status) {
  if (status && *status != HSTU_OK) return;
  int64_t rows = rows_cap;
  if (rows_dev) rows = min(rows, *rows_dev);
  const int lane = threadIdx.x & 31;
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  float x[kLnMaxPerLane];
  const float* orow = O + row * (int64_t)hdv;
  const Tu* urow = f1 + row * ld_f1;  // U occupies the first h*d_v columns
  Tu* zrow = Z + row * (int64_t)hdv;
  const int nch = hdv / 256;
  float sum = 0.f;
  uint4 uvec[kLnMaxPerLane / 8];  // U is loaded together with O (more bytes in flight)
  if (VEC) {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane / 8; ++k)
      if (k < nch) uvec[k] = *reinterpret_cast<const uint4*>(urow + (k * 32 + lane) * 8);
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane / 8; ++k) {
      if (k < nch) {
        const float4* p = reinterpret_cast<const float4*>(orow + (k * 32 + lane) * 8);
        const float4 a = p[0], b = p[1];
        x[k * 8 + 0] = a.x; x[k * 8 + 1] = a.y; x[k * 8 + 2] = a.z; x[k * 8 + 3] = a.w;
        x[k * 8 + 4] = b.x; x[k * 8 + 5] = b.y; x[k * 8 + 6] = b.z; x[k * 8 + 7] = b.w;
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += x[k * 8 + e];
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
      const int c = k * 32 + lane;
      x[k] = c < hdv ? orow[c] : 0.f;
      sum += x[k];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / (float)hdv;
  float ss = 0.f;
  if (VEC) {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane / 8; ++k)
      if (k < nch)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float dlt = x[k * 8 + e] - mean;
          ss += dlt * dlt;
        }
  } else {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
      const int c = k * 32 + lane;
      if (c < hdv) {
        const float dlt = x[k] - mean;
        ss += dlt * dlt;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = rsqrtf(ss / (float)hdv + eps);
  if (VEC) {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane / 8; ++k) {
      if (k < nch) {
        const int c0 = (k * 32 + lane) * 8;
        const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma + c0));
        const uint4 bv = __ldg(reinterpret_cast<const uint4*>(beta + c0));
        const uint4 uv = uvec[k];
        const uint32_t g[4] = {gv.x, gv.y, gv.z, gv.w}, bb[4] = {bv.x, bv.y, bv.z, bv.w},
                       u[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t out[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float z0 =
              ((x[k * 8 + 2 * e] - mean) * rstd * bf16lo(g[e]) + bf16lo(bb[e])) * f16lo(u[e]);
          const float z1 =
              ((x[k * 8 + 2 * e + 1] - mean) * rstd * bf16hi(g[e]) + bf16hi(bb[e])) * f16hi(u[e]);
          out[e] = pack_f16x2_sat(z0, z1);
        }
        *reinterpret_cast<uint4*>(zrow + c0) = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
      const int c = k * 32 + lane;
      if (c < hdv) {
        const float z = ((x[k] - mean) * rstd * Elem<Tg>::ld(gamma + c) + Elem<Tg>::ld(beta + c)) *
                        Elem<Tu>::ld(urow + c);
        Elem<Tu>::st(zrow + c, z);
      }
    }
  }
}

cudaError_t launch_ln_gate(int dtype, const void* O, const void* f1, int64_t ld_f1,
                           const void* gamma, const void* beta, float eps, void* Z, int hdv,
                           int64_t rows_cap, const int64_t* rows_dev, const int* status,
                           cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  if (hdv > 32 * kLnMaxPerLane) return cudaErrorInvalidValue;
  LaunchScope ls(K_LN_GATE, s);
  const int grid = (int)((rows_cap + 7) / 8);
  const float* Of = static_cast<const float*>(O);
  if (dtype == HSTU_BF16) {  // tensor-core path: U and Z fp16, gamma / beta bf16
    using U = __half;
    using G = __nv_bfloat16;
    if (hdv % 256 == 0)
      k_ln_gate<U, G, true><<<grid, 256, 0, s>>>(Of, (const U*)f1, ld_f1, (const G*)gamma,
                                                 (const G*)beta, eps, (U*)Z, hdv, rows_cap,
                                                 rows_dev, status);
    else
      k_ln_gate<U, G, false><<<grid, 256, 0, s>>>(Of, (const U*)f1, ld_f1, (const G*)gamma,
                                                  (const G*)beta, eps, (U*)Z, hdv, rows_cap,
                                                  rows_dev, status);
  } else {
    using T = float;
    k_ln_gate<T, T, false><<<grid, 256, 0, s>>>(Of, (const T*)f1, ld_f1, (const T*)gamma,
                                                (const T*)beta, eps, (T*)Z, hdv, rows_cap,
                                                rows_dev, status);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- LayerNorm * U from normalised O
// Z = ((O - mu) * rstd * gamma + beta) * U, one warp per row, with O given as
// the attention kernel stores it: per (row, head) its mean m and deviation s
// (fp32) and the normalised values x = (O - m) / s (fp16), so (O - mu) * rstd
// = a + b x with a = (m - mu) * rstd, b = s * rstd, and the row's moments
// follow from the heads' (m, s): mu = mean m, var = mean (s^2 + (m - mu)^2).
// Each lane takes 8 consecutive features per 256-feature chunk (all in one
// head); lane hh holds head hh's statistics and broadcasts them by shuffle.
__global__ void __launch_bounds__(256)
    k_ln_gate_norm(const __half* __restrict__ xn, const float2* __restrict__ stats,
                   const __half* __restrict__ f1, int64_t ld_f1,
                   const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                   float eps, __half* __restrict__ Z, int hdv, int h, int dv, int64_t rows_cap,
                   const int64_t* rows_dev, const int* status) {
  if (status && *status != HSTU_OK) return;
  int64_t rows = rows_cap;
  if (rows_dev) rows = min(rows, *rows_dev);
  const int lane = threadIdx.x & 31;
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float2 st = lane < h ? stats[row * h + lane] : make_float2(0.f, 0.f);
  float sm = st.x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
  const float mu = sm / (float)h;
  const float dm = st.x - mu;
  float sv = lane < h ? fmaf(st.y, st.y, dm * dm) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
  const float rstd = rsqrtf(sv / (float)h + eps);
  const float a_l = (st.x - mu) * rstd, b_l = st.y * rstd;  // this lane's head coefficients
  const __half* xr = xn + row * hdv;
  const __half* ur = f1 + row * ld_f1;
  __half* zr = Z + row * hdv;
  // every chunk's O and U loads are issued before the first is used
  constexpr int kMaxChunks = 8;  // h * d_v <= 2048
  uint4 xva[kMaxChunks], uva[kMaxChunks];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int k0 = lane * 8 + 256 * c;
    if (k0 < hdv) {
      xva[c] = *reinterpret_cast<const uint4*>(xr + k0);
      uva[c] = *reinterpret_cast<const uint4*>(ur + k0);
    }
  }
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int k0 = lane * 8 + 256 * c;
    const int head = min(k0, hdv - 1) / dv;
    const float a = __shfl_sync(0xffffffffu, a_l, head);
    const float b = __shfl_sync(0xffffffffu, b_l, head);
    if (k0 >= hdv) continue;
    const uint4 xv = xva[c];
    const uint4 uv = uva[c];
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(gamma + k0));
    const uint4 bv = __ldg(reinterpret_cast<const uint4*>(beta + k0));
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t zw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x2 = __half22float2(*reinterpret_cast<const __half2*>(&xw[e]));
      const float2 u2 = __half22float2(*reinterpret_cast<const __half2*>(&uw[e]));
      const float z0 = fmaf(fmaf(b, x2.x, a), bf16lo(gw[e]), bf16lo(bw[e])) * u2.x;
      const float z1 = fmaf(fmaf(b, x2.y, a), bf16hi(gw[e]), bf16hi(bw[e])) * u2.y;
      zw[e] = pack_f16x2_sat(z0, z1);
    }
    *reinterpret_cast<uint4*>(zr + k0) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
  }
}

cudaError_t launch_ln_gate_norm(const void* xn, const float* stats, const void* f1, int64_t ld_f1,
                                const void* gamma, const void* beta, float eps, void* Z, int hdv,
                                int h, int dv, int64_t rows_cap, const int64_t* rows_dev,
                                const int* status, cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  if (h > 32 || hdv % 8 != 0 || hdv > 2048 || dv % 8 != 0 || ld_f1 % 8 != 0)
    return cudaErrorInvalidValue;
  LaunchScope ls(K_LN_GATE, s);
  const int grid = (int)((rows_cap + 7) / 8);
  k_ln_gate_norm<<<grid, 256, 0, s>>>(static_cast<const __half*>(xn),
                                      reinterpret_cast<const float2*>(stats),
                                      static_cast<const __half*>(f1), ld_f1,
                                      static_cast<const __nv_bfloat16*>(gamma),
                                      static_cast<const __nv_bfloat16*>(beta), eps,
                                      static_cast<__half*>(Z), hdv, h, dv, rows_cap, rows_dev, status);
  return cudaGetLastError();
}

// One thread per row: the row's LayerNorm moments from its heads' (mean,
// deviation) pairs, mu = mean of m, var = mean of (s^2 + (m - mu)^2), then
// each head's coefficients a = (m - mu) rstd, b = s rstd as an fp16 pair.
__global__ void k_ln_coef(const float2* __restrict__ stats, int h, float eps,
                          uint32_t* __restrict__ coef, int64_t rows_cap,
                          const int64_t* __restrict__ rows_dev, const int* __restrict__ status) {
  if (status && *status != HSTU_OK) return;
  int64_t rows = rows_cap;
  if (rows_dev) rows = min(rows, *rows_dev);
  const float inv_h = 1.0f / (float)h;
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
       r += (int64_t)gridDim.x * blockDim.x) {
    const float2* st = stats + r * h;
    float sm = 0.f;
    for (int hh = 0; hh < h; ++hh) sm += st[hh].x;
    const float mu = sm * inv_h;
    float sv = 0.f;
    for (int hh = 0; hh < h; ++hh) {
      const float2 v = st[hh];
      const float dm = v.x - mu;
      sv = fmaf(v.y, v.y, fmaf(dm, dm, sv));
    }
    const float rstd = rsqrtf(sv * inv_h + eps);
    for (int hh = 0; hh < h; ++hh) {
      const float2 v = st[hh];
      const __half2 ab = __floats2half2_rn((v.x - mu) * rstd, v.y * rstd);
      coef[r * h + hh] = *reinterpret_cast<const uint32_t*>(&ab);
    }
  }
}

cudaError_t launch_ln_coef(const float* stats, int h, float eps, uint32_t* coef, int64_t rows_cap,
                           const int64_t* rows_dev, const int* status, cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  if (h < 1 || h > 32 || !stats || !coef) return cudaErrorInvalidValue;
  LaunchScope ls(K_LN_COEF, s);
  const int grid = (int)std::min<int64_t>((rows_cap + 255) / 256, 8 * (int64_t)num_sms());
  k_ln_coef<<<grid, 256, 0, s>>>(reinterpret_cast<const float2*>(stats), h, eps, coef, rows_cap,
                                 rows_dev, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- bf16 -> fp16
// One launch converts up to kMaxConvSegs segments (blockIdx.y = segment).
__global__ void k_bf16_to_f16(ConvBatch cb) {
  const ConvSeg sg = cb.seg[blockIdx.y];
  const uint4* src = static_cast<const uint4*>(sg.src);
  uint4* dst = static_cast<uint4*>(sg.dst);
  const int64_t n8 = sg.n / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    uint4 o;
    o.x = pack_f16x2_sat(bf16lo(v.x), bf16hi(v.x));
    o.y = pack_f16x2_sat(bf16lo(v.y), bf16hi(v.y));
    o.z = pack_f16x2_sat(bf16lo(v.z), bf16hi(v.z));
    o.w = pack_f16x2_sat(bf16lo(v.w), bf16hi(v.w));
    dst[i] = o;
  }
}

cudaError_t launch_bf16_to_f16(const ConvBatch& cb, cudaStream_t s) {
  if (cb.n <= 0) return cudaSuccess;
  int64_t mx = 0;
  for (int i = 0; i < cb.n; ++i) {
    if (cb.seg[i].n % 8 != 0) return cudaErrorInvalidValue;
    mx = std::max<int64_t>(mx, cb.seg[i].n);
  }
  LaunchScope ls(K_CONVERT, s);
  const int gx = (int)std::max<int64_t>(1, std::min<int64_t>((mx / 8 + 255) / 256, 2 * num_sms()));
  k_bf16_to_f16<<<dim3(gx, cb.n), 256, 0, s>>>(cb);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- M-FALCON plan
// For microbatch k: per user, rows [k*bm, min((k+1)*bm, m_b)) of its
// candidates; mb_off = prefix of those counts; attention items (b, q-tile,
// head) needing ceil(n_b/128) history KV tiles, longest first; request time
// relative to the user's first history timestamp.
__global__ void __launch_bounds__(kSchedThreads)
    k_mb_plan(const int64_t* __restrict__ hoff, const int64_t* __restrict__ coff, int64_t B,
              int64_t max_len, int64_t max_cands, int k, int bm, int h,
              const int64_t* __restrict__ hts, const int64_t* __restrict__ req_ts,
              int64_t* __restrict__ mb_off, AttnItem* __restrict__ items, int64_t item_cap,
              int32_t* __restrict__ t_req_rel, Header* hdr) {
  __shared__ long long s_part[kSchedThreads];
  __shared__ long long s_carry;
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    s_bad = 0;
    hdr->n_cand_items = 0;
    hdr->mb_rows = 0;
  }
  __syncthreads();
  if (hdr->status != HSTU_OK) return;
  if (k == 0) {
    if (threadIdx.x == 0 && coff[0] != 0) s_bad = 1;
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
      const int64_t m = coff[b + 1] - coff[b];
      if (m < 0 || m > max_cands) s_bad = 1;
    }
    __syncthreads();
    if (s_bad) {
      if (threadIdx.x == 0) set_status(&hdr->status, HSTU_ERR_BAD_OFFSETS);
      return;
    }
  }
  // prefix sum of per-user microbatch counts
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int64_t b0 = 0; b0 <= B; b0 += blockDim.x) {
    const int64_t b = b0 + threadIdx.x;
    long long cnt = 0;
    if (b < B) {
      const int64_t m = coff[b + 1] - coff[b];
      { const int64_t rem = m - (int64_t)k * bm; cnt = rem < 0 ? 0 : (rem > bm ? bm : rem); }
    }
    s_part[threadIdx.x] = cnt;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
      const long long v = threadIdx.x >= (unsigned)o ? s_part[threadIdx.x - o] : 0;
      __syncthreads();
      s_part[threadIdx.x] += v;
      __syncthreads();
    }
    if (b <= B) mb_off[b] = s_carry + s_part[threadIdx.x] - cnt;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry += s_part[threadIdx.x];
    __syncthreads();
  }
  // request time relative to the first history timestamp
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t n = hoff[b + 1] - hoff[b];
    const int64_t t_last = n > 0 ? hts[hoff[b + 1] - 1] : 0;
    const int64_t t_req = req_ts ? req_ts[b] : t_last;
    const int64_t base = n > 0 ? hts[hoff[b]] : t_req;
    const int64_t d = t_req - base;
    if (d >= (1ll << 30) || d <= -(1ll << 30)) {
      set_status(&hdr->status, HSTU_ERR_BAD_TIMESTAMPS);
      t_req_rel[b] = 0;
    } else {
      t_req_rel[b] = (int32_t)d;
    }
  }
  __syncthreads();
  // items, longest history first: level c = number of KV tiles (0..levels);
  // the items of one (user, head) are adjacent (they read the same history
  // K/V); users of one level are placed in any order (each item writes only
  // its own rows)
  __shared__ int s_hist[kMaxLevels + 1];    // candidate q-tiles per level
  __shared__ int s_cursor[kMaxLevels + 1];  // next q-tile position per level
  __shared__ long long s_base;
  const int levels = (int)((max_len + kTile - 1) / kTile);
  auto emit = [&](int64_t b, long long pos, int nkv) {
    const int64_t n = hoff[b + 1] - hoff[b];
    const int64_t rows = mb_off[b + 1] - mb_off[b];
    const int nq = (int)((rows + kTile - 1) / kTile);
    for (int hh = 0; hh < h; ++hh)
      for (int qt = 0; qt < nq; ++qt) {
        const long long idx = pos * h + (long long)hh * nq + qt;
        if (idx < item_cap)
          items[idx] = AttnItem{(int32_t)b, (int16_t)qt, (int16_t)hh, nkv, 0,
                                (int32_t)(mb_off[b] + (int64_t)qt * kTile), (int32_t)hoff[b],
                                (int32_t)rows, (int32_t)n};
      }
  };
  auto nkv_of = [&](int64_t b) { return (int)((hoff[b + 1] - hoff[b] + kTile - 1) / kTile); };
  auto nq_of = [&](int64_t b) { return (int)((mb_off[b + 1] - mb_off[b] + kTile - 1) / kTile); };
  if (levels <= kMaxLevels) {
    for (int i = threadIdx.x; i <= kMaxLevels; i += blockDim.x) s_hist[i] = 0;
    __syncthreads();
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
      const int nq = nq_of(b);
      if (nq > 0) atomicAdd(&s_hist[min(nkv_of(b), levels)], nq);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long long acc = 0;
      for (int c = levels; c >= 0; --c) {
        s_cursor[c] = (int)(acc < (1ll << 30) ? acc : (1ll << 30));
        acc += s_hist[c];
      }
      s_base = acc;
    }
    __syncthreads();
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
      const int nq = nq_of(b);
      if (nq == 0) continue;
      const int c = min(nkv_of(b), levels);
      emit(b, atomicAdd(&s_cursor[c], nq), c);
    }
  } else if (threadIdx.x == 0) {  // histories over kMaxLevels * 128 rows: one thread walks them
    long long pos = 0;
    for (int c = levels; c >= 0; --c)
      for (int64_t b = 0; b < B; ++b) {
        if (nkv_of(b) != c || nq_of(b) == 0) continue;
        emit(b, pos, c);
        pos += nq_of(b);
      }
    s_base = pos;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    hdr->n_cand_items = (int32_t)(s_base * h < item_cap ? s_base * h : item_cap);
    hdr->mb_rows = mb_off[B];
  }
}

void launch_mb_plan(const int64_t* hist_off, const int64_t* cand_off, int64_t B, int64_t max_len,
                    int64_t max_cands, int k, int microbatch, int n_heads,
                    const int64_t* hist_ts, const int64_t* request_ts, int64_t* mb_off,
                    AttnItem* items, int64_t item_cap, int32_t* t_req_rel, Header* hdr,
                    cudaStream_t s) {
  LaunchScope ls(K_MB_PLAN, s);
  k_mb_plan<<<1, kSchedThreads, 0, s>>>(hist_off, cand_off, B, max_len, max_cands, k, microbatch,
                                        n_heads, hist_ts, request_ts, mb_off, items, item_cap,
                                        t_req_rel, hdr);
}

// ---------------------------------------------------------------- gather / score
template <typename Tv>
__global__ void k_mb_gather(const Tv* __restrict__ cands, int64_t d,
                            const int64_t* __restrict__ coff, const int64_t* __restrict__ mb_off,
                            int64_t B, int k, int bm, Tv* __restrict__ xc, int64_t rows_cap,
                            const int64_t* rows_dev, const int* status) {
  if (*status != HSTU_OK) return;
  const int64_t rows = min(rows_cap, *rows_dev);
  const int64_t vec = (int64_t)(16 / sizeof(Tv));
  const int64_t per_row = d / vec;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < rows * per_row;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / per_row, c = i - r * per_row;
    const int64_t b = find_user(mb_off, B, r);
    const int64_t src = coff[b] + (int64_t)k * bm + (r - mb_off[b]);
    reinterpret_cast<uint4*>(xc + r * d)[c] = reinterpret_cast<const uint4*>(cands + src * d)[c];
  }
}

cudaError_t launch_mb_gather(int dtype, const void* cands, int64_t d, const int64_t* cand_off,
                             const int64_t* mb_off, int64_t B, int k, int microbatch, void* xc,
                             int64_t rows_cap, const int64_t* rows_dev, const int* status,
                             cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  LaunchScope ls(K_MB_GATHER, s);
  const int grid = 4 * num_sms();
  if (dtype == HSTU_BF16)
    k_mb_gather<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)cands, d, cand_off,
                                                     mb_off, B, k, microbatch,
                                                     (__nv_bfloat16*)xc, rows_cap, rows_dev,
                                                     status);
  else
    k_mb_gather<float><<<grid, 256, 0, s>>>((const float*)cands, d, cand_off, mb_off, B, k,
                                            microbatch, (float*)xc, rows_cap, rows_dev, status);
  return cudaGetLastError();
}

template <typename Tv>
__global__ void k_score(const float* __restrict__ xc, int64_t d, const Tv* __restrict__ w,
                        const int64_t* __restrict__ coff, const int64_t* __restrict__ mb_off,
                        int64_t B, int k, int bm, float* __restrict__ scores, int64_t rows_cap,
                        const int64_t* rows_dev, const int* status) {
  if (*status != HSTU_OK) return;
  const int64_t rows = min(rows_cap, *rows_dev);
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  if (r >= rows) return;
  float acc = 0.f;
  for (int64_t c = lane; c < d; c += 32) acc += xc[r * d + c] * Elem<Tv>::ld(w + c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const int64_t b = find_user(mb_off, B, r);
    scores[coff[b] + (int64_t)k * bm + (r - mb_off[b])] = acc;
  }
}

cudaError_t launch_score(int dtype, const float* xc, int64_t d, const void* head_vec,
                         const int64_t* cand_off, const int64_t* mb_off, int64_t B, int k,
                         int microbatch, float* scores, int64_t rows_cap,
                         const int64_t* rows_dev, const int* status, cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  LaunchScope ls(K_SCORE, s);
  const int grid = (int)((rows_cap + 7) / 8);
  if (dtype == HSTU_BF16)
    k_score<__nv_bfloat16><<<grid, 256, 0, s>>>(xc, d, (const __nv_bfloat16*)head_vec, cand_off,
                                                 mb_off, B, k, microbatch, scores, rows_cap,
                                                 rows_dev, status);
  else
    k_score<float><<<grid, 256, 0, s>>>(xc, d, (const float*)head_vec, cand_off, mb_off, B, k,
                                        microbatch, scores, rows_cap, rows_dev, status);
  return cudaGetLastError();
}

}  // namespace hstu

// sl.cu — Stochastic Length sampling and token embedding on the device.
//
// 'HSTUとGenerative Recommenders', section '2. Stochastic Lengthで学習時の履歴を
// 間引く': a long history is shortened to a random subset of its positions
// (k = min(n, floor(n^0.8)) of n, which maps the 4096 cap to 776).  The subset
// is the k positions with the smallest counter-based keys -- output number
// b * 2^32 + p + 1 of SplitMix64 started from `seed` (Steele, Lea and Flood,
// OOPSLA 2014) -- ties broken by position, kept in their original order; a
// kept token at an even original position takes its row of the content
// embedding table, at an odd position its row of the action table.
//
// k_sl_offsets (one block): validates the raw offsets and writes the kept
// offsets (prefix of the per-user keep counts).  k_sl_select (one block per
// user): a radix select, 8 bits per pass, finds the k-th smallest key (keys
// are recomputed each pass rather than stored; SplitMix64's output mix is a
// bijection, so the keys of one user are distinct and the tie rule never
// decides), then the positions are walked in order, 256 at a time, and the
// kept ones are compacted with ballot-based scans into codes (raw row and
// position parity).  k_sl_gather (all SMs) turns the codes into timestamps
// and copies the embedding rows at full memory bandwidth.
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace hstu {

constexpr int kSlThreads = 256;
constexpr int64_t kSlMaxLen = 32767;  // n^4 and (k+1)^5 stay within int64

__device__ __forceinline__ uint64_t sl_key(uint64_t seed, int64_t b, int64_t p) {
  uint64_t z = seed + ((uint64_t)(((uint64_t)b << 32) + (uint64_t)p) + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// min(n, floor(n^0.8)), at least 1 for n >= 1: the largest k with k^5 <= n^4.
__device__ __forceinline__ int64_t sl_keep(int64_t n) {
  if (n <= 0) return 0;
  const int64_t n4 = n * n * n * n;
  int64_t k = (int64_t)llround(pow((double)n, 0.8));
  auto p5 = [](int64_t x) { return x * x * x * x * x; };
  while (k > 0 && p5(k) > n4) --k;
  while (p5(k + 1) <= n4) ++k;
  k = k < n ? k : n;
  return k < 1 ? 1 : k;
}

__global__ void __launch_bounds__(1024)
    k_sl_offsets(const int64_t* __restrict__ raw_off, int64_t B, int64_t raw_total,
                 int64_t max_raw_len, int64_t* __restrict__ out_off, int* status) {
  __shared__ int s_bad;
  __shared__ long long s_part[1024];
  __shared__ long long s_carry;
  if (threadIdx.x == 0) {
    *status = HSTU_OK;
    s_bad = (raw_off[0] != 0 || raw_off[B] != raw_total) ? 1 : 0;
    s_carry = 0;
  }
  __syncthreads();
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t n = raw_off[b + 1] - raw_off[b];
    if (n < 0 || n > max_raw_len) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) *status = HSTU_ERR_BAD_OFFSETS;
    for (int64_t b = threadIdx.x; b <= B; b += blockDim.x) out_off[b] = 0;
    return;
  }
  for (int64_t b0 = 0; b0 <= B; b0 += blockDim.x) {
    const int64_t b = b0 + threadIdx.x;
    const long long x = b < B ? sl_keep(raw_off[b + 1] - raw_off[b]) : 0;
    s_part[threadIdx.x] = x;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
      const long long y = threadIdx.x >= (unsigned)o ? s_part[threadIdx.x - o] : 0;
      __syncthreads();
      s_part[threadIdx.x] += y;
      __syncthreads();
    }
    if (b <= B) out_off[b] = s_carry + s_part[threadIdx.x] - x;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry += s_part[threadIdx.x];
    __syncthreads();
  }
}

// Block-wide exclusive scan of two flags per thread (256 threads): returns
// this thread's prefix counts of `a` and `b`; *tot_a / *tot_b receive the
// block's totals.
__device__ __forceinline__ void block_flag_scan2(bool a, bool b, int* s_warp, int* pre_a,
                                                 int* pre_b, int* tot_a, int* tot_b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned ma = __ballot_sync(0xffffffffu, a), mb = __ballot_sync(0xffffffffu, b);
  const unsigned below = (1u << lane) - 1u;
  __syncthreads();  // s_warp is free (previous use done)
  if (lane == 0) s_warp[warp] = (__popc(ma) << 16) | __popc(mb);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSlThreads / 32; ++w) {
    before += w < warp ? s_warp[w] : 0;
    all += s_warp[w];
  }
  *pre_a = (before >> 16) + __popc(ma & below);
  *pre_b = (before & 0xffff) + __popc(mb & below);
  *tot_a = all >> 16;
  *tot_b = all & 0xffff;
}

// Selection, one block per user: the kept positions of user b, in order, as
// codes 2 * (raw row) + (position is odd) written to out_ts[o0 ..], which
// k_sl_gather then replaces by the timestamps.
__global__ void __launch_bounds__(kSlThreads)
    k_sl_select(const int64_t* __restrict__ raw_off, int64_t B, uint64_t seed,
                const int64_t* __restrict__ out_off, int64_t* __restrict__ out_code,
                const int* status) {
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_rem, s_cnt;
  __shared__ int s_warp[kSlThreads / 32];
  if (*status != HSTU_OK) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const int64_t r0 = raw_off[b];
    const int n = (int)(raw_off[b + 1] - r0);
    const int64_t o0 = out_off[b];
    const int k = (int)(out_off[b + 1] - o0);
    if (k <= 0) continue;
    // ---- radix select of the k-th smallest key, 8 bits per pass from the
    // top.  After each pass `prefix` holds the digits fixed so far (bits >=
    // sh) and `remaining` the rank of the wanted key among the keys that
    // share them.  When that bin holds exactly `remaining` keys, all of them
    // are kept and the lower digits do not matter: the selection stops.
    uint64_t prefix = 0;
    int remaining = k, sh = 64;
    if (k < n) {
      for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = tid; i < 256; i += kSlThreads) s_hist[i] = 0;
        __syncthreads();
        for (int p = tid; p < n; p += kSlThreads) {
          const uint64_t key = sl_key(seed, b, p);
          if (pass == 0 || (key >> sh) == (prefix >> sh)) atomicAdd(&s_hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
          // lane l owns bins 8l..8l+7: a warp scan of the lane sums finds the
          // lane holding the remaining-th key, which then walks its own bins
          int h[8], loc = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            h[j] = s_hist[lane * 8 + j];
            loc += h[j];
          }
          int incl = loc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const unsigned m = __ballot_sync(0xffffffffu, incl >= remaining);
          const int owner = m ? __ffs(m) - 1 : 31;
          if (lane == owner) {
            int acc = incl - loc, dgt = lane * 8 + 7;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (acc + h[j] >= remaining) {
                dgt = lane * 8 + j;
                break;
              }
              acc += h[j];
            }
            s_digit = dgt;
            s_rem = remaining - acc;
            s_cnt = s_hist[dgt];
          }
        }
        __syncthreads();
        prefix |= (uint64_t)s_digit << shift;
        remaining = s_rem;
        sh = shift;
        const bool done = s_cnt == remaining;
        __syncthreads();
        if (done) break;
      }
    }
    // ---- ordered compaction: a position is kept if its key's fixed digits
    // are below the prefix, or equal to it and among the first `remaining`
    // such positions.  (With k == n every position is kept: sh = 64.)
    int run_lt = 0, run_eq = 0;
    for (int base = 0; base < n; base += kSlThreads) {
      const int p = base + tid;
      bool lt = false, eq = false;
      if (p < n) {
        if (sh == 64) {
          lt = true;
        } else {
          const uint64_t hi = sl_key(seed, b, p) >> sh, ph = prefix >> sh;
          lt = hi < ph;
          eq = hi == ph;
        }
      }
      int pre_lt, pre_eq, n_lt, n_eq;
      block_flag_scan2(lt, eq, s_warp, &pre_lt, &pre_eq, &n_lt, &n_eq);
      const int eq_before = run_eq + pre_eq;
      const int eq_taken = min(eq_before, remaining);
      if (lt || (eq && eq_before < remaining))
        out_code[o0 + run_lt + pre_lt + eq_taken] = 2 * (r0 + p) + (p & 1);
      run_lt += n_lt;
      run_eq += n_eq;
    }
  }
}

// Gather, all SMs: every kept row t holds a code in out_ts[t]; its id and
// timestamp are read, the timestamp replaces the code, and the embedding row
// is copied (16 bytes per lane).  A warp takes 8 rows at a time: lanes 0..7
// read the codes, ids and timestamps, then the warp copies the 8 rows as one
// flat range of 16-byte words, 8 loads in flight per lane.
constexpr int kGatherRows = 8;
constexpr int kGatherUnroll = 8;

__global__ void __launch_bounds__(kSlThreads)
    k_sl_gather(const int64_t* __restrict__ total, const int64_t* __restrict__ ids,
                const int64_t* __restrict__ ts, const __nv_bfloat16* __restrict__ ctab,
                int64_t n_content, const __nv_bfloat16* __restrict__ atab, int64_t n_action,
                int d, __nv_bfloat16* __restrict__ X, int64_t* __restrict__ out_ts, int* status) {
  // No early exit on the status word: a bad id found by one block must not
  // stop the others (bad offsets leave *total = 0, so nothing runs then).
  const int lane = threadIdx.x & 31;
  const int64_t T = *total;
  const int d8 = d / 8;
  const int64_t n_batch = (T + kGatherRows - 1) / kGatherRows;
  const int64_t warps = (int64_t)gridDim.x * (kSlThreads / 32);
  for (int64_t bt = (int64_t)blockIdx.x * (kSlThreads / 32) + (threadIdx.x >> 5); bt < n_batch;
       bt += warps) {
    const int64_t t0 = bt * kGatherRows;
    const int nb = (int)min((int64_t)kGatherRows, T - t0);
    const uint4* src = nullptr;
    if (lane < nb) {
      const int64_t code = out_ts[t0 + lane];
      const int64_t row = code >> 1;
      const bool action = code & 1;
      const int64_t id = ids[row];
      const int64_t tsv = ts[row];
      if (id >= 0 && id < (action ? n_action : n_content))
        src = reinterpret_cast<const uint4*>((action ? atab : ctab) + id * (int64_t)d);
      else
        atomicCAS(status, HSTU_OK, HSTU_ERR_BAD_IDS);
      out_ts[t0 + lane] = tsv;
    }
    uint4* dst = reinterpret_cast<uint4*>(X + t0 * (int64_t)d);
    const int words = nb * d8;
    for (int w0 = 0; w0 < words; w0 += 32 * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int w = w0 + u * 32 + lane;
        const int r = min(w / d8, nb - 1);
        const uint4* sp = reinterpret_cast<const uint4*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r));
        v[u] = (w < words && sp) ? __ldg(sp + (w - r * d8)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int w = w0 + u * 32 + lane;
        if (w < words) dst[w] = v[u];
      }
    }
  }
}

}  // namespace hstu

// ---------------------------------------------------------------- C ABI
extern "C" {

size_t hstu_sl_embed_workspace_size(void) { return 256; }

hstu_status hstu_sl_embed(int64_t B, int64_t raw_total, int64_t max_raw_len,
                          const int64_t* raw_offsets, const int64_t* raw_ids,
                          const int64_t* raw_timestamps, uint64_t seed, const void* content_table,
                          int64_t n_content, const void* action_table, int64_t n_action,
                          int32_t d_model, int64_t* out_offsets, void* out_X,
                          int64_t* out_timestamps, void* ws, size_t ws_bytes, void* stream_ptr) {
  using namespace hstu;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (B < 0 || raw_total < 0 || max_raw_len < 0 || d_model <= 0 || d_model % 8 != 0)
    return HSTU_ERR_INVALID_ARG;
  if (max_raw_len > kSlMaxLen) return HSTU_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < hstu_sl_embed_workspace_size() || (reinterpret_cast<uintptr_t>(ws) & 255))
    return HSTU_ERR_WORKSPACE;
  if (!raw_offsets || !out_offsets) return HSTU_ERR_INVALID_ARG;
  if (raw_total > 0 && (!raw_ids || !raw_timestamps || !out_X || !out_timestamps ||
                        !content_table || !action_table))
    return HSTU_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(content_table) & 15) ||
      (reinterpret_cast<uintptr_t>(action_table) & 15) || (reinterpret_cast<uintptr_t>(out_X) & 15))
    return HSTU_ERR_INVALID_ARG;
  int* status = static_cast<int*>(ws);
  {
    LaunchScope ls(K_SL_OFFSETS, stream);
    k_sl_offsets<<<1, 1024, 0, stream>>>(raw_offsets, B, raw_total, max_raw_len, out_offsets,
                                         status);
  }
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  if (B > 0 && raw_total > 0) {
    {
      LaunchScope ls(K_SL_SELECT, stream);
      const int grid = (int)(B < 4 * num_sms() ? B : 4 * num_sms());
      k_sl_select<<<grid, kSlThreads, 0, stream>>>(raw_offsets, B, seed, out_offsets,
                                                   out_timestamps, status);
    }
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    {
      LaunchScope ls(K_SL_GATHER, stream);
      k_sl_gather<<<4 * num_sms(), kSlThreads, 0, stream>>>(
          out_offsets + B, raw_ids, raw_timestamps,
          static_cast<const __nv_bfloat16*>(content_table), n_content,
          static_cast<const __nv_bfloat16*>(action_table), n_action, d_model,
          static_cast<__nv_bfloat16*>(out_X), out_timestamps, status);
    }
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

}  // extern "C"

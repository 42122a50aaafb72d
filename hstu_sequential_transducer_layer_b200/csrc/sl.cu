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

constexpr int64_t kSlMaxLen = 32767;  // n^4 and (k+1)^5 stay within int64

__device__ __forceinline__ uint64_t sl_key(uint64_t seed, int64_t b, int64_t p) {
  uint64_t z = seed + ((uint64_t)(((uint64_t)b << 32) + (uint64_t)p) + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// min(n, floor(n^0.8)), at least 1 for n >= 1: the largest k with k^5 <= n^4.
__host__ __device__ __forceinline__ int64_t sl_keep(int64_t n) {
  if (n <= 0) return 0;
  const int64_t n4 = n * n * n * n;
  int64_t k = (int64_t)llround(pow((double)n, 0.8));
  auto p5 = [](int64_t x) { return x * x * x * x * x; };
  while (k > 0 && p5(k) > n4) --k;
  while (p5(k + 1) <= n4) ++k;
  k = k < n ? k : n;
  return k < 1 ? 1 : k;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while its predecessor runs; griddepcontrol.wait
// returns once the predecessor grid has finished and its writes are visible.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

__global__ void __launch_bounds__(1024)
    k_sl_offsets(const int64_t* __restrict__ raw_off, int64_t B, int64_t raw_total,
                 int64_t max_raw_len, int64_t* __restrict__ out_off, int* status) {
  __shared__ int s_bad;
  __shared__ long long s_part[1024];
  __shared__ long long s_carry;
  grid_dep_launch();  // k_sl_select may start; it waits for this grid to finish
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

// Block-wide exclusive scan of one int per thread (NT threads): returns this
// thread's prefix; *total receives the block's sum.  Used on packed pairs of
// 16-bit counts too (no field overflows: a block counts at most 4096).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();  // s_warp is free (previous use done)
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    before += w < warp ? s_warp[w] : 0;
    all += s_warp[w];
  }
  *total = all;
  return before + incl - v;
}

// Selection block size, positions per thread in one compaction chunk, the
// longest user whose keys stay in shared memory between passes (32 KB), and
// the largest batch whose kept offsets the selection computes itself.
constexpr int kSelThreads = 1024;
constexpr int kSlPerThread = 4;
constexpr int kSlChunk = kSelThreads * kSlPerThread;
constexpr int kSlKeyCache = 4096;
constexpr int kSlFusedMaxB = 2 * kSelThreads;

// Selection, one block per user: the kept positions of user b, in order, as
// codes 2 * (raw row) + (position is odd) written to out_code[o0 ..] (the
// kept-timestamp buffer, which k_sl_gather then fills with the timestamps).
// FUSED (B <= kSlFusedMaxB): every block validates the raw offsets and forms
// the kept offsets in shared memory itself; block 0 publishes them and the
// status word.  Otherwise k_sl_offsets has done that before.
template <bool FUSED>
__global__ void __launch_bounds__(kSelThreads)
    k_sl_select(const int64_t* __restrict__ raw_off, int64_t B, int64_t raw_total,
                int64_t max_raw_len, uint64_t seed, int64_t* __restrict__ out_off,
                int64_t* __restrict__ out_code, int* status) {
  __shared__ uint64_t s_key[kSlKeyCache];
  __shared__ int s_off[FUSED ? kSlFusedMaxB + 1 : 1];
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_rem, s_cnt;
  __shared__ int s_warp[kSelThreads / 32];
  grid_dep_launch();
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (FUSED) {
    const int64_t b0 = 2 * tid, b1 = b0 + 1;
    bool bad = tid == 0 && (raw_off[0] != 0 || raw_off[B] != raw_total);
    int k0 = 0, k1 = 0;
    if (b0 < B) {
      const int64_t n = raw_off[b0 + 1] - raw_off[b0];
      bad |= n < 0 || n > max_raw_len;
      k0 = (n < 0 || n > max_raw_len) ? 0 : (int)sl_keep(n);
    }
    if (b1 < B) {
      const int64_t n = raw_off[b1 + 1] - raw_off[b1];
      bad |= n < 0 || n > max_raw_len;
      k1 = (n < 0 || n > max_raw_len) ? 0 : (int)sl_keep(n);
    }
    if (__syncthreads_or(bad)) {
      if (blockIdx.x == 0) {
        if (tid == 0) *status = HSTU_ERR_BAD_OFFSETS;
        for (int64_t b = tid; b <= B; b += kSelThreads) out_off[b] = 0;
      }
      return;
    }
    int tot;
    const int pre = block_excl_scan<kSelThreads>(k0 + k1, s_warp, &tot);
    if (b0 <= B) s_off[b0] = pre;
    if (b1 <= B) s_off[b1] = pre + k0;
    __syncthreads();
    if (blockIdx.x == 0) {
      if (tid == 0) *status = HSTU_OK;
      for (int64_t b = tid; b <= B; b += kSelThreads) out_off[b] = s_off[b];
    }
  } else {
    if (*status != HSTU_OK) return;
  }
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const int64_t r0 = raw_off[b];
    const int n = (int)(raw_off[b + 1] - r0);
    const int64_t o0 = FUSED ? s_off[b] : out_off[b];
    const int k = (int)((FUSED ? s_off[b + 1] : out_off[b + 1]) - o0);
    if (k <= 0) continue;
    const bool cached = n <= kSlKeyCache;
    auto key_at = [&](int p) -> uint64_t { return cached ? s_key[p] : sl_key(seed, b, p); };
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
        for (int i = tid; i < 256; i += kSelThreads) s_hist[i] = 0;
        __syncthreads();
        for (int p = tid; p < n; p += kSelThreads) {
          uint64_t key;
          if (pass == 0) {
            key = sl_key(seed, b, p);
            if (cached) s_key[p] = key;
          } else {
            key = key_at(p);
          }
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
    // ---- ordered compaction, 4 consecutive positions per thread: a position
    // is kept if its key's fixed digits are below the prefix, or equal to it
    // and among the first `remaining` such positions.  (k == n keeps every
    // position: sh = 64.)
    const uint64_t ph = sh == 64 ? 0 : prefix >> sh;
    int run_lt = 0, run_eq = 0;
    for (int base = 0; base < n; base += kSlChunk) {
      const int p0 = base + tid * kSlPerThread;
      unsigned lt = 0, eq = 0;  // bit j: position p0 + j
#pragma unroll
      for (int j = 0; j < kSlPerThread; ++j) {
        const int p = p0 + j;
        if (p < n) {
          if (sh == 64) {
            lt |= 1u << j;
          } else {
            const uint64_t hi = key_at(p) >> sh;
            lt |= (unsigned)(hi < ph) << j;
            eq |= (unsigned)(hi == ph) << j;
          }
        }
      }
      int tot;
      const int pre =
          block_excl_scan<kSelThreads>((__popc(lt) << 16) | __popc(eq), s_warp, &tot);
      int c_lt = run_lt + (pre >> 16), c_eq = run_eq + (pre & 0xffff);
#pragma unroll
      for (int j = 0; j < kSlPerThread; ++j) {
        const bool l = (lt >> j) & 1, e = (eq >> j) & 1;
        if (l || (e && c_eq < remaining)) {
          const int p = p0 + j;
          out_code[o0 + c_lt + min(c_eq, remaining)] = 2 * (r0 + p) + (p & 1);
        }
        c_lt += l;
        c_eq += e;
      }
      run_lt += tot >> 16;
      run_eq += tot & 0xffff;
    }
    __syncthreads();  // s_key is reused by the next user of this block
  }
}

// Gather, all SMs: every kept row t holds a code in out_ts[t]; its id and
// timestamp are read, the timestamp replaces the code, and the embedding row
// is copied (16 bytes per lane).  A warp takes 8 rows at a time: lanes 0..7
// read the codes, ids and timestamps; the warp then copies two rows at a
// time, 8 loads in flight per lane.
constexpr int kGatherThreads = 256;
constexpr int kGatherRows = 8;
constexpr int kCopyWords = 4;

__global__ void __launch_bounds__(kGatherThreads, 4)
    k_sl_gather(const int64_t* __restrict__ total, const int64_t* __restrict__ ids,
                const int64_t* __restrict__ ts, const __nv_bfloat16* __restrict__ ctab,
                int64_t n_content, const __nv_bfloat16* __restrict__ atab, int64_t n_action,
                int d, __nv_bfloat16* __restrict__ X, int64_t* __restrict__ out_ts, int* status) {
  // No early exit on the status word: a bad id found by one block must not
  // stop the others (bad offsets leave *total = 0, so nothing runs then).
  grid_dep_wait();  // k_sl_select has written every code
  const int lane = threadIdx.x & 31;
  const int64_t T = *total;
  const int d8 = d / 8;
  const int64_t n_batch = (T + kGatherRows - 1) / kGatherRows;
  const int64_t warps = (int64_t)gridDim.x * (kGatherThreads / 32);
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t bt = (int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5);
       bt < n_batch; bt += warps) {
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
    for (int r = 0; r < nb; r += 2) {
      const bool two = r + 1 < nb;
      const uint4* s0 = reinterpret_cast<const uint4*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r));
      const uint4* s1 = reinterpret_cast<const uint4*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), two ? r + 1 : r));
      uint4* d0 = dst + (int64_t)r * d8;
      uint4* d1 = d0 + d8;
      for (int c0 = 0; c0 < d8; c0 += 32 * kCopyWords) {
        uint4 v[2 * kCopyWords];
#pragma unroll
        for (int u = 0; u < kCopyWords; ++u) {
          const int c = c0 + u * 32 + lane;
          v[u] = (c < d8 && s0) ? __ldg(s0 + c) : zero;
          v[kCopyWords + u] = (c < d8 && two && s1) ? __ldg(s1 + c) : zero;
        }
#pragma unroll
        for (int u = 0; u < kCopyWords; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < d8) {
            d0[c] = v[u];
            if (two) d1[c] = v[kCopyWords + u];
          }
        }
      }
    }
  }
}

}  // namespace hstu

// ---------------------------------------------------------------- C ABI
extern "C" {

size_t hstu_sl_embed_workspace_size(void) { return 256; }

int64_t hstu_sl_keep_count(int64_t n) {
  return (n < 0 || n > hstu::kSlMaxLen) ? -1 : hstu::sl_keep(n);
}

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
  // Kernels after the first are launched with programmatic stream
  // serialization: they start while their predecessor runs and wait for it
  // (griddepcontrol.wait) before touching its results.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const bool fused = B <= kSlFusedMaxB;
  if (!fused || raw_total == 0 || B == 0) {
    // validation and kept offsets in their own kernel (also the only launch
    // for an empty raw batch)
    LaunchScope ls(K_SL_OFFSETS, stream);
    k_sl_offsets<<<1, 1024, 0, stream>>>(raw_offsets, B, raw_total, max_raw_len, out_offsets,
                                         status);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  if (B > 0 && raw_total > 0) {
    {
      LaunchScope ls(K_SL_SELECT, stream);
      cfg.blockDim = dim3(kSelThreads);
      cfg.gridDim = dim3((unsigned)(B < 2 * num_sms() ? B : 2 * num_sms()));
      cudaError_t e = fused ? cudaLaunchKernelEx(&cfg, k_sl_select<true>, raw_offsets, B,
                                                 raw_total, max_raw_len, seed, out_offsets,
                                                 out_timestamps, status)
                            : cudaLaunchKernelEx(&cfg, k_sl_select<false>, raw_offsets, B,
                                                 raw_total, max_raw_len, seed, out_offsets,
                                                 out_timestamps, status);
      if (e != cudaSuccess) return HSTU_ERR_CUDA;
    }
    {
      static int per_sm = 0;
      if (per_sm == 0 &&
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_sl_gather, kGatherThreads, 0) !=
              cudaSuccess)
        return HSTU_ERR_CUDA;
      LaunchScope ls(K_SL_GATHER, stream);
      cfg.blockDim = dim3(kGatherThreads);
      cfg.gridDim = dim3((unsigned)(per_sm > 0 ? per_sm : 1) * num_sms());
      if (cudaLaunchKernelEx(&cfg, k_sl_gather, static_cast<const int64_t*>(out_offsets + B),
                             raw_ids, raw_timestamps,
                             static_cast<const __nv_bfloat16*>(content_table), n_content,
                             static_cast<const __nv_bfloat16*>(action_table), n_action,
                             (int)d_model, static_cast<__nv_bfloat16*>(out_X), out_timestamps,
                             status) != cudaSuccess)
        return HSTU_ERR_CUDA;
    }
  }
  return HSTU_OK;
}

}  // extern "C"

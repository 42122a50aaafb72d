// retrieval.cu — full-catalog scoring with top-K selection on the device.
//
// The GenRec explainer on techistory.net (the equation s = E^T h and its
// toy code): the user representation h is the encoder's hidden state at the
// sequence's last position, every catalog item is scored at once by one
// matrix product, and sorting the scores in descending order gives the
// ranking ('NetflixのGenRec解説――LLMを生成させず推薦rankerとして使う', section
// '全体像：LLMは入力を読み、ranking headが作品を採点する').  Here: the K highest
// scores per user, equal scores ordered by ascending item id.
//
// Steps (catalogs of 65,536 items or more): k_ret_gather (optional) copies
// each user's last encoder row into the workspace; the tcgen05 GEMM scores a
// 1-in-16 strided sample of the catalog and the top-K kernels below take each
// user's ks-th best sample score as its threshold; the GEMM then scores the
// whole catalog with an epilogue that only appends the (key, item) pairs at
// or above the user's threshold to a candidate list (the score matrix is
// never written); k_filter_merge picks the K best candidates per user
// exactly.  At least ks sample items reach the threshold, so whenever K or
// more candidates do, they hold the K best; if a user has fewer (or more than
// fit), a device flag makes the direct path below run instead.
// Direct path (smaller catalogs, or that fallback): the GEMM (EPI_SCORE)
// writes the fp32 scores [U, M]; k_topk_chunk selects, per user and
// 8192-item chunk, the chunk's K best items (radix select over
// order-preserving 32-bit keys held in shared memory); k_topk_merge selects
// the K best of those candidates per user and sorts them (bitonic sort of
// (key, id) pairs).
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace hstu {

constexpr int kTopkChunk = 8192;
constexpr int kTopkThreads = 256;
constexpr int kTopkMaxK = 1024;
constexpr int kMergeThreads = 1024;
constexpr uint32_t kPadKey = 0xffffffffu;
constexpr int32_t kPadId = 0x7fffffff;

// Block-wide exclusive scan of one int per thread (NT threads).
template <int NT>
__device__ __forceinline__ int ret_block_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
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

// One radix pass's digit choice (warp 0): among the 256 bins, the bin that
// holds the `remaining`-th smallest key; writes the digit, the rank left
// inside that bin and the bin's size.
__device__ __forceinline__ void ret_pick_digit(const int* s_hist, int remaining, int* s_digit,
                                               int* s_rem, int* s_cnt) {
  const int lane = threadIdx.x & 31;
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
    *s_digit = dgt;
    *s_rem = remaining - acc;
    *s_cnt = s_hist[dgt];
  }
}

// Radix select over n keys (read through key_at) of the k-th smallest, 8 bits
// per pass from the top, stopping once the chosen bin holds exactly the keys
// still to take.  On return *prefix holds the fixed high bits (bits >= *sh;
// *sh = 32 when k == n: everything is taken) and *remaining how many keys
// equal to the prefix on those bits are taken (the first ones in order).
template <int NT, typename KeyAt>
__device__ __forceinline__ void ret_radix_select(int n, int k, KeyAt key_at, int* s_hist,
                                                 int* s_digit, int* s_rem, int* s_cnt,
                                                 uint32_t* prefix, int* remaining, int* sh) {
  const int tid = threadIdx.x;
  uint32_t pre = 0;
  int rem = k, s = 32;
  if (k < n) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += NT) s_hist[i] = 0;
      __syncthreads();
      for (int p = tid; p < n; p += NT) {
        const uint32_t key = key_at(p);
        if (pass == 0 || (key >> s) == (pre >> s)) atomicAdd(&s_hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 32) ret_pick_digit(s_hist, rem, s_digit, s_rem, s_cnt);
      __syncthreads();
      pre |= (uint32_t)*s_digit << shift;
      rem = *s_rem;
      s = shift;
      const bool done = *s_cnt == rem;
      __syncthreads();
      if (done) break;
    }
  }
  *prefix = pre;
  *remaining = rem;
  *sh = s;
}

// The user vectors: h_u = Y[offsets[u+1] - 1] (bf16), zero for an empty
// user; offsets that are not monotone or pass the row count set the status.
__global__ void __launch_bounds__(256)
    k_ret_gather(const __nv_bfloat16* __restrict__ Y, int64_t rows, int d,
                 const int64_t* __restrict__ off, int64_t U, __nv_bfloat16* __restrict__ Hg,
                 int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); u < U;
       u += warps) {
    const int64_t a = off[u], b = off[u + 1];
    const bool bad = a < 0 || b < a || b > rows;
    if (bad && lane == 0) atomicCAS(status, HSTU_OK, HSTU_ERR_BAD_OFFSETS);
    uint4* dst = reinterpret_cast<uint4*>(Hg + u * (int64_t)d);
    if (!bad && b > a) {
      const uint4* src = reinterpret_cast<const uint4*>(Y + (b - 1) * (int64_t)d);
      for (int c = lane; c < d / 8; c += 32) dst[c] = __ldg(src + c);
    } else {
      for (int c = lane; c < d / 8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    }
  }
}

// Ordered compaction of `count` entries (entry j's key through key_at):
// entries whose fixed high bits are below the prefix, or equal to it and
// among the first `remaining` such, are passed in order to emit(idx, j).
// Each thread owns a run of consecutive entries (at most 32).
template <int NT, typename KeyAt, typename Emit>
__device__ __forceinline__ void ret_ordered_emit(int count, uint32_t prefix, int remaining, int sh,
                                                 KeyAt key_at, Emit emit, int* s_warp) {
  const int per = (count + NT - 1) / NT;  // <= 32
  const int j0 = threadIdx.x * per;
  const uint32_t ph = sh == 32 ? 0u : prefix >> sh;
  uint32_t lt = 0, eq = 0;
  for (int tt = 0; tt < per; ++tt) {
    // runs of 32: rotated by the thread index so a warp's lanes hit distinct
    // shared-memory banks (the bitmasks make the visiting order irrelevant)
    const int t = per == 32 ? ((tt + (int)threadIdx.x) & 31) : tt;
    const int j = j0 + t;
    if (j < count) {
      if (sh == 32) {
        lt |= 1u << t;
      } else {
        const uint32_t hi = key_at(j) >> sh;
        lt |= (uint32_t)(hi < ph) << t;
        eq |= (uint32_t)(hi == ph) << t;
      }
    }
  }
  int tot;
  const int pre = ret_block_scan<NT>((__popc(lt) << 16) | __popc(eq), s_warp, &tot);
  int c_lt = pre >> 16, c_eq = pre & 0xffff;
  for (int t = 0; t < per; ++t) {
    const bool l = (lt >> t) & 1u, e = (eq >> t) & 1u;
    if (l || (e && c_eq < remaining)) emit(c_lt + min(c_eq, remaining), j0 + t);
    c_lt += l;
    c_eq += e;
  }
}

// Per (chunk, user): the chunk's k = min(K, n) best items as (key, id)
// candidates in item order, padded to K with (kPadKey, kPadId).
// The k best lie among the positions at least as good as a threshold taken
// from a 1-in-16 sample of the chunk (its ks-th best, ks ~ 2K/16 + 8): at
// least ks sample keys pass it, so when k or more positions pass, they hold
// the k best.  Only those candidates (a few hundred) go through the exact
// radix select; with fewer than k, or more than fit, every position does.
constexpr int kSampleStride = 16;
constexpr int kCandCap = 4096;

__global__ void __launch_bounds__(kTopkThreads)
    k_topk_chunk(const float* __restrict__ S, int64_t ldS, int64_t M, int K, int n_chunks,
                 uint32_t* __restrict__ cand_key, int32_t* __restrict__ cand_id,
                 const int* status, const int* run_if) {
  __shared__ uint32_t s_key[kTopkChunk];
  __shared__ uint16_t s_pos[kCandCap];
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_rem, s_cnt;
  __shared__ int s_warp[kTopkThreads / 32];
  if (run_if && *run_if == 0) return;
  if (*status != HSTU_OK) return;
  const int tid = threadIdx.x;
  const int chunk = blockIdx.x;
  const int64_t u = blockIdx.y;
  const int64_t m0 = (int64_t)chunk * kTopkChunk;
  const int n = (int)min((int64_t)kTopkChunk, M - m0);
  const int k = min(K, n);
  const float* row = S + u * ldS + m0;  // 16-byte aligned: ldS % 4 == 0, m0 % 8192 == 0
  for (int i = tid * 4; i < n; i += kTopkThreads * 4) {
    if (i + 4 <= n) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
      s_key[i] = desc_key(v.x);
      s_key[i + 1] = desc_key(v.y);
      s_key[i + 2] = desc_key(v.z);
      s_key[i + 3] = desc_key(v.w);
    } else {
      for (int j = i; j < n; ++j) s_key[j] = desc_key(__ldg(row + j));
    }
  }
  __syncthreads();
  uint32_t prefix;
  int remaining, sh;
  // ---- candidates: positions at least as good as the sample threshold
  int n_cand = n;  // n_cand == n: every position (no filtering)
  const int ns = (n + kSampleStride - 1) / kSampleStride;
  const int ks = 2 * ((K + kSampleStride - 1) / kSampleStride) + 8;
  if (k < n && ks < ns) {
    ret_radix_select<kTopkThreads>(ns, ks, [&](int i) { return s_key[i * kSampleStride]; },
                                   s_hist, &s_digit, &s_rem, &s_cnt, &prefix, &remaining, &sh);
    // every key whose fixed high bits are <= the prefix's: >= ks sample keys
    const uint32_t thr = prefix | (uint32_t)((1ull << sh) - 1);
    // count and place the passing positions in order (one run of 32 per thread)
    const int p0 = tid * 32;
    uint32_t pass = 0;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) {
      const int jj = (j + tid) & 31;  // rotated: a warp's lanes hit distinct banks
      const int p = p0 + jj;
      if (p < n && s_key[p] <= thr) pass |= 1u << jj;
    }
    int tot;
    const int pre = ret_block_scan<kTopkThreads>(__popc(pass), s_warp, &tot);
    if (tot >= k && tot <= kCandCap) {
      int idx = pre;
      for (int jj = 0; jj < 32; ++jj)
        if ((pass >> jj) & 1u) s_pos[idx++] = (uint16_t)(p0 + jj);
      n_cand = tot;
    }
    __syncthreads();
  }
  const bool filtered = n_cand < n;
  auto cand_key_at = [&](int j) -> uint32_t { return s_key[filtered ? s_pos[j] : j]; };
  ret_radix_select<kTopkThreads>(n_cand, k, cand_key_at, s_hist, &s_digit, &s_rem, &s_cnt,
                                 &prefix, &remaining, &sh);
  uint32_t* ck = cand_key + (u * n_chunks + chunk) * (int64_t)K;
  int32_t* ci = cand_id + (u * n_chunks + chunk) * (int64_t)K;
  ret_ordered_emit<kTopkThreads>(
      n_cand, prefix, remaining, sh, cand_key_at,
      [&](int idx, int j) {
        const int p = filtered ? s_pos[j] : j;
        ck[idx] = s_key[p];
        ci[idx] = (int32_t)(m0 + p);
      },
      s_warp);
  for (int i = k + tid; i < K; i += kTopkThreads) {
    ck[i] = kPadKey;
    ci[i] = kPadId;
  }
}

// Ascending bitonic sort of n (key, id) pairs in shared memory by key, then
// id (padded to a power of two with (kPadKey, kPadId); the arrays hold at
// least that many entries).  Every thread of the block calls it.
template <int NT>
__device__ __forceinline__ void bitonic_sort_pairs(uint32_t* sk, int32_t* si, int n) {
  const int tid = threadIdx.x;
  int P = 1;
  while (P < n) P <<= 1;
  for (int i = n + tid; i < P; i += NT) {
    sk[i] = kPadKey;
    si[i] = kPadId;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P; i += NT) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const uint32_t ki = sk[i], kj = sk[j];
          const int32_t ii = si[i], ij = si[j];
          const bool gt = ki > kj || (ki == kj && ii > ij);  // (key, id) of i after j's
          if (gt == up) {
            sk[i] = kj;
            sk[j] = ki;
            si[i] = ij;
            si[j] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Per user: the K best of its n_cand candidates (item order = id order, so
// equal keys are taken lowest id first), sorted by (key, id).
__global__ void __launch_bounds__(kMergeThreads)
    k_topk_merge(const uint32_t* __restrict__ cand_key, const int32_t* __restrict__ cand_id,
                 int n_cand, int K, float* __restrict__ out_scores, int64_t* __restrict__ out_ids,
                 const int* status, const int* run_if) {
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_rem, s_cnt;
  __shared__ int s_warp[kMergeThreads / 32];
  __shared__ uint32_t s_k[kTopkMaxK];
  __shared__ int32_t s_i[kTopkMaxK];
  if (run_if && *run_if == 0) return;
  if (*status != HSTU_OK) return;
  const int tid = threadIdx.x;
  const int64_t u = blockIdx.x;
  const uint32_t* keys = cand_key + u * (int64_t)n_cand;
  const int32_t* ids = cand_id + u * (int64_t)n_cand;
  uint32_t prefix;
  int remaining, sh;
  ret_radix_select<kMergeThreads>(n_cand, K, [&](int p) { return __ldg(keys + p); }, s_hist,
                                  &s_digit, &s_rem, &s_cnt, &prefix, &remaining, &sh);
  const uint32_t ph = sh == 32 ? 0u : prefix >> sh;
  int run_lt = 0, run_eq = 0;
  for (int base = 0; base < n_cand; base += kMergeThreads * 4) {
    const int p0 = base + tid * 4;
    unsigned lt = 0, eq = 0;
    uint32_t kk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = p0 + j;
      kk[j] = p < n_cand ? __ldg(keys + p) : kPadKey;
      if (p < n_cand) {
        if (sh == 32) {
          lt |= 1u << j;
        } else {
          const uint32_t hi = kk[j] >> sh;
          lt |= (unsigned)(hi < ph) << j;
          eq |= (unsigned)(hi == ph) << j;
        }
      }
    }
    int tot;
    const int pre = ret_block_scan<kMergeThreads>((__popc(lt) << 16) | __popc(eq), s_warp, &tot);
    int c_lt = run_lt + (pre >> 16), c_eq = run_eq + (pre & 0xffff);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool l = (lt >> j) & 1u, e = (eq >> j) & 1u;
      if (l || (e && c_eq < remaining)) {
        const int idx = c_lt + min(c_eq, remaining);
        s_k[idx] = kk[j];
        s_i[idx] = __ldg(ids + p0 + j);
      }
      c_lt += l;
      c_eq += e;
    }
    run_lt += tot >> 16;
    run_eq += tot & 0xffff;
  }
  // sort the K selected pairs by (key, id)
  bitonic_sort_pairs<kMergeThreads>(s_k, s_i, K);
  for (int i = tid; i < K; i += kMergeThreads) {
    out_scores[u * K + i] = key_score(s_k[i]);
    out_ids[u * K + i] = s_i[i];
  }
}

// Per user, after the filtering GEMM: the K best of the candidates that
// reached the user's sample threshold (in no particular order), exactly: a
// radix select of the K-th smallest key, every candidate below it on the
// fixed high bits, and of those equal to it on those bits the best by
// (key, id) after a sort.  Too few or too many candidates, or more equal
// ones than fit, set *fallback (the exact unfused path then runs).
constexpr int kEqCap = 2048;

__global__ void __launch_bounds__(kMergeThreads)
    k_filter_merge(const uint32_t* __restrict__ cand_key, const int32_t* __restrict__ cand_id,
                   const int* __restrict__ cnt, int cap, int K, float* __restrict__ out_scores,
                   int64_t* __restrict__ out_ids, int* fallback, const int* status) {
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_rem, s_cnt;
  __shared__ uint32_t s_k[kTopkMaxK];
  __shared__ int32_t s_i[kTopkMaxK];
  __shared__ uint32_t e_k[kEqCap];
  __shared__ int32_t e_i[kEqCap];
  __shared__ int s_nlt, s_neq;
  if (*status != HSTU_OK) return;
  const int tid = threadIdx.x;
  const int64_t u = blockIdx.x;
  const int n = cnt[u];
  if (n < K || n > cap) {
    if (tid == 0) atomicExch(fallback, 1);
    return;
  }
  const uint32_t* keys = cand_key + u * (int64_t)cap;
  const int32_t* ids = cand_id + u * (int64_t)cap;
  uint32_t prefix;
  int remaining, sh;
  ret_radix_select<kMergeThreads>(n, K, [&](int p) { return __ldg(keys + p); }, s_hist, &s_digit,
                                  &s_rem, &s_cnt, &prefix, &remaining, &sh);
  if (tid == 0) {
    s_nlt = 0;
    s_neq = 0;
  }
  __syncthreads();
  const uint32_t ph = sh == 32 ? 0u : prefix >> sh;
  for (int p = tid; p < n; p += kMergeThreads) {
    const uint32_t key = __ldg(keys + p);
    const uint32_t hi = sh == 32 ? 0u : key >> sh;
    if (sh == 32 || hi < ph) {
      const int idx = atomicAdd(&s_nlt, 1);
      s_k[idx] = key;
      s_i[idx] = __ldg(ids + p);
    } else if (hi == ph) {
      const int idx = atomicAdd(&s_neq, 1);
      if (idx < kEqCap) {
        e_k[idx] = key;
        e_i[idx] = __ldg(ids + p);
      }
    }
  }
  __syncthreads();
  const int nlt = s_nlt, neq = s_neq;
  if (sh != 32) {
    if (neq > kEqCap) {  // (the sort below pads neq to a power of two <= kEqCap)
      if (tid == 0) atomicExch(fallback, 1);
      return;
    }
    bitonic_sort_pairs<kMergeThreads>(e_k, e_i, neq);
    for (int i = tid; i < remaining; i += kMergeThreads) {
      s_k[nlt + i] = e_k[i];
      s_i[nlt + i] = e_i[i];
    }
    __syncthreads();
  }
  bitonic_sort_pairs<kMergeThreads>(s_k, s_i, K);
  for (int i = tid; i < K; i += kMergeThreads) {
    out_scores[u * K + i] = key_score(s_k[i]);
    out_ids[u * K + i] = s_i[i];
  }
}

// Filtering path: a 1-in-kSampleStep sample of the catalog is scored first;
// each user's ks-th best sample score is its threshold.
constexpr int kSampleStep = 16;
constexpr int kFilterCap = 16384;           // candidates kept per user
constexpr int64_t kFilterMinItems = 65536;  // smaller catalogs take the direct path

static int sample_rank(int K) { return 4 * ((K + kSampleStep - 1) / kSampleStep) + 16; }

struct RetLayout {
  size_t hg, scores, ckey, cid;                  // direct path (and fallback)
  size_t s_scores, s_ckey, s_cid, tau, tau_id;   // sample
  size_t fcnt, fkey, fid;                        // filtered candidates
  size_t total;
  int64_t ldS, ldSs, Ms;
  int n_chunks, n_chunks_s, ks;
  bool filter;
};

static bool ret_layout(int64_t U, int64_t M, int32_t d, int32_t K, bool gather, RetLayout* L) {
  if (U < 0 || U > 65535 || M < 1 || M > (1ll << 31) - 256 || d < 64 || d % 64 != 0 || K < 1 ||
      K > kTopkMaxK || K > M)
    return false;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  L->ldS = (M + 63) / 64 * 64;
  L->n_chunks = (int)((M + kTopkChunk - 1) / kTopkChunk);
  L->Ms = (M + kSampleStep - 1) / kSampleStep;
  L->ldSs = (L->Ms + 63) / 64 * 64;
  L->n_chunks_s = (int)((L->Ms + kTopkChunk - 1) / kTopkChunk);
  L->ks = sample_rank(K);
  L->filter = M >= kFilterMinItems && L->ks <= kTopkMaxK && L->ks * 4 <= L->Ms;
  size_t o = 256;  // status word, fallback flag
  L->hg = o;
  o += up(gather ? (size_t)U * d * 2 : 0);
  L->scores = o;
  o += up((size_t)U * L->ldS * 4);
  L->ckey = o;
  o += up((size_t)U * L->n_chunks * K * 4);
  L->cid = o;
  o += up((size_t)U * L->n_chunks * K * 4);
  const int ks = L->filter ? L->ks : 1;
  L->s_scores = o;
  o += up(L->filter ? (size_t)U * L->ldSs * 4 : 0);
  L->s_ckey = o;
  o += up(L->filter ? (size_t)U * L->n_chunks_s * ks * 4 : 0);
  L->s_cid = o;
  o += up(L->filter ? (size_t)U * L->n_chunks_s * ks * 4 : 0);
  L->tau = o;
  o += up(L->filter ? (size_t)U * ks * 4 : 0);
  L->tau_id = o;
  o += up(L->filter ? (size_t)U * ks * 8 : 0);
  L->fcnt = o;
  o += up(L->filter ? (size_t)U * 4 : 0);
  L->fkey = o;
  o += up(L->filter ? (size_t)U * kFilterCap * 4 : 0);
  L->fid = o;
  o += up(L->filter ? (size_t)U * kFilterCap * 4 : 0);
  L->total = o;
  return (int64_t)L->n_chunks * K <= (1ll << 30);
}

}  // namespace hstu

// ---------------------------------------------------------------- C ABI
extern "C" {

size_t hstu_retrieval_workspace_size(int64_t U, int64_t M, int32_t d, int32_t K,
                                     int32_t from_rows) {
  hstu::RetLayout L;
  return hstu::ret_layout(U, M, d, K, from_rows != 0, &L) ? L.total : 0;
}

hstu_status hstu_retrieval_topk(int64_t U, int64_t M, int32_t d, const void* H,
                                const int64_t* user_offsets, int64_t total_rows, const void* E,
                                int32_t K, float* out_scores, int64_t* out_ids, void* ws,
                                size_t ws_bytes, void* stream_ptr) {
  using namespace hstu;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const bool gather = user_offsets != nullptr;
  RetLayout L;
  if (!ret_layout(U, M, d, K, gather, &L)) return HSTU_ERR_INVALID_ARG;
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return HSTU_ERR_WORKSPACE;
  if (U == 0)  // nothing to score; the status word still reflects this call
    return cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream_ptr)) == cudaSuccess
               ? HSTU_OK
               : HSTU_ERR_CUDA;
  if (!H || !E || !out_scores || !out_ids) return HSTU_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(H) & 15) || (reinterpret_cast<uintptr_t>(E) & 15))
    return HSTU_ERR_INVALID_ARG;
  if (gather && total_rows < 0) return HSTU_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w);
  int* fallback = status + 1;
  if (cudaMemsetAsync(w, 0, 256, stream) != cudaSuccess) return HSTU_ERR_CUDA;
  if (L.filter && cudaMemsetAsync(w + L.fcnt, 0, (size_t)U * 4, stream) != cudaSuccess)
    return HSTU_ERR_CUDA;
  const void* A = H;
  if (gather) {
    LaunchScope ls(K_RET_GATHER, stream);
    const int grid = (int)std::min<int64_t>((U + 7) / 8, 4 * num_sms());
    k_ret_gather<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(H), total_rows, d,
                                           user_offsets, U,
                                           reinterpret_cast<__nv_bfloat16*>(w + L.hg), status);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    A = w + L.hg;
  }
  // the exact direct path: every score written, per-chunk top-K, merge;
  // with run_if set it runs only if the filtering path gave up
  auto direct = [&](const int* run_if) -> hstu_status {
    float* S = reinterpret_cast<float*>(w + L.scores);
    if (launch_gemm_scores(A, d, E, d, 0, U, M, d, S, L.ldS, status, stream, K_GEMM_SCORES, 1,
                           run_if) != cudaSuccess)
      return HSTU_ERR_CUDA;
    uint32_t* ck = reinterpret_cast<uint32_t*>(w + L.ckey);
    int32_t* ci = reinterpret_cast<int32_t*>(w + L.cid);
    {
      LaunchScope ls(K_TOPK_CHUNK, stream);
      k_topk_chunk<<<dim3((unsigned)L.n_chunks, (unsigned)U), kTopkThreads, 0, stream>>>(
          S, L.ldS, M, K, L.n_chunks, ck, ci, status, run_if);
      if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    }
    {
      LaunchScope ls(K_TOPK_MERGE, stream);
      k_topk_merge<<<(unsigned)U, kMergeThreads, 0, stream>>>(ck, ci, L.n_chunks * K, K,
                                                             out_scores, out_ids, status, run_if);
      if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    }
    return HSTU_OK;
  };
  if (!L.filter) return direct(nullptr);
  // ---- threshold per user from a strided sample of the catalog
  const int ks = L.ks;
  float* Ss = reinterpret_cast<float*>(w + L.s_scores);
  if (launch_gemm_scores(A, d, E, d, 0, U, L.Ms, d, Ss, L.ldSs, status, stream, K_GEMM_SCORES,
                         kSampleStep) != cudaSuccess)
    return HSTU_ERR_CUDA;
  float* tau = reinterpret_cast<float*>(w + L.tau);
  {
    uint32_t* sck = reinterpret_cast<uint32_t*>(w + L.s_ckey);
    int32_t* sci = reinterpret_cast<int32_t*>(w + L.s_cid);
    LaunchScope ls(K_TOPK_CHUNK, stream);
    k_topk_chunk<<<dim3((unsigned)L.n_chunks_s, (unsigned)U), kTopkThreads, 0, stream>>>(
        Ss, L.ldSs, L.Ms, ks, L.n_chunks_s, sck, sci, status, nullptr);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    LaunchScope ls2(K_TOPK_MERGE, stream);
    k_topk_merge<<<(unsigned)U, kMergeThreads, 0, stream>>>(
        sck, sci, L.n_chunks_s * ks, ks, tau, reinterpret_cast<int64_t*>(w + L.tau_id), status,
        nullptr);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  // ---- every score at or above the user's threshold becomes a candidate
  uint32_t* fk = reinterpret_cast<uint32_t*>(w + L.fkey);
  int32_t* fi = reinterpret_cast<int32_t*>(w + L.fid);
  int* fc = reinterpret_cast<int*>(w + L.fcnt);
  if (launch_gemm_filter(A, d, E, d, 0, U, M, d, tau + (ks - 1), ks, fk, fi, fc, kFilterCap,
                         fallback, status, stream, K_GEMM_FILTER) != cudaSuccess)
    return HSTU_ERR_CUDA;
  {
    LaunchScope ls(K_FILTER_MERGE, stream);
    k_filter_merge<<<(unsigned)U, kMergeThreads, 0, stream>>>(fk, fi, fc, kFilterCap, K, out_scores,
                                                             out_ids, fallback, status);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return direct(fallback);
}

hstu_status hstu_retrieval_fallback_taken(const void* workspace, size_t workspace_bytes,
                                          int32_t* taken, void* stream) {
  if (!workspace || workspace_bytes < 256 || !taken) return HSTU_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(taken, static_cast<const int32_t*>(workspace) + 1, sizeof(int32_t),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  return HSTU_OK;
}

}  // extern "C"


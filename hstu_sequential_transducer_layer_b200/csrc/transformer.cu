// transformer.cu — a softmax-Transformer encoder layer, the comparator of the
// HSTU layer, on the same jagged batches.
//
// The GenRec explainer on techistory.net (attention equations and its toy
// self-attention): Q = X W_Q, K = X W_K, V = X W_V, per head
// softmax(Q K^T / sqrt(d_k)) V, heads concatenated and projected by W_O.
// 'HSTUとGenerative Recommenders', section '2. QKᵀで「どの履歴を見るか」を決める':
// an ordinary Transformer turns each query's scores into weights summing to
// 1 with a softmax (HSTU uses SiLU instead); section 'Production評価の12.4%を
// どう読むか': the comparison against a FlashAttention-2 Transformer at 8,192
// tokens, d = 512, 8 heads.  The layer (pre-LayerNorm, causal per user):
//   A = LN1(X); [Q|K|V] = A W_QKV^T; ctx = causal softmax attention;
//   X1 = X + ctx W_O^T; Y = X1 + SiLU(LN2(X1) W_1^T + b_1) W_2^T + b_2.
//
// k_softmax_attn: one work item = (user, 128-row query tile, head) from the
// same causal work list as the HSTU attention (only tiles at or left of the
// diagonal).  Warp 0 loads Q (lane 0, with the K tiles) and V (lane 1) by TMA
// through 2-stage rings; warp 1 issues S = Q K^T (two TMEM buffers) and
// O += P V (P from TMEM); warps 4-11 hold the score rows, two threads per
// query row (64 columns each, in registers), which exchange their row maxima
// and sums through shared memory.  Online softmax in base 2: the running maximum moves only
// when a tile's maximum exceeds it by more than 8 (then O is rescaled in TMEM
// by 2^(m_old - m_new)), so P = 2^(x - m) stays below 256 and fits fp16.  At
// the end of an item the row of O is divided by the running sum and stored.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>
#include <type_traits>

#include "ptx.cuh"

namespace hstu {

struct SoftmaxAttnDev {
  const AttnItem* items;
  const int32_t* n_items;
  int q_col, k_col, v_col;
  float scale_log2;             // log2(e) / sqrt(D)
  __half* ctx;                  // [T, h*D]
  int64_t ldc;
  int* status;
};

template <int D>
struct SmaxCfg {
  static constexpr uint32_t TILE = 128u * D * 2;
  static constexpr int NA = D / 64;
  static constexpr uint32_t Q_OFF = 0, K_OFF = 2 * TILE, V_OFF = 4 * TILE;
  static constexpr uint32_t BAR_OFF = 6 * TILE;
  static constexpr uint32_t XCH_OFF = BAR_OFF + 256;  // [2 parities][2 halves][128 rows] floats
  static constexpr uint32_t SMEM = XCH_OFF + 2 * 2 * 128 * 4 + 1024;
  static constexpr uint32_t O_COL = 256;  // TMEM: S0 | S1 | O
  // warp 0 loads, 1 MMA, 4-7 and 8-11 softmax (columns 0-63 / 64-127 of S)
  static constexpr int THREADS = 384;
};

DEVI float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Item k of this CTA: items are sorted longest first; CTA c takes c,
// 2G-1-c, 2G+c, 4G-1-c, ... so every CTA gets a similar mix.
DEVI int snake_item(int k, int c, int G) {
  return (k >> 1) * 2 * G + ((k & 1) ? (2 * G - 1 - c) : c);
}

template <int D>
__global__ void __launch_bounds__(SmaxCfg<D>::THREADS, 1)
    k_softmax_attn(const __grid_constant__ CUtensorMap tmQKV, const SoftmaxAttnDev a) {
  using C = SmaxCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars + 0;    // [2]
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* k_full = bars + 4;    // [2]
  uint64_t* k_empty = bars + 6;   // [2]
  uint64_t* v_full = bars + 8;    // [2]
  uint64_t* v_empty = bars + 10;  // [2]
  uint64_t* s_full = bars + 12;   // [2]
  uint64_t* p_full = bars + 14;   // [2]
  uint64_t* o_done = bars + 16;   // one phase per P.V
  uint64_t* o_free = bars + 17;   // one phase per item (O read out)
  uint64_t* drain = bars + 18;
  uint64_t* xch = bars + 19;      // [4] per lane quarter: the two halves of a row met
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
  int* s_go = reinterpret_cast<int*>(ab + 1);
  int* s_nitems = s_go + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    const int st = a.status ? *reinterpret_cast<volatile int*>(a.status) : 0;
    *s_go = (st == 0);
    *s_nitems = *a.n_items;
    ab->flag = 0;
    ab->limit_us = kWaitLimitUs;
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 8);
    }
    mbar_init(o_done, 1);
    mbar_init(o_free, 8);
    for (int i = 0; i < 4; ++i) mbar_init(xch + i, 2);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmQKV);
  __syncthreads();
  if (!*s_go) return;
  const int n_items = *s_nitems;
  const int G = gridDim.x, cta = blockIdx.x;

  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;

  if (warp == 0) {
    // ------------------------------------------------ TMA loaders
    if (lane < 2) {
      const bool kq = lane == 0;
      uint64_t* full = kq ? k_full : v_full;
      uint64_t* empty = kq ? k_empty : v_empty;
      uint8_t* buf = kq ? sK : sV;
      const int col = kq ? a.k_col : a.v_col;
      uint32_t st = 0, ph = 0, issued = 0, last_par = 0, q_issued = 0, q_last = 0;
      bool ok = true;
      for (int k = 0;; ++k) {
        const int it = snake_item(k, cta, G);
        if (it >= n_items) break;
        const AttnItem w = a.items[it];
        if (kq) {
          const int qs = k & 1;
          if (!mbar_wait(q_empty + qs, ((k >> 1) & 1) ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(q_full + qs, C::TILE);
#pragma unroll
          for (int at = 0; at < C::NA; ++at)
            tma_load_2d(sQ + qs * C::TILE + at * 16384, &tmQKV, a.q_col + w.head * D + at * 64,
                        w.q_row0, q_full + qs);
          q_issued |= 1u << qs;
          q_last = (q_last & ~(1u << qs)) | ((uint32_t)((k >> 1) & 1) << qs);
        }
        for (int j = 0; j < w.nkv; ++j) {
          if (!mbar_wait(empty + st, ph ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + st, C::TILE);
#pragma unroll
          for (int at = 0; at < C::NA; ++at)
            tma_load_2d(buf + st * C::TILE + at * 16384, &tmQKV, col + w.head * D + at * 64,
                        w.kv_row0 + j * 128, full + st);
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (ph << st);
          if (++st == 2) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
      }
      if (!ok) {  // let every load already in flight land before the CTA exits
        AbortState tmp{0, kWaitLimitUs};
        for (uint32_t s2 = 0; s2 < 2; ++s2) {
          if ((issued >> s2) & 1u) mbar_wait(full + s2, (last_par >> s2) & 1u, &tmp, nullptr);
          if ((q_issued >> s2) & 1u) mbar_wait(q_full + s2, (q_last >> s2) & 1u, &tmp, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f16_f32(128, 128, 0, 0, 1);
      constexpr uint32_t IDESC_O = idesc_f16_f32(128, D, 0, 1, 1);  // V is MN-major
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0, scount = 0, pcount = 0;
      bool ok = true, any = false;
      auto issue_pv = [&](int jj, int li) -> bool {
        const int pb = (int)(pcount & 1);  // P_j sits in S_j's buffer
        if (!mbar_wait(p_full + pb, (pcount >> 1) & 1, ab, a.status)) return false;
        if (jj == 0 && !mbar_wait(o_free, (li & 1) ^ 1, ab, a.status)) return false;
        if (!mbar_wait(v_full + vst, vph, ab, a.status)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sV + vst * C::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // 16 KV rows per MMA = 8 packed P columns
          tc_mma_f16_ts(tmem + C::O_COL, tmem + pb * 128 + kk * 8,
                        sdesc_sw128(v_base + kk * 2048, 16384, 1024), IDESC_O,
                        (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(v_empty + vst);
        tc_commit(o_done);
        if (++vst == 2) {
          vst = 0;
          vph ^= 1;
        }
        ++pcount;
        any = true;
        return true;
      };
      int pend_j = -1, pend_li = 0;
      auto flush = [&]() -> bool {
        if (pend_j < 0) return true;
        const bool r = issue_pv(pend_j, pend_li);
        pend_j = -1;
        return r;
      };
      for (int k = 0; ok; ++k) {
        const int it = snake_item(k, cta, G);
        if (it >= n_items) break;
        const AttnItem w = a.items[it];
        const int qs = k & 1;
        const uint32_t q_base = smem_u32(sQ + qs * C::TILE);
        if (!mbar_wait(q_full + qs, (k >> 1) & 1, ab, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < w.nkv; ++j) {
          if (!mbar_wait(k_full + kst, kph, ab, a.status)) {
            ok = false;
            break;
          }
          // S_j reuses the buffer of S_{j-2}, whose P was read by a P.V
          // issued before this MMA (MMAs run in issue order)
          const int sb = scount & 1;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + kst * C::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc_mma_f16_ss(tmem + sb * 128,
                          sdesc_sw128(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                          sdesc_sw128(k_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                          IDESC_S, kk > 0 ? 1u : 0u);
          tc_commit(s_full + sb);
          tc_commit(k_empty + kst);
          if (j == w.nkv - 1) tc_commit(q_empty + qs);
          if (++kst == 2) {
            kst = 0;
            kph ^= 1;
          }
          ++scount;
          any = true;
          if (!flush()) {
            ok = false;
            break;
          }
          pend_j = j;
          pend_li = k;
        }
      }
      if (ok) flush();
      if (any) {
        tc_commit(drain);
        AbortState tmp{0, kWaitLimitUs};
        mbar_wait(drain, 0, &tmp, nullptr);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax warps: half a row each
    // Warps 4-7 take columns 0-63 of their lane quarter's 32 rows, warps 8-11
    // columns 64-127; the two halves of a row exchange their maxima (each
    // tile) and sums (each item) through shared memory, meeting on the lane
    // quarter's mbarrier (bounded waits).
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const float sl2 = a.scale_log2;
    float* xbuf = reinterpret_cast<float*>(smem + C::XCH_OFF);  // [par][half][128]
    uint32_t scount = 0, pvwait = 0, nx = 0;
    bool alive = true;
    // publish v, meet the partner, return the partner's value
    auto exchange = [&](float v) -> float {
      const int par = nx & 1;
      xbuf[(par * 2 + half) * 128 + r] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(xch + q);
      if (!mbar_wait_warp(xch + q, par, ab, a.status)) {
        alive = false;
        return 0.f;
      }
      ++nx;
      return xbuf[(par * 2 + (half ^ 1)) * 128 + r];
    };
    for (int k = 0; alive; ++k) {
      const int it = snake_item(k, cta, G);
      if (it >= n_items) break;
      const AttnItem w = a.items[it];
      const int rows_valid = min(128, w.n_q - (int)w.qt * 128);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < w.nkv; ++j) {
        const int sb = scount & 1;
        if (!mbar_wait_warp(s_full + sb, (scount >> 1) & 1, ab, a.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_addr = tmem + sb * 128 + half * 64 + lane_base;
        uint32_t sr[64];
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_ld_wait();
        float pm = -INFINITY;
        if (j == (int)w.qt) {  // diagonal tile: column c > row r is masked
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            float x = __uint_as_float(sr[c]) * sl2;
            if (half * 64 + c > r) x = -INFINITY;
            sr[c] = __float_as_uint(x);
            pm = fmaxf(pm, x);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float x = __uint_as_float(sr[c]) * sl2;
            sr[c] = __float_as_uint(x);
            pm = fmaxf(pm, x);
          }
        }
        // both halves have read their S columns once they meet here, so the
        // P writes below cannot overwrite scores the partner still needs
        const float mt = fmaxf(pm, exchange(pm));
        if (!alive) break;
        const bool resc = mt > m + 8.f;
        const float m_new = resc ? mt : m;
        const float alpha = resc ? ex2_approx(m - m_new) : 1.f;
        float ls = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2_approx(__uint_as_float(sr[2 * c]) - m_new);
          const float p1 = ex2_approx(__uint_as_float(sr[2 * c + 1]) - m_new);
          ls += p0 + p1;
          pk[c] = pack_f16x2_sat(p0, p1);
        }
        // this half of O is rescaled once the previous P.V has landed in it
        // (tile 0's P.V overwrites O, so it needs none)
        if (j > 0) {
          if (!mbar_wait_warp(o_done, pvwait & 1, ab, a.status)) {
            alive = false;
            break;
          }
          ++pvwait;
          if (__any_sync(0xffffffffu, resc)) {
            tc_fence_after();
#pragma unroll
            for (int c16 = 0; c16 < D / 32; ++c16) {
              const uint32_t oa = tmem + C::O_COL + half * (D / 2) + c16 * 16 + lane_base;
              uint32_t o[16];
              tmem_ld16(oa, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st16(oa, o);
            }
          }
        }
        tmem_st32(tmem + sb * 128 + half * 32 + lane_base, pk);
        tmem_st_wait();
        l = l * alpha + ls;
        m = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + sb);
        ++scount;
      }
      if (!alive) break;
      // ---- epilogue: this half of O / (both halves' sums)
      if (!mbar_wait_warp(o_done, pvwait & 1, ab, a.status)) break;
      ++pvwait;
      tc_fence_after();
      uint32_t o[D / 2];
#pragma unroll
      for (int c16 = 0; c16 < D / 32; ++c16)
        tmem_ld16(tmem + C::O_COL + half * (D / 2) + c16 * 16 + lane_base,
                  *reinterpret_cast<uint32_t(*)[16]>(o + c16 * 16));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);  // the next item's first P.V may overwrite O
      const float lt = l + exchange(l);
      if (!alive) break;
      if (r < rows_valid) {
        const float inv = 1.f / lt;
        uint4* dst = reinterpret_cast<uint4*>(a.ctx + (int64_t)(w.q_row0 + r) * a.ldc + w.head * D +
                                              half * (D / 2));
#pragma unroll
        for (int c8 = 0; c8 < D / 16; ++c8) {
          uint4 v;
          v.x = pack_f16x2_sat(__uint_as_float(o[c8 * 8 + 0]) * inv, __uint_as_float(o[c8 * 8 + 1]) * inv);
          v.y = pack_f16x2_sat(__uint_as_float(o[c8 * 8 + 2]) * inv, __uint_as_float(o[c8 * 8 + 3]) * inv);
          v.z = pack_f16x2_sat(__uint_as_float(o[c8 * 8 + 4]) * inv, __uint_as_float(o[c8 * 8 + 5]) * inv);
          v.w = pack_f16x2_sat(__uint_as_float(o[c8 * 8 + 6]) * inv, __uint_as_float(o[c8 * 8 + 7]) * inv);
          dst[c8] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// LayerNorm of one row per warp (d % 256 == 0, d <= 1024): fp32 statistics
// (two passes over the row held in registers), gamma/beta bf16, fp16 out.
template <typename Tin>
__global__ void __launch_bounds__(256)
    k_ln_plain(const Tin* __restrict__ X, int64_t T, int d, const __nv_bfloat16* __restrict__ gamma,
               const __nv_bfloat16* __restrict__ beta, float eps, __half* __restrict__ Y,
               const int* status) {
  if (*status != HSTU_OK) return;
  constexpr int kMaxPer = 4;  // 256-element chunks per row
  const int lane = threadIdx.x & 31;
  const int per = d / 256;
  const int64_t warps = (int64_t)gridDim.x * 8;
  for (int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); row < T; row += warps) {
    float v[kMaxPer][8];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      if (i < per) {
        const uint4 u = *reinterpret_cast<const uint4*>(X + row * d + (i * 32 + lane) * 8);
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (sizeof(Tin) == 2 && std::is_same<Tin, __half>::value) {
            v[i][2 * k] = f16lo(wv[k]);
            v[i][2 * k + 1] = f16hi(wv[k]);
          } else {
            v[i][2 * k] = bf16lo(wv[k]);
            v[i][2 * k + 1] = bf16hi(wv[k]);
          }
          sum += v[i][2 * k] + v[i][2 * k + 1];
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / (float)d;
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
      if (i < per)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float c = v[i][k] - mean;
          sq += c * c;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = rsqrtf(sq / (float)d + eps);
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      if (i < per) {
        const int c0 = (i * 32 + lane) * 8;
        const uint4 gu = *reinterpret_cast<const uint4*>(gamma + c0);
        const uint4 bu = *reinterpret_cast<const uint4*>(beta + c0);
        const uint32_t gw[4] = {gu.x, gu.y, gu.z, gu.w}, bw[4] = {bu.x, bu.y, bu.z, bu.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          o[k] = pack_f16x2_sat((v[i][2 * k] - mean) * rstd * bf16lo(gw[k]) + bf16lo(bw[k]),
                                (v[i][2 * k + 1] - mean) * rstd * bf16hi(gw[k]) + bf16hi(bw[k]));
        *reinterpret_cast<uint4*>(Y + row * d + c0) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

struct TfLayout {
  size_t items, ubase, zeros, a, qkv, ctx, x1, f, total;
  int64_t item_cap;
};

static bool tf_layout(int32_t d, int32_t h, int32_t ff, int64_t B, int64_t T, TfLayout* L) {
  if (d <= 0 || h <= 0 || d % h != 0 || ff <= 0 || B < 0 || T < 0) return false;
  const int D = d / h;
  if (d % 256 != 0 || d > 1024 || (D != 64 && D != 128) || ff % 256 != 0) return false;
  if (T > (1ll << 31) - 1024 || B > (1ll << 30)) return false;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  L->item_cap = ((T + kTile - 1) / kTile + B) * (int64_t)h;
  size_t o = sizeof(Header) <= 256 ? 256 : up(sizeof(Header));
  L->items = o;
  o += up((size_t)L->item_cap * sizeof(AttnItem));
  L->ubase = o;
  o += up((size_t)(B + 1) * 8);
  L->zeros = o;
  o += up((size_t)3 * d * 2);
  L->a = o;
  o += up((size_t)T * d * 2);
  L->qkv = o;
  o += up((size_t)T * 3 * d * 2);
  L->ctx = o;
  o += up((size_t)T * d * 2);
  L->x1 = o;
  o += up((size_t)T * d * 2);
  L->f = o;
  o += up((size_t)T * ff * 2);
  L->total = o;
  return true;
}

template <int D>
static cudaError_t launch_softmax_attn(const CUtensorMap& tm, const SoftmaxAttnDev& dev,
                                       cudaStream_t s) {
  using C = SmaxCfg<D>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(k_softmax_attn<D>), C::SMEM);
  if (e != cudaSuccess) return e;
  LaunchScope ls(K_TF_ATTN, s);
  k_softmax_attn<D><<<num_sms(), C::THREADS, C::SMEM, s>>>(tm, dev);
  return cudaGetLastError();
}

}  // namespace hstu

// ---------------------------------------------------------------- C ABI
extern "C" {

size_t hstu_transformer_workspace_size(int32_t d_model, int32_t n_heads, int32_t d_ff, int64_t B,
                                       int64_t total_tokens) {
  hstu::TfLayout L;
  return hstu::tf_layout(d_model, n_heads, d_ff, B, total_tokens, &L) ? L.total : 0;
}

hstu_status hstu_transformer_layer_fwd(int32_t d_model, int32_t n_heads, int32_t d_ff, float ln_eps,
                                       const hstu_transformer_weights* w, int64_t B,
                                       int64_t total_tokens, int64_t max_len,
                                       const int64_t* offsets, const void* X, void* out, void* ws,
                                       size_t ws_bytes, void* stream_ptr) {
  using namespace hstu;
  cudaStream_t s = static_cast<cudaStream_t>(stream_ptr);
  TfLayout L;
  const int64_t T = total_tokens;
  if (!tf_layout(d_model, n_heads, d_ff, B, T, &L)) return HSTU_ERR_INVALID_ARG;
  if (max_len < 1 || max_len > (1ll << 30)) return HSTU_ERR_INVALID_ARG;
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return HSTU_ERR_WORKSPACE;
  if (!w || !offsets || (T > 0 && (!X || !out))) return HSTU_ERR_INVALID_ARG;
  const void* wp[10] = {w->ln1_gamma, w->ln1_beta, w->W_qkv, w->W_o, w->ln2_gamma,
                        w->ln2_beta, w->W_1, w->b_1, w->W_2, w->b_2};
  for (const void* p : wp)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15)) return HSTU_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return HSTU_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  Header* hdr = reinterpret_cast<Header*>(base);
  int* status = &hdr->status;
  const int d = d_model, h = n_heads, D = d / h, ff = d_ff;
  auto at = [&](size_t off) { return static_cast<void*>(base + off); };
  __half* A = static_cast<__half*>(at(L.a));
  __half* QKV = static_cast<__half*>(at(L.qkv));
  __half* ctx = static_cast<__half*>(at(L.ctx));
  __half* X1 = static_cast<__half*>(at(L.x1));
  __half* F = static_cast<__half*>(at(L.f));
  if (cudaMemsetAsync(at(L.zeros), 0, (size_t)3 * d * 2, s) != cudaSuccess) return HSTU_ERR_CUDA;
  launch_schedule(offsets, B, T, max_len, h, static_cast<AttnItem*>(at(L.items)), L.item_cap,
                  static_cast<int64_t*>(at(L.ubase)), INT32_MAX, hdr, s);
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  if (T == 0) return HSTU_OK;
  const int ln_grid = (int)std::min<int64_t>((T + 7) / 8, 8 * num_sms());
  {
    LaunchScope ls(K_TF_LN, s);
    k_ln_plain<__nv_bfloat16><<<ln_grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(X), T, d, static_cast<const __nv_bfloat16*>(w->ln1_gamma),
        static_cast<const __nv_bfloat16*>(w->ln1_beta), ln_eps, A, status);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  auto gemm = [&](const void* a_, int64_t lda, const void* W, int N, int K, const void* bias,
                  void* o, int o_f16, int64_t ldo, int epi, const void* resid, int64_t ldr,
                  int rk, int kid) {
    GemmCall g{};
    g.A = a_;
    g.lda = lda;
    g.W = W;
    g.ldw = K;
    g.ab_f16 = 1;
    g.M_cap = T;
    g.M_dev = nullptr;
    g.N = N;
    g.K = K;
    g.n_off = 0;
    g.bias = bias;
    g.out = o;
    g.out_f16 = o_f16;
    g.ldo = ldo;
    g.out32 = nullptr;
    g.resid = resid;
    g.ldr = ldr;
    g.resid_kind = rk;
    g.epi = epi;
    g.status = status;
    return launch_gemm_tc(g, s, kid);
  };
  if (gemm(A, d, w->W_qkv, 3 * d, d, at(L.zeros), QKV, 1, 3 * d, EPI_BIAS, nullptr, 0, 0,
           K_TF_QKV) != cudaSuccess)
    return HSTU_ERR_CUDA;
  CUtensorMap tm;
  if (!encode_tmap_2d(&tm, QKV, (uint64_t)T, (uint64_t)3 * d, (uint64_t)3 * d * 2, 64, 128, true))
    return HSTU_ERR_CUDA;
  SoftmaxAttnDev dev{};
  dev.items = static_cast<const AttnItem*>(at(L.items));
  dev.n_items = &hdr->n_items;
  dev.q_col = 0;
  dev.k_col = d;
  dev.v_col = 2 * d;
  dev.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dev.ctx = ctx;
  dev.ldc = d;
  dev.status = status;
  if ((D == 64 ? launch_softmax_attn<64>(tm, dev, s) : launch_softmax_attn<128>(tm, dev, s)) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  if (gemm(ctx, d, w->W_o, d, d, at(L.zeros), X1, 1, d, EPI_RESID, X, d, RESID_BF16,
           K_TF_OPROJ) != cudaSuccess)
    return HSTU_ERR_CUDA;
  {
    LaunchScope ls(K_TF_LN, s);
    k_ln_plain<__half><<<ln_grid, 256, 0, s>>>(X1, T, d,
                                               static_cast<const __nv_bfloat16*>(w->ln2_gamma),
                                               static_cast<const __nv_bfloat16*>(w->ln2_beta),
                                               ln_eps, A, status);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  if (gemm(A, d, w->W_1, ff, d, w->b_1, F, 1, ff, EPI_SILU, nullptr, 0, 0, K_TF_FFN1) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  if (gemm(F, ff, w->W_2, d, ff, w->b_2, out, 0, d, EPI_RESID, X1, d, RESID_F16, K_TF_FFN2) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  return HSTU_OK;
}

}  // extern "C"

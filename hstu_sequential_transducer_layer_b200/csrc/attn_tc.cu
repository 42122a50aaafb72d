// attn_tc.cu — pointwise (softmax-free) attention with the relative bias on
// the tcgen05 tensor cores, over jagged batches.
//
// 'HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか',
// subsection '2. QKᵀで「どの履歴を見るか」を決める': per head,
//   s_ij = Q_i.K_j + pos_bias(i - j) + time_bias(t_i - t_j), j <= i,
//   O_i  = (1/n) sum_j SiLU(s_ij) V_j          (no softmax, no running max)
// and section '長い履歴を現実の計算量へ収める4つの工夫', subsection
// '4. M-FALCONで候補間の履歴計算を共有する': candidates attend to their user's
// whole cached history and to themselves only.
//
// One work item = (user, 128-row query tile, head).  The schedule lists, for
// each item, only the KV tiles at or left of the causal diagonal, so fully
// masked tiles are never loaded or multiplied.  Items are taken dynamically
// (one atomic counter per launch) in an order that keeps the q-tiles of one
// (user, head) adjacent, so CTAs running at the same time read the same K/V
// tiles from L2.  Because there is no softmax, KV tiles combine by plain
// accumulation in TMEM.
//
// Roles (768 threads, six warpgroups): warp 2 claims items and publishes them
// into a 2-slot ring; warp 0 issues the TMA loads (lane 0: Q once per item and
// the K tiles, lane 1: the V tiles, each through a 2-stage ring); warp 1
// issues the MMAs: S = Q K^T into one of two TMEM buffers, then O += P V (P
// from TMEM) into a TMEM accumulator; warps 4-19 ("P warps", four per TMEM
// lane quarter, 32 of the 128 columns each) read S with tcgen05.ld, add the
// bias, apply SiLU, mask, round to fp16 and write P back into TMEM (two
// buffers), from where the P.V MMA reads its A operand; warps 20-23 (one per
// lane quarter) read O at the end of an item, scale by 1/n (and, for
// candidates, add the self term), and store its mean and deviation per
// (row, head) and the normalised values in fp16 through TMA bulk stores
// (the statistics let the output projection apply LayerNorm without another
// pass over O) while the P warps already work on the next item.  Sixteen P warps with little
// state each hide the latency of the bias look-ups better than fewer warps
// with more registers; every role fits in 80 registers.
// Bias per element (causal self-attention): the position bias comes from a
// per-warp window of the 63 distances its 32 x 32 block spans; the time
// bucket comes precomputed (one byte per element, shared by all heads and
// layers of a call) and indexes the head's table, which the producer warp
// stores next to the item in the ring.  Both tables hold half the bias so that
// y = s/2 + bias/2 feeds SiLU(x) = y + y tanh(y) (x = 2y) directly.  The P
// warps fetch the next tile's bucket words and window while computing the
// current tile.  For candidates the bias depends only on the history column:
// one shared-memory broadcast per element.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "ptx.cuh"

namespace hstu {

struct AttnDev {
  const AttnItem* items;
  const int32_t* n_items;
  const int64_t* q_off;
  const int64_t* kv_off;
  const int32_t* t_rel;
  const int32_t* t_req_rel;
  const uint32_t* tbuckets;
  const float* rab_pos;
  const float* rab_time;
  int Np, Nt, Sp, St;
  int q_col, k_col, v_col;
  const __half* q_buf;         // for the candidate self term (fp16 f1 output)
  int64_t ld_f1;
  // O of each (row, head), stored as its mean m and standard deviation s over
  // the head's D values (fp32, [rows, h]) and the normalised values
  // (O - m) / s in fp16 ([rows, ldo]).  LayerNorm subtracts a mean that is
  // most of O's magnitude; normalised values keep fp16's relative precision
  // for what remains, and the statistics give LayerNorm's row moments exactly.
  __half* O;
  int64_t ldo;
  float2* ostats;
  int32_t* work_next;
  int32_t* work_done;
  int* status;
  int h;                       // heads (row stride of ostats)
  uint32_t wait_limit_us;      // bound of every in-kernel wait
  int inject_stall;            // test hook: CTA 0 stops handing out work after two items
};

template <int D>
struct AttnCfg {
  static constexpr int NA = D / 64;                       // 64-column swizzle atoms
  static constexpr uint32_t TILE = 128u * D * 2;          // Q, K or V tile bytes
  static constexpr uint32_t Q_OFF = 0;
  static constexpr int QS = 2, KS = 2, VS = 2;            // Q, K and V ring stages
  static constexpr uint32_t K_OFF = Q_OFF + QS * TILE;
  static constexpr uint32_t V_OFF = K_OFF + KS * TILE;
  // Warp roles: 0 loaders, 1 MMA, 2 item fetcher, 3 idle (warpgroup 0);
  // 4..19 P warps, four per TMEM lane quarter (warpgroups 1-4); 20..23 O
  // epilogue, one per lane quarter (warpgroup 5).
  static constexpr int PW = 16, EW = 4;
  static constexpr int FETCH_WARP = 2, P_WARP0 = 4, EPI_WARP0 = P_WARP0 + PW;
  static constexpr int THREADS = 32 * (EPI_WARP0 + EW);
  static constexpr uint32_t WIN_OFF = V_OFF + VS * TILE;          // PW warps x 2 x 64 floats
  static constexpr uint32_t RT_OFF = WIN_OFF + PW * 2 * 64 * 4;   // 2 ring slots x 256 floats
  static constexpr uint32_t STG_OFF = RT_OFF + 2 * 256 * 4;       // EW warps x 2 x 32 x 16 floats
  static constexpr uint32_t BAR_OFF = STG_OFF + EW * 4096;
  static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
  static_assert(QS == 2 && KS <= 4 && VS <= 4, "barrier slots");
  static_assert(SMEM <= 232448, "shared memory per CTA");
  // TMEM columns: S0 | S1 (128 each; P_j, 128 fp16 per row packed in pairs,
  // is written over S_j: the P of S columns 32g .. 32g + 31 over columns
  // 32g .. 32g + 15, which only the P warp that read them touches), then O0 | O1.
  static constexpr uint32_t O_COL = 256;
};

enum { MODE_SELF = 0, MODE_CAND = 1 };

// Item ring entry (the item carries its row offsets).
typedef AttnItem RingItem;

// y = x / 2 (score plus bias, halved); returns SiLU(x) = y + y tanh(y).
DEVI float silu_half(float y) { return fmaf(y, tanh_approx(y), y); }

// A shared-memory float at base + OFF bytes (the offset in the instruction).
template <int OFF>
DEVI float lds_f32_at(uint32_t base) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(base), "n"(OFF) : "memory");
  return v;
}

// Causal P for columns C and C+1 of this warp's 32 x 32 block, then the next
// pair: P = SiLU(S + position bias + time bias).  wa: shared address of the
// lane's window entry (column c takes entry 31 - c after it); ra: shared
// address of the head's halved time table; bw: the block's bucket bytes, 4
// columns per word.  The causal mask is in the window: a future column's
// entry is kMaskedHalfBias, for which SiLU gives exactly zero.
template <int C>
struct PPair {
  static DEVI void run(uint32_t (&pk)[16], const uint32_t (&sr)[32], const uint32_t (&bw)[8],
                       uint32_t wa, uint32_t ra) {
    const uint32_t b0 = __byte_perm(bw[C >> 2], 0u, 0x4440u | (C & 3));
    const uint32_t b1 = __byte_perm(bw[C >> 2], 0u, 0x4440u | ((C + 1) & 3));
    float p0 = silu_half(fmaf(__uint_as_float(sr[C]), 0.5f, lds_f32_at<4 * (31 - C)>(wa)) +
                         lds_f32(ra + 4u * b0));
    float p1 = silu_half(fmaf(__uint_as_float(sr[C + 1]), 0.5f, lds_f32_at<4 * (30 - C)>(wa)) +
                         lds_f32(ra + 4u * b1));
    pk[C >> 1] = pack_f16x2_sat(p0, p1);
    PPair<C + 2>::run(pk, sr, bw, wa, ra);
  }
};
template <>
struct PPair<32> {
  static DEVI void run(uint32_t (&)[16], const uint32_t (&)[32], const uint32_t (&)[8], uint32_t,
                       uint32_t) {}
};

// The window entry of a distance j - i > 0 (a future column): with it, y =
// s/2 + entry + time bias is below -1e29 for any finite score, tanh.approx(y)
// is exactly -1, and SiLU's y + y tanh(y) is exactly +0 -- the masked P,
// with no per-element select.
constexpr float kMaskedHalfBias = -1e30f;

template <int D, int MODE>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
              const __grid_constant__ CUtensorMap tmO, const AttnDev a) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars + 0;      // [QS]
  uint64_t* q_empty = bars + 2;     // [QS]
  uint64_t* k_full = bars + 25;     // [KS]
  uint64_t* k_empty = bars + 29;    // [KS]
  uint64_t* s_full = bars + 6;      // [2]
  uint64_t* p_full = bars + 10;     // [2]
  uint64_t* o_full = bars + 12;     // [2]
  uint64_t* o_free = bars + 14;     // [2]
  uint64_t* drain = bars + 16;
  uint64_t* it_full = bars + 17;    // [2] item ring
  uint64_t* it_empty = bars + 19;   // [2]
  uint64_t* v_full = bars + 33;     // [VS]
  uint64_t* v_empty = bars + 37;    // [VS]
  RingItem* ring = reinterpret_cast<RingItem*>(bars + 41);   // [2], 32 B each
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + 2);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
  int* s_go = reinterpret_cast<int*>(ab + 1);
  int* s_nitems = s_go + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    const int st = a.status ? *reinterpret_cast<volatile int*>(a.status) : 0;
    *s_go = (st == 0);
    *s_nitems = *a.n_items;
    ab->flag = 0;
    ab->limit_us = a.wait_limit_us;
    for (int i = 0; i < C::QS; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
    }
    for (int i = 0; i < C::KS; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::VS; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, C::PW);
      mbar_init(o_full + i, 1);
      mbar_init(o_free + i, C::EW);
      mbar_init(it_full + i, 1);
      mbar_init(it_empty + i, 3 + C::PW + C::EW);  // loader lanes, MMA thread, P and O warps
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
    tma_prefetch_desc(&tmO);
  }
  __syncthreads();
  if (!*s_go) return;
  const int n_items = *s_nitems;

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
    // Lane 0 loads Q (once per item) and the K tiles, lane 1 the V tiles, each
    // through its own 2-stage ring: a K stage is free again as soon as its
    // S = Q K^T has run, so K runs ahead of V by the length of the P stage.
    if (lane < 2) {
      const bool kq = (lane == 0);
      uint64_t* full = kq ? k_full : v_full;
      uint64_t* empty = kq ? k_empty : v_empty;
      uint8_t* buf = kq ? sK : sV;
      const int col = kq ? a.k_col : a.v_col;
      const uint32_t nst = kq ? C::KS : C::VS;
      uint32_t ncon = 0, st = 0, ph = 0, issued = 0, last_par = 0, q_issued = 0, q_last = 0;
      int litem = 0;
      bool ok = true;
      for (;;) {
        const int slot = ncon & 1;
        if (!mbar_wait(it_full + slot, (ncon >> 1) & 1, ab, a.status)) {
          ok = false;
          break;
        }
        const AttnItem w = ring[slot];
        mbar_arrive(it_empty + slot);
        ++ncon;
        if (w.b < 0) break;
        if (kq) {
          const int qs = litem & 1;  // Q stage of this item
          if (!mbar_wait(q_empty + qs, ((litem >> 1) & 1) ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(q_full + qs, C::TILE);
#pragma unroll
          for (int at = 0; at < C::NA; ++at)
            tma_load_2d(sQ + qs * C::TILE + at * 16384, &tmQ, a.q_col + w.head * D + at * 64,
                        w.q_row0, q_full + qs);
          q_issued |= 1u << qs;
          q_last = (q_last & ~(1u << qs)) | ((uint32_t)((litem >> 1) & 1) << qs);
        }
        for (int j = 0; j < w.nkv; ++j) {
          if (!mbar_wait(empty + st, ph ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + st, C::TILE);
#pragma unroll
          for (int at = 0; at < C::NA; ++at)
            tma_load_2d(buf + st * C::TILE + at * 16384, &tmKV, col + w.head * D + at * 64,
                        w.kv_row0 + j * 128, full + st);
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (ph << st);
          if (++st == nst) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ++litem;
      }
      if (!ok) {  // let every load already in flight land before the CTA exits
        AbortState tmp{0, kWaitLimitUs};
        for (uint32_t s2 = 0; s2 < nst; ++s2)
          if ((issued >> s2) & 1u) mbar_wait(full + s2, (last_par >> s2) & 1u, &tmp, nullptr);
        for (int s2 = 0; s2 < C::QS; ++s2)
          if ((q_issued >> s2) & 1u) mbar_wait(q_full + s2, (q_last >> s2) & 1u, &tmp, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f16_f32(128, 128, 0, 0, 1);
      constexpr uint32_t IDESC_O = idesc_f16_f32(128, D, 0, 1, 1);  // V is MN-major
      int litem = 0;
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0, scount = 0, pcount = 0, ncon = 0;
      bool ok = true, any = false;
      const uint32_t q_base0 = smem_u32(sQ);
      // P.V of tile jj of an item with nkv tiles; `li` is that item's index
      // on this CTA (the O accumulator's phase).
      auto issue_pv = [&](int jj, int nkv, int li) -> bool {
        const int pb = (int)(pcount & 1);  // P_j sits in S_j's buffer
        const uint32_t pph = (pcount >> 1) & 1;
        const int ob = li & 1;             // O buffer of this item
        if (!mbar_wait(p_full + pb, pph, ab, a.status)) return false;
        if (jj == 0 && !mbar_wait(o_free + ob, ((li >> 1) & 1) ^ 1, ab, a.status)) return false;
        if (!mbar_wait(v_full + vst, vph, ab, a.status)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + pb * 128;
        const uint32_t v_base = smem_u32(sV + vst * C::TILE);
        // 16 KV rows per MMA = 8 packed P columns; the P of KV columns
        // 32g .. 32g + 31 sits at TMEM columns 32g .. 32g + 15 of the buffer
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_f16_ts(tmem + C::O_COL + ob * D, p_tmem + (kk >> 1) * 32 + (kk & 1) * 8,
                        sdesc_sw128(v_base + kk * 2048, 16384, 1024), IDESC_O,
                        (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(v_empty + vst);
        if (jj == nkv - 1) tc_commit(o_full + ob);
        if (++vst == C::VS) {
          vst = 0;
          vph ^= 1;
        }
        ++pcount;
        any = true;
        return true;
      };
      // The P.V of each tile is issued after the next S, across item
      // boundaries too, so the first S of an item overlaps the last P of the
      // one before it.
      int pend_j = -1, pend_n = 0, pend_li = 0;
      auto flush = [&]() -> bool {
        if (pend_j < 0) return true;
        const bool r = issue_pv(pend_j, pend_n, pend_li);
        pend_j = -1;
        return r;
      };
      for (;;) {
        const int slot = ncon & 1;
        if (!mbar_wait(it_full + slot, (ncon >> 1) & 1, ab, a.status)) {
          ok = false;
          break;
        }
        const AttnItem w = ring[slot];
        mbar_arrive(it_empty + slot);
        ++ncon;
        if (w.b < 0) break;
        const int nkv = w.nkv;
        const int qs = litem & 1;
        const uint32_t q_base = q_base0 + qs * C::TILE;
        if (!mbar_wait(q_full + qs, (litem >> 1) & 1, ab, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < nkv; ++j) {
          if (!mbar_wait(k_full + kst, kph, ab, a.status)) {
            ok = false;
            break;
          }
          // S_j reuses the buffer of S_{j-2}; P_{j-2}, written there, was read
          // by a P.V issued before this MMA, and MMAs run in issue order.
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
          if (j == nkv - 1) tc_commit(q_empty + qs);  // P.V does not read Q: free it early
          if (++kst == C::KS) {
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
          pend_n = nkv;
          pend_li = litem;
        }
        if (!ok) break;
        if (nkv == 0) {
          // nothing to accumulate: O is taken as zero; the previous item's
          // last P.V goes first so that O's phases stay in item order
          if (!flush()) {
            ok = false;
            break;
          }
          const int ob = litem & 1;  // O's phases stay in item order per buffer
          if (!mbar_wait(o_free + ob, ((litem >> 1) & 1) ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          tc_commit(o_full + ob);
          tc_commit(q_empty + qs);
        }
        ++litem;
      }
      if (ok) flush();
      if (any) {
        tc_commit(drain);
        AbortState tmp{0, kWaitLimitUs};
        mbar_wait(drain, 0, &tmp, nullptr);
      }
    }
  } else if (warp >= C::P_WARP0 && warp < C::EPI_WARP0) {
    // ------------------------------------------------ P warps
    const int pw = warp - C::P_WARP0;  // 0..15
    const int q = warp & 3;          // TMEM lane quarter
    const int g = pw >> 2;           // which 32 of the 128 S columns
    const int r = q * 32 + lane;     // row inside the 128-row tile
    float* win2 = reinterpret_cast<float*>(smem + C::WIN_OFF) + pw * 2 * 64;  // 2 buffers
    const float* rt_ring = reinterpret_cast<const float*>(smem + C::RT_OFF);
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t scount = 0, ncon = 0;
    for (;;) {
      const int slot = ncon & 1;
      if (!mbar_wait_warp(it_full + slot, (ncon >> 1) & 1, ab, a.status)) break;
      const AttnItem w = ring[slot];
      const float* rt = rt_ring + slot * 256;   // valid while this item holds the slot
      ++ncon;
      if (w.b < 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(it_empty + slot);
        break;
      }
      const int64_t kv0 = w.kv_row0;
      const int n_kv = w.n_kv;                   // history / sequence length
      const float* Rp = a.rab_pos + (size_t)w.head * a.Np;
      const float* Rt = a.rab_time + (size_t)w.head * a.Nt;
      const int t_i = (MODE == MODE_SELF) ? 0 : a.t_req_rel[w.b];
      // Candidate mode: history time of this lane's column of KV tile jt, and
      // the halved bias of that column from it.
      auto cand_trel = [&](int jt) -> int {
        const int jc = jt * 128 + g * 32 + lane;
        return jc < n_kv ? a.t_rel[kv0 + jc] : 0;
      };
      // A column past the history (the last tile's ragged end) gets
      // kMaskedHalfBias: its P is exactly zero.
      auto cand_bias = [&](int jt, int trel) -> float {
        const int jc = jt * 128 + g * 32 + lane;
        if (jc >= n_kv) return kMaskedHalfBias;
        const int gap = max(t_i - trel, 0);
        return 0.5f * (__ldg(Rp + log_bucket(n_kv - jc, a.Sp, a.Np)) +
                       __ldg(Rt + log_bucket(gap, a.St, a.Nt)));
      };
      // Bias inputs of KV tile jt into window buffer `buf` (and, causal mode,
      // the tile's time-bucket words into bwn).  Causal mode: the warp's
      // 32 x 32 block spans the 63 distances base .. base + 62.
      auto prep = [&](int jt, int buf, uint32_t (&bwn)[8]) {
        float* win = win2 + buf * 64;
        if (MODE == MODE_SELF) {
          const uint32_t* tbw = a.tbuckets + (size_t)(w.tile0 + jt) * kBucketTileWords +
                                (g * 8) * 128 + r;
#pragma unroll
          for (int m = 0; m < 8; ++m) bwn[m] = __ldg(tbw + m * 128);
          const int base = (w.qt - jt) * 128 + q * 32 - g * 32 - 31;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int k = lane + 32 * u;
            if (k < 63) {
              const int dist = base + k;
              win[k] = dist >= 0 ? 0.5f * __ldg(Rp + log_bucket(dist, a.Sp, a.Np))
                                 : kMaskedHalfBias;
            }
          }
        } else {
          win[lane] = cand_bias(jt, cand_trel(jt));
        }
      };
      uint32_t bw[8], bwn[8];
      if (w.nkv > 0) prep(0, 0, bw);
      // candidate mode: the next tile's bias is looked up while this tile
      // computes and stored after it, from history times read a tile earlier
      int tr_n = (MODE == MODE_CAND && w.nkv > 1) ? cand_trel(1) : 0;
      bool alive = true;
      for (int j = 0; j < w.nkv; ++j) {
        __syncwarp();  // this tile's window is written; the one before it is free
        const float* win = win2 + (j & 1) * 64;
        // ---- S tile from TMEM: this warp's 32 rows x 32 columns
        const int sb = scount & 1;
        if (!mbar_wait_warp(s_full + sb, (scount >> 1) & 1, ab, a.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(tmem + sb * 128 + g * 32 + lane_base, sr);
        // fetch the next tile's bias inputs while this tile computes
        float nb = 0.f;
        if (j + 1 < w.nkv) {
          if (MODE == MODE_SELF) {
            prep(j + 1, (j + 1) & 1, bwn);
          } else {
            nb = cand_bias(j + 1, tr_n);
            if (j + 2 < w.nkv) tr_n = cand_trel(j + 2);
          }
        }
        tmem_ld_wait();
        ++scount;
        // ---- P = SiLU(S + bias), masked, fp16
        uint32_t pk[16];
        // window and time table by shared-space loads: element c of this
        // lane's row takes window entry lane + 31 - c and table entry b_c
        const uint32_t wa = smem_u32(win) + 4u * (uint32_t)lane;
        const uint32_t ra = smem_u32(rt);
        if (MODE == MODE_SELF) {
          PPair<0>::run(pk, sr, bw, wa, ra);  // (the diagonal tile's mask is in the window)
        } else {
          // (columns past the history carry kMaskedHalfBias in the window)
          const uint32_t wc = smem_u32(win);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = silu_half(fmaf(__uint_as_float(sr[c]), 0.5f, lds_f32(wc + 4u * c)));
            const float p1 =
                silu_half(fmaf(__uint_as_float(sr[c + 1]), 0.5f, lds_f32(wc + 4u * (c + 1))));
            pk[c >> 1] = pack_f16x2_sat(p0, p1);
          }
          if (j + 1 < w.nkv) win2[((j + 1) & 1) * 64 + lane] = nb;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) bw[m] = bwn[m];
        // ---- write P over the first half of this warp's own 32 columns of
        // S_j (already in registers; no other warp reads them): 32 rows, 32
        // fp16 as 16 packed columns
        tmem_st16(tmem + sb * 128 + g * 32 + lane_base, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + sb);
      }
      // the ring slot (and its time table) may be refilled from here on
      __syncwarp();
      if (lane == 0) mbar_arrive(it_empty + slot);
      if (!alive) break;
    }
  } else if (warp == C::FETCH_WARP) {
    // ------------------------------------------------ item fetcher
    // Claims work items (dynamic, one atomic per item), publishes each into
    // the 2-slot ring with its head's halved time-bias table (causal mode),
    // and warms L2 with the item's Q tile, two items ahead of the P warps.
    float* rt_ring = reinterpret_cast<float*>(smem + C::RT_OFF);
    auto claim = [&]() {
      int v = 0;
      if (lane == 0) v = atomicAdd(a.work_next, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    // An item is claimed only once a ring slot is free, so a CTA never holds
    // more than two unstarted items (a short tail at the end of the launch).
    uint32_t npub = 0;
    for (;;) {
      // Test hook: CTA 0's fetcher stops after publishing two items, without
      // the terminator, so every other role of this CTA waits for a third
      // item that never comes; those bounded waits give up (HSTU_ERR_TIMEOUT)
      // and the CTA winds down.  No load is skipped or left unwaited.
      if (a.inject_stall && blockIdx.x == 0 && npub == 2) break;
      const int slot = npub & 1;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(it_empty + slot, ((npub >> 1) & 1) ^ 1, ab, a.status);
      if (!__shfl_sync(0xffffffffu, okw ? 1 : 0, 0)) break;
      const int idx = claim();
      RingItem x;
      if (idx < n_items) x = a.items[idx];
      else x = AttnItem{-1, 0, 0, 0, 0, 0, 0, 0, 0};
      if (MODE == MODE_SELF && x.b >= 0) {
        const float* Rt = a.rab_time + (size_t)x.head * a.Nt;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = lane + 32 * u;
          if (k < a.Nt) rt_ring[slot * 256 + k] = 0.5f * __ldg(Rt + k);
        }
      }
      if (lane == 0) ring[slot] = x;
      __syncwarp();
      if (lane == 0) mbar_arrive(it_full + slot);  // release: slot contents visible to waiters
      ++npub;
      if (x.b < 0) break;
      // only the item's Q tile: warming L2 with its whole K/V as well (two
      // items ahead on every CTA) overflowed L2 on long histories and made
      // the history be read twice (measured: candidate attention 14 % slower,
      // the 8-layer stack's attention 4 %)
      if (lane == 0) {
#pragma unroll
        for (int at = 0; at < C::NA; ++at)
          tma_prefetch_l2_2d(&tmQ, a.q_col + x.head * D + at * 64, x.q_row0);
      }
    }
  } else if (warp >= C::EPI_WARP0) {
    // ------------------------------------------------ epilogue warps
    // One per TMEM lane quarter: 32 rows x D columns of O each, streamed out of
    // TMEM 16 columns at a time, scaled by 1/n (candidates: plus the self
    // term) and stored fp32 -- a full 32-row block through swizzled staging and
    // a TMA bulk store, a block at the user's ragged end row by row (the rows
    // after it belong to the next user).  The P warps meanwhile go on with the
    // next item.
    const int ew = warp - C::EPI_WARP0;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint8_t* stg = smem + C::STG_OFF + ew * 4096;  // two 2 KB buffers
    uint32_t ncon = 0, nbuf = 0;
    int litem = 0;
    for (;;) {
      const int slot = ncon & 1;
      if (!mbar_wait_warp(it_full + slot, (ncon >> 1) & 1, ab, a.status)) break;
      const AttnItem w = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(it_empty + slot);
      ++ncon;
      if (w.b < 0) break;
      const int64_t q0 = w.q_row0;
      const int rows_valid = min(128, w.n_q - (int)w.qt * 128);
      const bool row_ok = r < rows_valid;
      const bool full_rows = q * 32 + 32 <= rows_valid;
      const float inv_n = 1.0f / (float)max(w.n_kv, 1);
      float p_self = 0.f;
      const __half* rowp = a.q_buf + (q0 + (row_ok ? r : 0)) * a.ld_f1;
      if (MODE == MODE_CAND && row_ok) {
        // self term: the candidate attends to itself at distance 0, gap 0
        const uint4* qp = reinterpret_cast<const uint4*>(rowp + a.q_col + w.head * D);
        const uint4* kp = reinterpret_cast<const uint4*>(rowp + a.k_col + w.head * D);
        float dot = 0.f;
#pragma unroll 2
        for (int i = 0; i < D / 8; ++i) {
          const uint4 qa = qp[i], ka = kp[i];
          const uint32_t qw[4] = {qa.x, qa.y, qa.z, qa.w}, kw[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dot += f16lo(qw[k]) * f16lo(kw[k]) + f16hi(qw[k]) * f16hi(kw[k]);
        }
        const float s_self = dot + __ldg(a.rab_pos + (size_t)w.head * a.Np) +
                             __ldg(a.rab_time + (size_t)w.head * a.Nt);
        p_self = __half2float(__float2half_rn(silu_fast(s_self)));
      }
      const int ob = litem & 1;
      if (!mbar_wait_warp(o_full + ob, (litem >> 1) & 1, ab, a.status)) break;
      tc_fence_after();
      // n O of this row and head, 16 columns from c16 * 16: the accumulator
      // (or zero), plus the candidate's self term.  The 1/n of O cancels in
      // the normalised values (O - mean) / sd and is applied to the stored
      // mean and deviation only.
      auto load_o = [&](int c16, float (&o)[16]) {
        if (w.nkv > 0) {
          uint32_t orr[16];
          tmem_ld16(tmem + C::O_COL + ob * D + c16 * 16 + lane_base, orr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __uint_as_float(orr[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = 0.f;
        }
        if (MODE == MODE_CAND && row_ok) {
          const uint4* vp = reinterpret_cast<const uint4*>(rowp + a.v_col + w.head * D + c16 * 16);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 va = vp[i];
            const uint32_t vw[4] = {va.x, va.y, va.z, va.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              o[i * 8 + 2 * k] += p_self * f16lo(vw[k]);
              o[i * 8 + 2 * k + 1] += p_self * f16hi(vw[k]);
            }
          }
        }
      };
      // pass 1: mean and deviation of the row's D values, from sums shifted
      // by the first value (no cancellation when the mean dominates)
      float shift = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll 1
      for (int c16 = 0; c16 < D / 16; ++c16) {
        float o[16];
        load_o(c16, o);
        if (c16 == 0) shift = o[0];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float dv = o[i] - shift;
          s1 += dv;
          s2 = fmaf(dv, dv, s2);
        }
      }
      const float mean = shift + s1 * (1.0f / D);
      const float sd = sqrtf(fmaxf(s2 - s1 * s1 * (1.0f / D), 0.f) * (1.0f / D));
      const float inv_sd = sd > 0.f ? 1.0f / sd : 0.f;
      const float nmean = -mean * inv_sd;  // (o - mean) / sd = o inv_sd + nmean
      if (row_ok) a.ostats[(q0 + r) * a.h + w.head] = make_float2(mean * inv_n, sd * inv_n);
      // pass 2: (O - mean) / sd in fp16, 32 columns per store -- a full
      // 32-row block through swizzled staging and a TMA bulk store, a block
      // at the user's ragged end row by row (the rows after it belong to the
      // next user)
#pragma unroll 1
      for (int c32 = 0; c32 < D / 32; ++c32) {
        uint32_t pk[16];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float o[16];
          load_o(c32 * 2 + hf, o);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[hf * 8 + i] = pack_f16x2_sat(fmaf(o[2 * i], inv_sd, nmean),
                                            fmaf(o[2 * i + 1], inv_sd, nmean));
        }
        if (c32 == D / 32 - 1) {  // O is fully read: the next item may accumulate
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free + ob);
        }
        if (full_rows) {
          uint8_t* buf = stg + (nbuf & 1) * 2048;
          if (lane == 0) bulk_wait_read<1>();  // the store two blocks back has read `buf`
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmO, w.head * D + c32 * 32, (int)(q0 + q * 32), buf);
            bulk_commit();
          }
          ++nbuf;
        } else if (row_ok) {
          uint4* op = reinterpret_cast<uint4*>(a.O + (q0 + r) * a.ldo + w.head * D + c32 * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) op[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      ++litem;
    }
    if (lane == 0) bulk_wait_all();  // O stores complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) {
    // The last CTA to finish re-arms the work counter for the next launch
    // (launches on one stream never overlap).
    __threadfence();
    if (atomicAdd(a.work_done, 1) == (int)gridDim.x - 1) {
      atomicExch(a.work_next, 0);
      atomicExch(a.work_done, 0);
      __threadfence();
    }
  }
}

template <int D, int MODE>
static cudaError_t launch_attn_inst(const CUtensorMap& tq, const CUtensorMap& tkv,
                                    const CUtensorMap& to, const AttnDev& ad, int grid,
                                    cudaStream_t s) {
  using C = AttnCfg<D>;
  auto kfn = k_attn_tc<D, MODE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<grid, C::THREADS, C::SMEM, s>>>(tq, tkv, to, ad);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnCall& c, cudaStream_t s) {
  if (c.dqk != c.dv || (c.dqk != 64 && c.dqk != 128)) return cudaErrorInvalidValue;
  if (c.mode == MODE_SELF && c.Nt > 256) return cudaErrorInvalidValue;
  if (c.item_cap <= 0 || c.q_rows_cap <= 0) return cudaSuccess;
  CUtensorMap tq, tkv;
  const uint64_t F = (uint64_t)c.ld_f1;
  if (!encode_tmap_2d(&tq, c.q_buf, (uint64_t)c.q_rows_cap, F, F * 2, 64, 128, true))
    return cudaErrorInvalidValue;
  // With no history rows there is nothing to load from the KV buffer; any
  // valid map will do (no KV tile is ever requested).
  if (c.kv_rows_cap > 0) {
    if (!encode_tmap_2d(&tkv, c.kv_buf, (uint64_t)c.kv_rows_cap, F, F * 2, 64, 128, true))
      return cudaErrorInvalidValue;
  } else {
    tkv = tq;
  }
  // normalised O: fp16 [q_rows_cap, h * d_v] with row stride ldo; 32-column
  // x 32-row boxes (64-byte rows) for the epilogue's bulk stores.
  if (!c.ostats || c.ldo % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap to;
  if (!encode_tmap_2d_ex(&to, c.O, (uint64_t)c.q_rows_cap, (uint64_t)c.h * c.dv,
                         (uint64_t)c.ldo * 2, 32, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                         CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  AttnDev ad;
  ad.items = c.items;
  ad.n_items = c.n_items;
  ad.q_off = c.q_off;
  ad.kv_off = c.kv_off;
  ad.t_rel = c.t_rel;
  ad.t_req_rel = c.t_req_rel;
  ad.tbuckets = c.tbuckets;
  ad.rab_pos = c.rab_pos;
  ad.rab_time = c.rab_time;
  ad.Np = c.Np;
  ad.Nt = c.Nt;
  ad.Sp = c.Sp;
  ad.St = c.St;
  ad.q_col = c.q_col;
  ad.k_col = c.k_col;
  ad.v_col = c.v_col;
  ad.q_buf = static_cast<const __half*>(c.q_buf);
  ad.ld_f1 = c.ld_f1;
  ad.O = static_cast<__half*>(c.O);
  ad.ldo = c.ldo;
  ad.ostats = reinterpret_cast<float2*>(c.ostats);
  ad.h = c.h;
  ad.work_next = c.work_next;
  ad.work_done = c.work_done;
  ad.status = c.status;
  take_wait_test(&ad.wait_limit_us, &ad.inject_stall);
  const int grid = (int)std::min<int64_t>(c.item_cap, num_sms());
  LaunchScope ls(c.mode == MODE_SELF ? K_ATTN : K_ATTN_CAND, s);
  if (c.mode == MODE_SELF)
    return c.dqk == 64 ? launch_attn_inst<64, MODE_SELF>(tq, tkv, to, ad, grid, s)
                       : launch_attn_inst<128, MODE_SELF>(tq, tkv, to, ad, grid, s);
  return c.dqk == 64 ? launch_attn_inst<64, MODE_CAND>(tq, tkv, to, ad, grid, s)
                     : launch_attn_inst<128, MODE_CAND>(tq, tkv, to, ad, grid, s);
}

}  // namespace hstu

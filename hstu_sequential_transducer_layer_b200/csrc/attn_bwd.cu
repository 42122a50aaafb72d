// attn_bwd.cu — backward pass of the pointwise (softmax-free) attention on
// the tcgen05 tensor cores, over jagged batches.
//
// 'HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか',
// subsection '2. QKᵀで「どの履歴を見るか」を決める' gives the forward per head:
//   s_ij = Q_i.K_j + pos_bias(i - j) + time_bias(t_i - t_j),  j <= i,
//   O_i  = (1/n) sum_j SiLU(s_ij) V_j.
// Its derivatives, with dO the gradient of O (chain rule, nothing else):
//   dA_ij = (1/n) dO_i . V_j          dV_j = (1/n) sum_i SiLU(s_ij) dO_i
//   dS_ij = dA_ij SiLU'(s_ij)         dK_j = sum_i dS_ij Q_i
//   dQ_i  = sum_j dS_ij K_j           d pos_bias[b]  = sum of dS_ij over pairs in bucket b
//                                     d time_bias[b] = likewise over the time buckets
// where SiLU'(s) = sig(s) (1 + s (1 - sig(s))).  Because there is no softmax,
// nothing of the forward has to be kept but its inputs: S is recomputed.
//
// Two kernels, one template:
//   MODE_DKV: one work item = (user, 128-row KV tile j, head); it walks the
//     query rows i >= j in units of 64 rows, recomputing S^T = K_j Q_u^T and
//     dA^T = V_j dO_u^T in tensor memory (one TMEM lane per key row), forms
//     P^T = SiLU(S^T)/n and dS^T in fp16 and writes them back into tensor
//     memory over the S^T columns they came from, from where the MMAs
//     dV_j += P^T dO_u and dK_j += dS^T Q_u read their A operand; it also sums
//     dS into the bias gradients.  The epilogue multiplies dK, dV by SiLU' of
//     the f1 pre-activation (the gradient of f1's own SiLU) and stores them
//     into the f1-shaped gradient buffer.
//   MODE_DQ: one work item = (user, query tile i, head); it walks the KV rows
//     j <= i in units of 64, recomputing S = Q_i K_u^T and dA = dO_i V_u^T,
//     forms dS, and accumulates dQ_i += dS K_u.
// Computing dQ in its own pass costs two more MMAs per tile pair but needs no
// atomic accumulation of dQ across KV tiles.
//
// Pipeline: S and dA of a unit occupy one of two 64-column halves of their
// TMEM regions, so the MMAs of unit u+1 run while the elementwise warps work
// on unit u; the MMA thread issues S of unit u+1 before the accumulation of
// unit u, and tcgen05 MMAs execute in issue order, so the accumulation has
// read P^T and dS^T of unit u before S of unit u+2 overwrites them.  The
// streamed 64-row units (two [64 x D] tiles each) arrive by TMA through a
// ring of 4 (D = 128) or 6 (D = 64) stages.
//
// Roles (640 threads): warp 0 lane 0 issues the TMA loads (the item's fixed
// tiles once, the streamed units through the ring), warp 1 lane 0 issues the
// MMAs, warp 2 claims items (dynamic scheduling) into a 2-slot ring, warps
// 4-19 (four per TMEM lane quarter, 16 of a unit's 64 columns each) do the
// elementwise work and the epilogue.  Each elementwise warp writes its P^T
// and dS^T (8 packed columns each) into the 16 TMEM columns it read S from,
// so no warp overwrites columns another warp has yet to read.  The bias tables
// of every head sit in shared memory (when they fit) and the timestamps of a
// unit's 16 streamed rows reach the lanes by shuffle.
// Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace hstu {

enum { MODE_DKV = 0, MODE_DQ = 1 };

struct AttnBwdDev {
  const AttnItem* items;
  const int32_t* n_items;
  int q_col, k_col, v_col;
  const __half* pre;        // f1 pre-activation [T, F] fp16 (row stride ld_f1)
  __half* dP;               // f1-shaped gradient [T, F] fp16: d(pre-activation)
  int64_t ld_f1;
  const int32_t* t_rel;
  const float* rab_pos;
  const float* rab_time;
  unsigned long long* rab_acc;  // MODE_DKV: [h][Np + Nt] bias-table gradients, fixed point
  int Np, Nt, Sp, St, h;
  int32_t* work_next;
  int32_t* work_done;
  int* status;
};

template <int D>
struct BwdCfg {
  static constexpr uint32_t FIX_TILE = 128u * D * 2;  // one [128 x D] fp16 tile
  static constexpr uint32_t HALF = 64u * D * 2;       // one [64 x D] fp16 tile
  static constexpr uint32_t UNIT = 2 * HALF;          // a streamed unit: two [64 x D] tiles
  static constexpr int STAGES = D == 64 ? 6 : 4;
  static constexpr uint32_t FIX_OFF = 0;               // 2 fixed tiles
  static constexpr uint32_t STR_OFF = FIX_OFF + 2 * FIX_TILE;
  // the bias tables of every head ([h][Np + Nt] fp32) and, for MODE_DKV, this
  // CTA's fixed-point sums of their gradients (low words, then high words),
  // when they fit
  static constexpr int TAB_CAP = 2048;
  static constexpr uint32_t TAB_OFF = STR_OFF + STAGES * UNIT;
  static constexpr uint32_t BIN_OFF = TAB_OFF + TAB_CAP * 4;
  static constexpr uint32_t BAR_OFF = BIN_OFF + TAB_CAP * 8;
  static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
  static constexpr int EW0 = 4, NEW = 16;            // elementwise warps 4..19
  static constexpr int THREADS = 32 * (EW0 + NEW);
  static constexpr uint32_t DA_COL = 128;            // TMEM: S halves | dA halves | accumulators
  static constexpr uint32_t ACC = 256;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(STAGES <= 8, "barrier slots");
};

DEVI float sigmoid_acc(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// 8 registers per thread -> 32 lanes x 8 consecutive 32-bit TMEM columns.
DEVI void tmem_st8(uint32_t taddr, const uint32_t (&r)[16]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// Bias-table gradients are summed in 64-bit fixed point (units of 2^-32):
// integer sums do not depend on the order of the additions, so the result is
// the same on every run.  A CTA keeps its sums in shared memory as low and
// high 32-bit words (the carry out of the low word is added to the high one)
// and adds them into the global 64-bit accumulators at its end.
constexpr float kFixScale = 4294967296.0f;  // 2^32
DEVI long long to_fix(float v) {
  return __float2ll_rn(fminf(fmaxf(v, -1073741824.0f), 1073741824.0f) * kFixScale);
}

DEVI void fix_add_shared(uint32_t lo_addr, uint32_t hi_addr, long long q) {
  const uint32_t ql = (uint32_t)q, qh = (uint32_t)((unsigned long long)q >> 32);
  uint32_t old;
  asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(lo_addr), "r"(ql) : "memory");
  const uint32_t hc = qh + (old + ql < old ? 1u : 0u);
  if (hc) asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(hi_addr), "r"(hc) : "memory");
}

// Where one item's bias look-ups and gradient sums go: shared memory (SM) or
// global memory.
struct BiasCtx {
  uint32_t tp_s, tt_s;       // shared addresses of the head's position / time tables
  uint32_t bp_s, bt_s;       // shared addresses of the head's low-word bins (high: + kHiOff)
  const float* tp_g;
  const float* tt_g;
  unsigned long long* bp_g;  // global accumulators of the head
  unsigned long long* bt_g;
};

template <bool SM>
DEVI float bias_at(const BiasCtx& c, int bp, int bt) {
  if (SM) return lds_f32(c.tp_s + 4u * bp) + lds_f32(c.tt_s + 4u * bt);
  return __ldg(c.tp_g + bp) + __ldg(c.tt_g + bt);
}
template <bool SM, int HI_OFF>
DEVI void bias_flush(const BiasCtx& c, bool pos, int b, float v) {
  const long long q = to_fix(v);
  if (SM) {
    const uint32_t lo = (pos ? c.bp_s : c.bt_s) + 4u * b;
    fix_add_shared(lo, lo + HI_OFF, q);
  } else {
    atomicAdd((pos ? c.bp_g : c.bt_g) + b, (unsigned long long)q);
  }
}

// The 16 elements of one thread in one unit: the thread's fixed row (MODE_DKV:
// key row j; MODE_DQ: query row i) against streamed rows c0 .. c0+15 of the
// same user.  sr / dr: S and dA as read from TMEM.  out: packed fp16 P^T then
// dS^T (MODE_DKV) or dS (MODE_DQ, first 8 words).  tv: lane e < 16 holds the
// relative timestamp of streamed row c0 + e.  MASKED: some element may lie
// outside the user or the causal region (else none does).  SM: bias tables
// and gradient bins in shared memory.
template <int MODE, bool MASKED, bool SM, int HI_OFF>
DEVI void bwd_elems(const uint32_t (&sr)[16], const uint32_t (&dr)[16], uint32_t (&out)[16],
                    int c0, int fixed_row, bool row_ok, int n, int tv, int t_row, float inv_n,
                    const BiasCtx& bc, int Sp, int Np, int St, int Nt, int& cur_p, int& cur_t,
                    float& acc_p, float& acc_t) {
  float pv[16], dv[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int col = c0 + e;
    const int tc = __shfl_sync(0xffffffffu, tv, e);
    const int qi = MODE == MODE_DKV ? col : fixed_row;
    const int kj = MODE == MODE_DKV ? fixed_row : col;
    const int ti = MODE == MODE_DKV ? tc : t_row;
    const int tj = MODE == MODE_DKV ? t_row : tc;
    const int bp = (int)log_bucket_nb(MASKED ? max(qi - kj, 0) : qi - kj, Sp, Np);
    const int bt = (int)log_bucket_nb(max(ti - tj, 0), St, Nt);
    const float s = __uint_as_float(sr[e]) + bias_at<SM>(bc, bp, bt);
    const float sg = sigmoid_acc(s);
    float p = s * sg * inv_n;
    float ds = __uint_as_float(dr[e]) * inv_n * sg * fmaf(s, 1.0f - sg, 1.0f);
    bool ok = true;
    if (MASKED) {
      ok = row_ok && col < n && kj <= qi;
      p = ok ? p : 0.f;
      ds = ok ? ds : 0.f;
    }
    if (MODE == MODE_DKV && ok) {
      // the bias-table gradients: along a key row the query rows increase, so
      // buckets change rarely; one addition per run of equal buckets
      if (bp != cur_p) {
        if (cur_p >= 0) bias_flush<SM, HI_OFF>(bc, true, cur_p, acc_p);
        cur_p = bp;
        acc_p = 0.f;
      }
      acc_p += ds;
      if (bt != cur_t) {
        if (cur_t >= 0) bias_flush<SM, HI_OFF>(bc, false, cur_t, acc_t);
        cur_t = bt;
        acc_t = 0.f;
      }
      acc_t += ds;
    }
    pv[e] = p;
    dv[e] = ds;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (MODE == MODE_DKV) {
      out[k] = pack_f16x2_sat(pv[2 * k], pv[2 * k + 1]);
      out[8 + k] = pack_f16x2_sat(dv[2 * k], dv[2 * k + 1]);
    } else {
      out[k] = pack_f16x2_sat(dv[2 * k], dv[2 * k + 1]);
      out[8 + k] = 0u;
    }
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmdO,
               const __grid_constant__ CUtensorMap tmF64,
               const __grid_constant__ CUtensorMap tmdO64, const AttnBwdDev a) {
  using C = BwdCfg<D>;
  constexpr int NA = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* fix_full = bars + 0;
  uint64_t* fix_empty = bars + 1;
  uint64_t* str_full = bars + 2;    // [STAGES]
  uint64_t* str_empty = bars + 10;  // [STAGES]
  uint64_t* s_full = bars + 18;     // [2] S and dA of a unit in TMEM half r
  uint64_t* p_full = bars + 20;     // [2] P^T / dS^T of a unit written back
  uint64_t* acc_full = bars + 22;
  uint64_t* acc_free = bars + 23;
  uint64_t* it_full = bars + 24;    // [2]
  uint64_t* it_empty = bars + 26;   // [2]
  uint64_t* drain = bars + 28;
  AttnItem* ring = reinterpret_cast<AttnItem*>(bars + 32);   // [2] x 32 B
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + 2);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 2);
  int* s_go = reinterpret_cast<int*>(ab + 1);
  int* s_nitems = s_go + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbt = a.Np + a.Nt;
  const int nbin = a.h * nbt;
  const bool in_smem = nbin <= C::TAB_CAP;
  float* tab = reinterpret_cast<float*>(smem + C::TAB_OFF);
  uint32_t* bins = reinterpret_cast<uint32_t*>(smem + C::BIN_OFF);  // [lo: TAB_CAP][hi: TAB_CAP]
  if (in_smem) {
    for (int i = threadIdx.x; i < nbin; i += blockDim.x) {
      const int hh = i / nbt, k = i - hh * nbt;
      tab[i] = k < a.Np ? __ldg(a.rab_pos + (size_t)hh * a.Np + k)
                        : __ldg(a.rab_time + (size_t)hh * a.Nt + (k - a.Np));
      if (MODE == MODE_DKV) bins[i] = bins[C::TAB_CAP + i] = 0u;
    }
  }
  if (threadIdx.x == 0) {
    const int st = a.status ? *reinterpret_cast<volatile int*>(a.status) : 0;
    *s_go = (st == 0);
    *s_nitems = *a.n_items;
    ab->flag = 0;
    ab->limit_us = kWaitLimitUs;
    mbar_init(fix_full, 1);
    mbar_init(fix_empty, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(str_full + i, 1);
      mbar_init(str_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, C::NEW);
      mbar_init(it_full + i, 1);
      mbar_init(it_empty + i, 2 + C::NEW);  // loader, MMA thread, elementwise warps
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_free, C::NEW);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmF);
    tma_prefetch_desc(&tmdO);
    tma_prefetch_desc(&tmF64);
    tma_prefetch_desc(&tmdO64);
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
  uint8_t* sFix = smem + C::FIX_OFF;
  uint8_t* sStr = smem + C::STR_OFF;

  // Units of an item: DKV walks query rows qt*128 .. n-1, DQ KV rows
  // 0 .. min(n, qt*128 + 128) - 1, 64 rows per unit.
  auto n_units_of = [&](const AttnItem& w) -> int {
    const int rows = MODE == MODE_DKV ? w.n_q - w.qt * 128 : min(w.n_q, w.qt * 128 + 128);
    return (rows + 63) / 64;
  };
  auto first_row_of = [&](const AttnItem& w) -> int { return MODE == MODE_DKV ? w.qt * 128 : 0; };

  if (warp == 0) {
    // ------------------------------------------------ TMA loads
    if (lane == 0) {
      uint32_t ncon = 0, st = 0, ph = 0, issued = 0, last_par = 0;
      int litem = 0;
      bool fix_issued = false;
      uint32_t fix_par = 0;
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
        // the fixed tiles of this item (DKV: K_j, V_j; DQ: Q_i, dO_i), once the
        // previous item's last S MMA has read them
        if (!mbar_wait(fix_empty, (litem & 1) ^ 1, ab, a.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(fix_full, 2 * C::FIX_TILE);
        const int r0 = w.kv_row0 + w.qt * 128;  // rows of tile qt of this user
#pragma unroll
        for (int at = 0; at < NA; ++at) {
          if (MODE == MODE_DKV) {
            tma_load_2d(sFix + at * 16384, &tmF, a.k_col + w.head * D + at * 64, r0, fix_full);
            tma_load_2d(sFix + C::FIX_TILE + at * 16384, &tmF, a.v_col + w.head * D + at * 64, r0,
                        fix_full);
          } else {
            tma_load_2d(sFix + at * 16384, &tmF, a.q_col + w.head * D + at * 64, r0, fix_full);
            tma_load_2d(sFix + C::FIX_TILE + at * 16384, &tmdO, w.head * D + at * 64, r0,
                        fix_full);
          }
        }
        fix_issued = true;
        fix_par = litem & 1;
        const int nu = n_units_of(w);
        const int row0 = w.kv_row0 + first_row_of(w);
        for (int u = 0; u < nu; ++u) {
          const int rr = row0 + 64 * u;
          if (!mbar_wait(str_empty + st, ph ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(str_full + st, C::UNIT);
          uint8_t* dst = sStr + st * C::UNIT;
#pragma unroll
          for (int at = 0; at < NA; ++at) {
            if (MODE == MODE_DKV) {  // Q_u, dO_u
              tma_load_2d(dst + at * 8192, &tmF64, a.q_col + w.head * D + at * 64, rr,
                          str_full + st);
              tma_load_2d(dst + C::HALF + at * 8192, &tmdO64, w.head * D + at * 64, rr,
                          str_full + st);
            } else {                 // K_u, V_u
              tma_load_2d(dst + at * 8192, &tmF64, a.k_col + w.head * D + at * 64, rr,
                          str_full + st);
              tma_load_2d(dst + C::HALF + at * 8192, &tmF64, a.v_col + w.head * D + at * 64, rr,
                          str_full + st);
            }
          }
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (ph << st);
          if (++st == (uint32_t)C::STAGES) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ++litem;
      }
      if (!ok) {  // every load in flight lands before the CTA exits
        AbortState tmp{0, kWaitLimitUs};
        for (int s2 = 0; s2 < C::STAGES; ++s2)
          if ((issued >> s2) & 1u) mbar_wait(str_full + s2, (last_par >> s2) & 1u, &tmp, nullptr);
        if (fix_issued) mbar_wait(fix_full, fix_par, &tmp, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f16_f32(128, 64, 0, 0, 1);
      constexpr uint32_t IDESC_ACC = idesc_f16_f32(128, D, 0, 1, 1);  // B MN-major
      uint32_t ncon = 0, st = 0, ph = 0, g = 0;
      int litem = 0;
      bool ok = true, any = false;
      // the unit whose S was issued last and whose accumulation is pending
      bool pend = false, p_first = false, p_last = false;
      uint32_t p_g = 0, p_st = 0;
      int p_item = 0;
      const uint32_t fix0 = smem_u32(sFix);
      // Accumulation of the pending unit (A = P^T / dS^T / dS from TMEM over
      // the unit's S half, 16 streamed rows = 8 packed columns per MMA;
      // B = the unit's streamed tiles read MN-major).
      auto issue_acc = [&]() -> bool {
        if (!mbar_wait(p_full + (p_g & 1), (p_g >> 1) & 1, ab, a.status)) return false;
        if (p_first && p_item > 0 && !mbar_wait(acc_free, (p_item - 1) & 1, ab, a.status))
          return false;
        tc_fence_after();
        const uint32_t str0 = smem_u32(sStr + p_st * C::UNIT);
        const uint32_t sreg = tmem + (p_g & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (!p_first || kk > 0) ? 1u : 0u;
          if (MODE == MODE_DKV) {
            tc_mma_f16_ts(tmem + C::ACC, sreg + kk * 16,
                          sdesc_sw128(str0 + C::HALF + kk * 2048, 8192, 1024), IDESC_ACC, acc);
            tc_mma_f16_ts(tmem + C::ACC + D, sreg + kk * 16 + 8,
                          sdesc_sw128(str0 + kk * 2048, 8192, 1024), IDESC_ACC, acc);
          } else {
            tc_mma_f16_ts(tmem + C::ACC, sreg + kk * 16,
                          sdesc_sw128(str0 + kk * 2048, 8192, 1024), IDESC_ACC, acc);
          }
        }
        tc_commit(str_empty + p_st);
        if (p_last) tc_commit(acc_full);
        pend = false;
        return true;
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
        if (w.b < 0) {
          if (pend) ok = issue_acc();
          break;
        }
        if (!mbar_wait(fix_full, litem & 1, ab, a.status)) {
          ok = false;
          break;
        }
        const int nu = n_units_of(w);
        for (int u = 0; u < nu; ++u, ++g) {
          if (!mbar_wait(str_full + st, ph, ab, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t str0 = smem_u32(sStr + st * C::UNIT);
          const uint32_t r = g & 1;
          // S (or S^T) = A0 B0^T and dA (or dA^T) = A1 B1^T over D, N = 64:
          // DKV: A0 = K_j, B0 = Q_u, A1 = V_j, B1 = dO_u; DQ: A0 = Q_i, B0 = K_u,
          // A1 = dO_i, B1 = V_u (all K-major)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t oa = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t ob = (kk >> 2) * 8192 + (kk & 3) * 32;
            tc_mma_f16_ss(tmem + r * 64, sdesc_sw128(fix0 + oa, 16, 1024),
                          sdesc_sw128(str0 + ob, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            tc_mma_f16_ss(tmem + C::DA_COL + r * 64, sdesc_sw128(fix0 + C::FIX_TILE + oa, 16, 1024),
                          sdesc_sw128(str0 + C::HALF + ob, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + r);
          if (u == nu - 1) tc_commit(fix_empty);
          any = true;
          if (pend && !issue_acc()) {
            ok = false;
            break;
          }
          pend = true;
          p_g = g;
          p_st = st;
          p_first = (u == 0);
          p_last = (u == nu - 1);
          p_item = litem;
          if (++st == (uint32_t)C::STAGES) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ++litem;
      }
      if (any) {
        tc_commit(drain);
        AbortState tmp{0, kWaitLimitUs};
        mbar_wait(drain, 0, &tmp, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ item fetcher
    uint32_t npub = 0;
    for (;;) {
      const int slot = npub & 1;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(it_empty + slot, ((npub >> 1) & 1) ^ 1, ab, a.status);
      if (!__shfl_sync(0xffffffffu, okw ? 1 : 0, 0)) break;
      int idx = 0;
      if (lane == 0) idx = atomicAdd(a.work_next, 1);
      idx = __shfl_sync(0xffffffffu, idx, 0);
      AttnItem x;
      if (idx < n_items) x = a.items[idx];
      else x = AttnItem{-1, 0, 0, 0, 0, 0, 0, 0, 0};
      if (lane == 0) {
        ring[slot] = x;
        mbar_arrive(it_full + slot);
      }
      __syncwarp();
      ++npub;
      if (x.b < 0) break;
    }
  } else if (warp >= C::EW0) {
    // ------------------------------------------------ elementwise warps + epilogue
    const int ew = warp - C::EW0;
    const int q = warp & 3;           // TMEM lane quarter (rows q*32 .. q*32+31)
    const int cb = ew >> 2;           // columns cb*16 .. cb*16+15 of a unit
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t ncon = 0, g = 0;
    int litem = 0;
    for (;;) {
      const int slot = ncon & 1;
      if (!mbar_wait_warp(it_full + slot, (ncon >> 1) & 1, ab, a.status)) break;
      const AttnItem w = ring[slot];
      ++ncon;
      if (w.b < 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(it_empty + slot);
        break;
      }
      const int n = w.n_q;                       // the user's length
      const float inv_n = 1.0f / (float)max(n, 1);
      const int64_t u0 = w.kv_row0;              // the user's first row
      const int fixed_row = w.qt * 128 + q * 32 + lane;  // this thread's row within the user
      const bool row_ok = fixed_row < n;
      const int t_row = row_ok ? __ldg(a.t_rel + u0 + fixed_row) : 0;
      BiasCtx bc;
      bc.tp_s = smem_u32(tab + w.head * nbt);
      bc.tt_s = bc.tp_s + 4u * a.Np;
      bc.bp_s = smem_u32(bins + w.head * nbt);
      bc.bt_s = bc.bp_s + 4u * a.Np;
      bc.tp_g = a.rab_pos + (size_t)w.head * a.Np;
      bc.tt_g = a.rab_time + (size_t)w.head * a.Nt;
      bc.bp_g = a.rab_acc + (size_t)w.head * nbt;
      bc.bt_g = bc.bp_g + a.Np;
      const int nu = n_units_of(w);
      const int row0 = first_row_of(w);
      int cur_p = -1, cur_t = -1;
      float acc_p = 0.f, acc_t = 0.f;
      bool alive = true;
      for (int u = 0; u < nu; ++u, ++g) {
        const uint32_t r = g & 1;
        const int c0 = row0 + 64 * u + cb * 16;  // streamed row of this warp's element 0
        const int tv = __ldg(a.t_rel + u0 + min(c0 + (lane & 15), n - 1));
        if (!mbar_wait_warp(s_full + r, (g >> 1) & 1, ab, a.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[16], dr[16], out[16];
        tmem_ld16(tmem + r * 64 + cb * 16 + lane_base, sr);
        tmem_ld16(tmem + C::DA_COL + r * 64 + cb * 16 + lane_base, dr);
        tmem_ld_wait();
        constexpr int HI = 4 * C::TAB_CAP;
        // every unit runs through the masked code: a second, unmasked copy of
        // the loop for the blocks inside the causal region and the user (a
        // measured 7-12 % slower) costs more in instruction fetch than the
        // masks cost
        if (in_smem) {
          bwd_elems<MODE, true, true, HI>(sr, dr, out, c0, fixed_row, row_ok, n, tv, t_row, inv_n,
                                          bc, a.Sp, a.Np, a.St, a.Nt, cur_p, cur_t, acc_p, acc_t);
        } else {
          bwd_elems<MODE, true, false, HI>(sr, dr, out, c0, fixed_row, row_ok, n, tv, t_row, inv_n,
                                           bc, a.Sp, a.Np, a.St, a.Nt, cur_p, cur_t, acc_p, acc_t);
        }
        // P^T and dS^T (DQ: dS) into the 16 columns this warp read S from
        if (MODE == MODE_DKV) tmem_st16(tmem + r * 64 + cb * 16 + lane_base, out);
        else tmem_st8(tmem + r * 64 + cb * 16 + lane_base, out);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + r);
      }
      if (MODE == MODE_DKV) {
        constexpr int HI = 4 * C::TAB_CAP;
        if (in_smem) {
          if (cur_p >= 0) bias_flush<true, HI>(bc, true, cur_p, acc_p);
          if (cur_t >= 0) bias_flush<true, HI>(bc, false, cur_t, acc_t);
        } else {
          if (cur_p >= 0) bias_flush<false, HI>(bc, true, cur_p, acc_p);
          if (cur_t >= 0) bias_flush<false, HI>(bc, false, cur_t, acc_t);
        }
      }
      if (alive) {
        // ---- epilogue: the accumulators times SiLU' of the f1 pre-activation
        if (!mbar_wait_warp(acc_full, litem & 1, ab, a.status)) {
          alive = false;
        } else {
          tc_fence_after();
          const int nacc = MODE == MODE_DKV ? 2 : 1;
          for (int ai = 0; ai < nacc; ++ai) {
            // DKV: acc0 = dV (columns of V), acc1 = dK; DQ: acc0 = dQ
            const int col0 = (MODE == MODE_DKV ? (ai == 0 ? a.v_col : a.k_col) : a.q_col) +
                             w.head * D + cb * (D / 4);
            const __half* prow = a.pre + (u0 + (row_ok ? fixed_row : 0)) * a.ld_f1 + col0;
            __half* grow = a.dP + (u0 + (row_ok ? fixed_row : 0)) * a.ld_f1 + col0;
#pragma unroll 1
            for (int c16 = 0; c16 < D / 64; ++c16) {
              uint32_t orr[16];
              tmem_ld16(tmem + C::ACC + ai * D + cb * (D / 4) + c16 * 16 + lane_base, orr);
              tmem_ld_wait();
              if (row_ok) {
                const uint4* pp = reinterpret_cast<const uint4*>(prow + c16 * 16);
                const uint4 p0 = pp[0], p1 = pp[1];
                const uint32_t pr[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                uint32_t ow[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const float x0 = f16lo(pr[k]), x1 = f16hi(pr[k]);
                  const float s0 = sigmoid_acc(x0), s1 = sigmoid_acc(x1);
                  const float g0 = __uint_as_float(orr[2 * k]) * s0 * fmaf(x0, 1.0f - s0, 1.0f);
                  const float g1 = __uint_as_float(orr[2 * k + 1]) * s1 * fmaf(x1, 1.0f - s1, 1.0f);
                  ow[k] = pack_f16x2_sat(g0, g1);
                }
                uint4* gp = reinterpret_cast<uint4*>(grow + c16 * 16);
                gp[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                gp[1] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_free);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(it_empty + slot);
      ++litem;
      if (!alive) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (MODE == MODE_DKV && in_smem) {  // this CTA's bias-gradient sums into the global ones
    for (int i = threadIdx.x; i < nbin; i += blockDim.x) {
      const unsigned long long v =
          ((unsigned long long)bins[C::TAB_CAP + i] << 32) | (unsigned long long)bins[i];
      if (v) atomicAdd(a.rab_acc + i, v);
    }
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish re-arms the work counter for the next launch
    __threadfence();
    if (atomicAdd(a.work_done, 1) == (int)gridDim.x - 1) {
      atomicExch(a.work_next, 0);
      atomicExch(a.work_done, 0);
      __threadfence();
    }
  }
}

template <int D, int MODE>
static cudaError_t launch_bwd_inst(const CUtensorMap& tf, const CUtensorMap& tdo,
                                   const CUtensorMap& tf64, const CUtensorMap& tdo64,
                                   const AttnBwdDev& ad, int grid, cudaStream_t s) {
  using C = BwdCfg<D>;
  auto kfn = k_attn_bwd<D, MODE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<grid, C::THREADS, C::SMEM, s>>>(tf, tdo, tf64, tdo64, ad);
  return cudaGetLastError();
}

static cudaError_t launch_attn_bwd_kernels(const AttnBwdCall& c, cudaStream_t s);

// drab_pos[hh][k] and drab_time[hh][k] from the fixed-point sums [h][Np + Nt].
__global__ void k_rab_grad_out(const unsigned long long* __restrict__ acc, float* __restrict__ dpos,
                               float* __restrict__ dtime, int h, int Np, int Nt,
                               const int* __restrict__ status) {
  if (status && *status != HSTU_OK) return;
  const int nbt = Np + Nt;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h * nbt; i += gridDim.x * blockDim.x) {
    const int hh = i / nbt, k = i - hh * nbt;
    const float v = (float)((double)(long long)acc[i] * (1.0 / 4294967296.0));
    if (k < Np) dpos[hh * Np + k] = v;
    else dtime[hh * Nt + (k - Np)] = v;
  }
}

cudaError_t launch_attn_bwd(const AttnBwdCall& c, cudaStream_t s) {
  if (c.dqk != c.dv || (c.dqk != 64 && c.dqk != 128)) return cudaErrorInvalidValue;
  if (!c.drab_pos || !c.drab_time || !c.rab_acc || c.ld_f1 % 8 != 0 || c.ld_do % 8 != 0)
    return cudaErrorInvalidValue;
  const int nbin = c.h * (c.Np + c.Nt);
  cudaError_t e = cudaMemsetAsync(c.rab_acc, 0, (size_t)nbin * 8, s);
  if (e != cudaSuccess) return e;
  if (c.item_cap > 0 && c.rows > 0) {
    e = launch_attn_bwd_kernels(c, s);
    if (e != cudaSuccess) return e;
  }
  LaunchScope ls(K_SUM_ROWS, s);
  k_rab_grad_out<<<(nbin + 255) / 256, 256, 0, s>>>(c.rab_acc, c.drab_pos, c.drab_time, c.h, c.Np,
                                                    c.Nt, c.status);
  return cudaGetLastError();
}

static cudaError_t launch_attn_bwd_kernels(const AttnBwdCall& c, cudaStream_t s) {
  // 128-row boxes for an item's fixed tiles, 64-row boxes for the streamed units
  CUtensorMap tf, tdo, tf64, tdo64;
  const uint64_t F = (uint64_t)c.ld_f1;
  const uint64_t HD = (uint64_t)c.h * c.dv;
  if (!encode_tmap_2d(&tf, c.f1, (uint64_t)c.rows, F, F * 2, 64, 128, true) ||
      !encode_tmap_2d(&tf64, c.f1, (uint64_t)c.rows, F, F * 2, 64, 64, true) ||
      !encode_tmap_2d(&tdo, c.dO, (uint64_t)c.rows, HD, (uint64_t)c.ld_do * 2, 64, 128, true) ||
      !encode_tmap_2d(&tdo64, c.dO, (uint64_t)c.rows, HD, (uint64_t)c.ld_do * 2, 64, 64, true))
    return cudaErrorInvalidValue;
  AttnBwdDev ad{};
  ad.items = c.items;
  ad.n_items = c.n_items;
  ad.q_col = c.q_col;
  ad.k_col = c.k_col;
  ad.v_col = c.v_col;
  ad.pre = static_cast<const __half*>(c.pre);
  ad.dP = static_cast<__half*>(c.dP);
  ad.ld_f1 = c.ld_f1;
  ad.t_rel = c.t_rel;
  ad.rab_pos = c.rab_pos;
  ad.rab_time = c.rab_time;
  ad.rab_acc = c.rab_acc;
  ad.Np = c.Np;
  ad.Nt = c.Nt;
  ad.Sp = c.Sp;
  ad.St = c.St;
  ad.h = c.h;
  ad.work_next = c.work_next;
  ad.work_done = c.work_done;
  ad.status = c.status;
  const int grid = (int)std::min<int64_t>(c.item_cap, num_sms());
  cudaError_t e;
  {
    LaunchScope ls(K_ATTN_BWD_DKV, s);
    e = c.dqk == 64 ? launch_bwd_inst<64, MODE_DKV>(tf, tdo, tf64, tdo64, ad, grid, s)
                    : launch_bwd_inst<128, MODE_DKV>(tf, tdo, tf64, tdo64, ad, grid, s);
  }
  if (e != cudaSuccess) return e;
  LaunchScope ls(K_ATTN_BWD_DQ, s);
  return c.dqk == 64 ? launch_bwd_inst<64, MODE_DQ>(tf, tdo, tf64, tdo64, ad, grid, s)
                     : launch_bwd_inst<128, MODE_DQ>(tf, tdo, tf64, tdo64, ad, grid, s);
}

}  // namespace hstu

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
//     query tiles i >= j, recomputing S^T = K_j Q_i^T and dA^T = V_j dO_i^T in
//     tensor memory (one TMEM lane per key row), forms P^T = SiLU(S^T)/n and
//     dS^T in fp16 in shared memory, and accumulates dV_j += P^T dO_i and
//     dK_j += dS^T Q_i in tensor memory; it also sums dS into the bias
//     gradients.  The epilogue multiplies dK, dV by SiLU' of the f1
//     pre-activation (the gradient of f1's own SiLU) and stores them into
//     the f1-shaped gradient buffer.
//   MODE_DQ: one work item = (user, query tile i, head); it walks the KV tiles
//     j <= i, recomputing S = Q_i K_j^T and dA = dO_i V_j^T, forms dS, and
//     accumulates dQ_i += dS K_j.
// Computing dQ in its own pass costs two more MMAs per tile pair but needs no
// atomic accumulation of dQ across KV tiles.
//
// Roles (384 threads): warp 0 lane 0 issues the TMA loads (the item's fixed
// tiles once, the streamed tiles through a ring), warp 1 lane 0 issues the
// MMAs, warp 2 claims items (dynamic scheduling) into a 2-slot ring, warps 4-11
// (two per TMEM lane quarter, 64 of the 128 columns each) do the elementwise
// work and the epilogue.  Every wait is bounded.
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
  float* drab_pos;          // MODE_DKV: [h, Np] fp32, accumulated (atomic adds)
  float* drab_time;         // MODE_DKV: [h, Nt]
  int Np, Nt, Sp, St, h;
  int32_t* work_next;
  int32_t* work_done;
  int* status;
};

template <int D>
struct BwdCfg {
  static constexpr uint32_t TILE = 128u * D * 2;   // one [128 x D] fp16 tile
  static constexpr int RING = D == 64 ? 2 : 1;    // streamed tile-pair stages
  static constexpr uint32_t FIX_OFF = 0;            // 2 fixed tiles
  static constexpr uint32_t STR_OFF = FIX_OFF + 2 * TILE;   // RING x 2 streamed tiles
  static constexpr uint32_t PS_OFF = STR_OFF + RING * 2 * TILE;  // P^T and dS (2 x 32 KB)
  // MODE_DKV: this CTA's bias-table gradient sums ([h][Np + Nt] fp32, when
  // they fit), added to the global tables once at the end
  static constexpr int BIN_FLOATS = 4096;
  static constexpr uint32_t BIN_OFF = PS_OFF + 2 * 32768;
  static constexpr uint32_t BAR_OFF = BIN_OFF + BIN_FLOATS * 4;
  static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
  static constexpr int EW0 = 4, NEW = 8;            // elementwise warps 4..11
  static constexpr int THREADS = 32 * (EW0 + NEW);
  static constexpr uint32_t ACC = 256;              // TMEM: S | dA | acc0 | acc1
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

DEVI float sigmoid_acc(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// Writes a 32-wide chunk (columns c0..c0+31 of a 128 x 128 fp16 K-major
// operand in two 64-column swizzle atoms) of row r.
DEVI void st_op_chunk(uint8_t* base, int r, int c0, const uint32_t (&w)[16]) {
  uint8_t* atom = base + (c0 >> 6) * 16384 + r * 128;
  const int ch0 = (c0 & 63) >> 3;  // first 16-byte chunk in the 128-byte row
#pragma unroll
  for (int k = 0; k < 4; ++k)
    *reinterpret_cast<uint4*>(atom + (((ch0 + k) ^ (r & 7)) << 4)) =
        make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
}

template <int D, int MODE>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmdO,
               const AttnBwdDev a) {
  using C = BwdCfg<D>;
  constexpr int NA = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* fix_full = bars + 0;
  uint64_t* fix_empty = bars + 1;
  uint64_t* str_full = bars + 2;    // [2]
  uint64_t* str_empty = bars + 4;   // [2]
  uint64_t* s_full = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* pd_free = bars + 8;
  uint64_t* acc_full = bars + 9;
  uint64_t* acc_free = bars + 10;
  uint64_t* it_full = bars + 11;    // [2]
  uint64_t* it_empty = bars + 13;   // [2]
  uint64_t* drain = bars + 15;
  AttnItem* ring = reinterpret_cast<AttnItem*>(bars + 16);   // [2] x 32 B
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + 2);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
  int* s_go = reinterpret_cast<int*>(ab + 1);
  int* s_nitems = s_go + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // bias-gradient bins in shared memory when every head's tables fit (shared
  // atomics; the many CTAs of a head would otherwise all add into the same
  // few global words near the diagonal's buckets)
  float* bins = reinterpret_cast<float*>(smem + C::BIN_OFF);
  const int nbin = a.h * (a.Np + a.Nt);
  const bool use_bins = MODE == MODE_DKV && nbin <= C::BIN_FLOATS;
  if (use_bins)
    for (int i = threadIdx.x; i < nbin; i += blockDim.x) bins[i] = 0.f;
  if (threadIdx.x == 0) {
    const int st = a.status ? *reinterpret_cast<volatile int*>(a.status) : 0;
    *s_go = (st == 0);
    *s_nitems = *a.n_items;
    ab->flag = 0;
    ab->limit_us = kWaitLimitUs;
    mbar_init(fix_full, 1);
    mbar_init(fix_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(str_full + i, 1);
      mbar_init(str_empty + i, 1);
      mbar_init(it_full + i, 1);
      mbar_init(it_empty + i, 2 + C::NEW);  // loader, MMA thread, elementwise warps
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, C::NEW);
    mbar_init(pd_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, C::NEW);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmF);
    tma_prefetch_desc(&tmdO);
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
  uint8_t* sP = smem + C::PS_OFF;          // MODE_DKV: P^T
  uint8_t* sS = smem + C::PS_OFF + 32768;  // dS (MODE_DKV: dS^T)

  // Tile counts of an item: DKV walks query tiles j..nq-1, DQ kv tiles 0..i.
  auto n_tiles_of = [&](const AttnItem& w) -> int {
    const int nq = (w.n_q + 127) / 128;
    return MODE == MODE_DKV ? nq - w.qt : w.qt + 1;
  };

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
        // previous item's last MMA has read them
        if (!mbar_wait(fix_empty, (litem & 1) ^ 1, ab, a.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(fix_full, 2 * C::TILE);
        const int r0 = w.kv_row0 + w.qt * 128;  // rows of tile qt of this user
#pragma unroll
        for (int at = 0; at < NA; ++at) {
          if (MODE == MODE_DKV) {
            tma_load_2d(sFix + at * 16384, &tmF, a.k_col + w.head * D + at * 64, r0, fix_full);
            tma_load_2d(sFix + C::TILE + at * 16384, &tmF, a.v_col + w.head * D + at * 64, r0,
                        fix_full);
          } else {
            tma_load_2d(sFix + at * 16384, &tmF, a.q_col + w.head * D + at * 64, r0, fix_full);
            tma_load_2d(sFix + C::TILE + at * 16384, &tmdO, w.head * D + at * 64, r0, fix_full);
          }
        }
        fix_issued = true;
        fix_par = litem & 1;
        const int nt = n_tiles_of(w);
        for (int t = 0; t < nt; ++t) {
          const int tile = MODE == MODE_DKV ? w.qt + t : t;   // the streamed tile's index
          const int rr = w.kv_row0 + tile * 128;
          if (!mbar_wait(str_empty + st, ph ^ 1, ab, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(str_full + st, 2 * C::TILE);
          uint8_t* dst = sStr + st * 2 * C::TILE;
#pragma unroll
          for (int at = 0; at < NA; ++at) {
            if (MODE == MODE_DKV) {  // Q_i, dO_i
              tma_load_2d(dst + at * 16384, &tmF, a.q_col + w.head * D + at * 64, rr, str_full + st);
              tma_load_2d(dst + C::TILE + at * 16384, &tmdO, w.head * D + at * 64, rr, str_full + st);
            } else {                 // K_j, V_j
              tma_load_2d(dst + at * 16384, &tmF, a.k_col + w.head * D + at * 64, rr, str_full + st);
              tma_load_2d(dst + C::TILE + at * 16384, &tmF, a.v_col + w.head * D + at * 64, rr,
                          str_full + st);
            }
          }
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (ph << st);
          if (++st == (uint32_t)C::RING) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        ++litem;
      }
      if (!ok) {  // every load in flight lands before the CTA exits
        AbortState tmp{0, kWaitLimitUs};
        for (int s2 = 0; s2 < C::RING; ++s2)
          if ((issued >> s2) & 1u) mbar_wait(str_full + s2, (last_par >> s2) & 1u, &tmp, nullptr);
        if (fix_issued) mbar_wait(fix_full, fix_par, &tmp, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f16_f32(128, 128, 0, 0, 1);
      constexpr uint32_t IDESC_ACC = idesc_f16_f32(128, D, 0, 1, 1);  // B MN-major
      uint32_t ncon = 0, st = 0, ph = 0, g = 0;
      int litem = 0;
      bool ok = true, any = false;
      const uint32_t fix0 = smem_u32(sFix);
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
        if (!mbar_wait(fix_full, litem & 1, ab, a.status)) {
          ok = false;
          break;
        }
        const int nt = n_tiles_of(w);
        for (int t = 0; t < nt; ++t, ++g) {
          if (!mbar_wait(str_full + st, ph, ab, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t str0 = smem_u32(sStr + st * 2 * C::TILE);
          // S (or S^T) = A0 B0^T and dA (or dA^T) = A1 B1^T over D:
          // DKV: A0 = K_j, B0 = Q_i, A1 = V_j, B1 = dO_i; DQ: A0 = Q_i, B0 = K_j,
          // A1 = dO_i, B1 = V_j (all K-major [128 x D] tiles)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc_mma_f16_ss(tmem, sdesc_sw128(fix0 + o, 16, 1024), sdesc_sw128(str0 + o, 16, 1024),
                          IDESC_S, kk > 0 ? 1u : 0u);
            tc_mma_f16_ss(tmem + 128, sdesc_sw128(fix0 + C::TILE + o, 16, 1024),
                          sdesc_sw128(str0 + C::TILE + o, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          any = true;
          if (!mbar_wait(p_full, g & 1, ab, a.status)) {
            ok = false;
            break;
          }
          if (t == 0 && litem > 0 && !mbar_wait(acc_free, (litem - 1) & 1, ab, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sP0 = smem_u32(sP), sS0 = smem_u32(sS);
          // 128-wide contraction over the streamed tile's rows, 16 per MMA:
          // A = P^T / dS^T / dS (K-major, two 64-column atoms), B = the
          // streamed (DKV: dO_i, Q_i) or (DQ: K_j) tile read MN-major
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
            if (MODE == MODE_DKV) {
              tc_mma_f16_ss(tmem + C::ACC, sdesc_sw128(sP0 + ao, 16, 1024),
                            sdesc_sw128(str0 + C::TILE + kk * 2048, 16384, 1024), IDESC_ACC, acc);
              tc_mma_f16_ss(tmem + C::ACC + D, sdesc_sw128(sS0 + ao, 16, 1024),
                            sdesc_sw128(str0 + kk * 2048, 16384, 1024), IDESC_ACC, acc);
            } else {
              tc_mma_f16_ss(tmem + C::ACC, sdesc_sw128(sS0 + ao, 16, 1024),
                            sdesc_sw128(str0 + kk * 2048, 16384, 1024), IDESC_ACC, acc);
            }
          }
          tc_commit(pd_free);
          tc_commit(str_empty + st);
          if (t == nt - 1) {
            tc_commit(acc_full);
            tc_commit(fix_empty);
          }
          if (++st == (uint32_t)C::RING) {
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
    const int half = ew >> 2;         // columns half*64 .. half*64+63
    const int r = q * 32 + lane;      // row of this thread inside the 128-row tile
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
      const int fixed_row = w.qt * 128 + r;      // this thread's row within the user
      const bool row_ok = fixed_row < n;
      const int t_row = row_ok ? __ldg(a.t_rel + u0 + fixed_row) : 0;
      const float* Rp = a.rab_pos + (size_t)w.head * a.Np;
      const float* Rt = a.rab_time + (size_t)w.head * a.Nt;
      float* dRp = use_bins ? bins + (size_t)w.head * (a.Np + a.Nt)
                            : a.drab_pos + (size_t)w.head * a.Np;
      float* dRt = use_bins ? bins + (size_t)w.head * (a.Np + a.Nt) + a.Np
                            : a.drab_time + (size_t)w.head * a.Nt;
      const int nt = n_tiles_of(w);
      bool alive = true;
      for (int t = 0; t < nt; ++t, ++g) {
        const int tile = MODE == MODE_DKV ? w.qt + t : t;   // the streamed tile's index
        if (!mbar_wait_warp(s_full, g & 1, ab, a.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        // run-length sums of dS per bias bucket along this thread's row
        int cur_p = -1, cur_t = -1;
        float acc_p = 0.f, acc_t = 0.f;
        uint32_t pw[2][16], sw[2][16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c0 = half * 64 + cc * 32;
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + c0 + lane_base, sr);
          tmem_ld32(tmem + 128 + c0 + lane_base, dr);
          tmem_ld_wait();
          // branch-free over the 32 elements: masked ones give P = dS = 0
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = tile * 128 + c0 + e;              // streamed row within the user
            const int qi = MODE == MODE_DKV ? col : fixed_row;  // query row i
            const int kj = MODE == MODE_DKV ? fixed_row : col;  // key row j
            const bool ok_e = row_ok && col < n && kj <= qi;
            const int tcol = __ldg(a.t_rel + u0 + min(col, n - 1));
            const int ti = MODE == MODE_DKV ? tcol : t_row;
            const int tj = MODE == MODE_DKV ? t_row : tcol;
            const int bp = (int)log_bucket_nb(max(qi - kj, 0), a.Sp, a.Np);
            const int bt = (int)log_bucket_nb(max(ti - tj, 0), a.St, a.Nt);
            const float s = __uint_as_float(sr[e]) + __ldg(Rp + bp) + __ldg(Rt + bt);
            const float sg = sigmoid_acc(s);
            const float p = ok_e ? s * sg * inv_n : 0.f;
            const float ds = ok_e ? __uint_as_float(dr[e]) * inv_n * sg * fmaf(s, 1.0f - sg, 1.0f)
                                  : 0.f;
            sr[e] = __float_as_uint(p);
            dr[e] = __float_as_uint(ds);
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            pw[cc][e >> 1] = pack_f16x2_sat(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            sw[cc][e >> 1] = pack_f16x2_sat(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1]));
          }
          if (MODE == MODE_DKV) {
            // the bias-table gradients: buckets change rarely along a row, so
            // one atomic add per run of equal buckets
#pragma unroll 4
            for (int e = 0; e < 32; ++e) {
              const int col = tile * 128 + c0 + e;
              if (!(row_ok && col < n && fixed_row <= col)) continue;
              const float ds = __uint_as_float(dr[e]);
              const int bp = (int)log_bucket_nb(col - fixed_row, a.Sp, a.Np);
              const int bt =
                  (int)log_bucket_nb(max(__ldg(a.t_rel + u0 + col) - t_row, 0), a.St, a.Nt);
              if (bp != cur_p) {
                if (cur_p >= 0) atomicAdd(dRp + cur_p, acc_p);
                cur_p = bp;
                acc_p = 0.f;
              }
              acc_p += ds;
              if (bt != cur_t) {
                if (cur_t >= 0) atomicAdd(dRt + cur_t, acc_t);
                cur_t = bt;
                acc_t = 0.f;
              }
              acc_t += ds;
            }
          }
        }
        if (MODE == MODE_DKV) {
          if (cur_p >= 0) atomicAdd(dRp + cur_p, acc_p);
          if (cur_t >= 0) atomicAdd(dRt + cur_t, acc_t);
        }
        tc_fence_before();
        // P^T / dS may be written once the previous tile's MMAs have read them
        if (g > 0 && !mbar_wait_warp(pd_free, (g - 1) & 1, ab, a.status)) {
          alive = false;
          break;
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          if (MODE == MODE_DKV) st_op_chunk(sP, r, half * 64 + cc * 32, pw[cc]);
          st_op_chunk(sS, r, half * 64 + cc * 32, sw[cc]);
        }
        fence_proxy_async_smem();  // the tensor cores read what these threads wrote
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
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
                             w.head * D + half * (D / 2);
            const __half* prow = a.pre + (u0 + (row_ok ? fixed_row : 0)) * a.ld_f1 + col0;
            __half* grow = a.dP + (u0 + (row_ok ? fixed_row : 0)) * a.ld_f1 + col0;
#pragma unroll 1
            for (int c16 = 0; c16 < D / 32; ++c16) {
              uint32_t orr[16];
              tmem_ld16(tmem + C::ACC + ai * D + half * (D / 2) + c16 * 16 + lane_base, orr);
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
  if (use_bins) {  // this CTA's bias-gradient sums into the global tables
    for (int i = threadIdx.x; i < nbin; i += blockDim.x) {
      const float v = bins[i];
      if (v != 0.f) {
        const int hh = i / (a.Np + a.Nt), k = i - hh * (a.Np + a.Nt);
        if (k < a.Np) atomicAdd(a.drab_pos + (size_t)hh * a.Np + k, v);
        else atomicAdd(a.drab_time + (size_t)hh * a.Nt + (k - a.Np), v);
      }
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
                                   const AttnBwdDev& ad, int grid, cudaStream_t s) {
  using C = BwdCfg<D>;
  auto kfn = k_attn_bwd<D, MODE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<grid, C::THREADS, C::SMEM, s>>>(tf, tdo, ad);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const AttnBwdCall& c, cudaStream_t s) {
  if (c.dqk != c.dv || (c.dqk != 64 && c.dqk != 128)) return cudaErrorInvalidValue;
  if (c.item_cap <= 0 || c.rows <= 0) return cudaSuccess;
  if (!c.drab_pos || !c.drab_time || c.ld_f1 % 8 != 0 || c.ld_do % 8 != 0)
    return cudaErrorInvalidValue;
  CUtensorMap tf, tdo;
  const uint64_t F = (uint64_t)c.ld_f1;
  if (!encode_tmap_2d(&tf, c.f1, (uint64_t)c.rows, F, F * 2, 64, 128, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tdo, c.dO, (uint64_t)c.rows, (uint64_t)c.h * c.dv, (uint64_t)c.ld_do * 2,
                      64, 128, true))
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
  ad.drab_pos = c.drab_pos;
  ad.drab_time = c.drab_time;
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
    e = c.dqk == 64 ? launch_bwd_inst<64, MODE_DKV>(tf, tdo, ad, grid, s)
                    : launch_bwd_inst<128, MODE_DKV>(tf, tdo, ad, grid, s);
  }
  if (e != cudaSuccess) return e;
  LaunchScope ls(K_ATTN_BWD_DQ, s);
  return c.dqk == 64 ? launch_bwd_inst<64, MODE_DQ>(tf, tdo, ad, grid, s)
                     : launch_bwd_inst<128, MODE_DQ>(tf, tdo, ad, grid, s);
}

}  // namespace hstu

// gemm_tc.cu — GEMM on the 5th-generation tensor cores (tcgen05) with fused
// epilogues, used for both projections of the HSTU layer and for catalog
// scoring:
//   f1:  G = SiLU(X W1^T + b1)         (EPI_SILU; output = [U | V | Q | K])
//   f2:  Y = X + Z W2^T + b2           (EPI_RESID)
//   scores: S = H E^T                  (EPI_SCORE; fp32, ragged item count)
//   plain:  C = A W^T + b              (EPI_BIAS; 16-bit output)
//   filter: (score, column) of A W^T at or above a per-row threshold, appended
//           to per-row candidate lists (EPI_FILTER; nothing else is stored)
// ('HSTUとGenerative Recommenders', section 'HSTUはTransformerと何が違うのか':
// one projection f1 followed by SiLU and a split; f2 back to d_model plus
// the residual connection.)
//
// Design (B200, sm_100a): persistent CTAs (one per SM), 128 x BN output tiles
// walked n-fastest so that a wave of CTAs shares the A rows through L2.
// Warp 0 streams A and W tiles with TMA (128-byte swizzle) into a STAGES-deep
// ring; warp 1 issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM
// accumulators; warps 2-9 (two per TMEM lane quarter, half of the columns
// each) drain the other accumulator 32 columns at a time, loading the next
// chunk (accumulator and bias) while they finish the current one, and write
// each 32 x 32 result through a swizzled shared-memory buffer with TMA bulk
// tensor stores (whole lines, asynchronous).  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>

#include "ptx.cuh"

namespace hstu {

struct GemmDev {
  int64_t M_cap;
  const int64_t* M_dev;
  int N, K, n_off;
  int ab_f16;                  // operand format: fp16 (1) or bf16 (0)
  const __nv_bfloat16* bias;
  int has_out16;               // 16-bit output (fp16 if out_f16, else bf16)
  int out_f16;
  int has_out32;               // EPI_RESID: fp32 copy of the output
  const void* resid;           // EPI_RESID: residual (resid_kind: bf16, fp32 or fp16)
  int64_t ldr;
  int resid_kind;
  int* status;
  const int* run_if;           // if set, the launch does nothing unless *run_if != 0
  // EPI_FILTER: per-row threshold and candidate lists
  const float* tau;
  int tau_stride;
  uint32_t* cand_key;
  int32_t* cand_id;
  int* cand_cnt;
  int cand_cap;
  int* overflow;
  // LNA: the A operand is LayerNorm(O) * U, built in shared memory
  const __half* ln_x;          // normalised O [M, K] fp16: (O - m) / s per (row, head)
  const uint32_t* ln_coef;     // [M, ln_h] (a, b) fp16 pairs per (row, head)
  const __half* ln_u;          // U: the first K columns of the f1 output, row stride ld_u
  int64_t ld_u;
  const __nv_bfloat16* ln_gamma;
  const __nv_bfloat16* ln_beta;
  float ln_eps;
  int ln_h, ln_dv;
  __half* z_dbg;               // optional: Z [M, K] fp16, written by the CTAs of n-tile 0
  // split-K: the K blocks are cut into `splits` ranges of kb_split blocks;
  // split s stores its partial product at output rows s * split_rows + m
  int splits, kb_split;
  int64_t split_rows;
  int has_pre;                 // EPI_SILU: also store the pre-activation (16-bit, tmO32)
};

constexpr int kEpiThreads = 256;      // 8 epilogue warps
constexpr int kLnaThreads = 128;      // LNA: 4 warps that form the A operand
constexpr int kLnaRows = 128 / (kLnaThreads / 8);  // rows of each K block per such thread
constexpr uint32_t kStageBuf = 4096;  // per-warp output staging bytes (32 x 32 fp32)

// COMPACT (EPI_RESID with 16-bit residual and output only): 2 KB output and
// 2 KB residual buffers per epilogue warp, leaving room for one more A/B stage.
// LNA: TMA brings the normalised attention output (as A) and U; the epilogue
// warps turn A into LayerNorm(O) * U in place before the MMAs read it.
template <int BN, int STAGES, int EPI, int COMPACT, int LNA = 0>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  // LNA: each stage also holds the U tile; A arrives as the normalised O and
  // is turned into Z in place
  static constexpr uint32_t U_BYTES = LNA ? A_BYTES : 0;
  static constexpr uint32_t B_OFF = A_BYTES + U_BYTES;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + U_BYTES + B_BYTES;
  static constexpr uint32_t BUF = COMPACT ? 2048 : kStageBuf;         // per-warp buffers
  static constexpr uint32_t OUT_OFF = STAGES * STAGE_BYTES;             // 8 output staging buffers
  // EPI_RESID: 8 buffers that TMA fills with the next residual chunk
  static constexpr uint32_t RES_OFF = OUT_OFF + (kEpiThreads / 32) * BUF;
  static constexpr uint32_t BAR_OFF = RES_OFF + (EPI == EPI_RESID ? (kEpiThreads / 32) * BUF : 0);
  static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr int THREADS = 64 + kEpiThreads + (LNA ? kLnaThreads : 0);
};



// Applies the epilogue to one 32-column chunk of this thread's row and stores
// the warp's 32 x 32 tile: the fp32 copy through a 128-byte-swizzled buffer
// and/or the 16-bit output through a 64-byte-swizzled one, each with one TMA
// store issued by lane 0.  `stage` is the warp's 4 KB buffer; `parity` picks
// the 2 KB half of a 16-bit-only output (double buffering).  Returns whether
// the warp stored anything (not when all its 32 rows are past the end).
template <int EPI>
DEVI bool gemm_chunk(const GemmDev& g, const CUtensorMap* tmO16, const CUtensorMap* tmO32,
                     int64_t row, bool valid, int col, int y0, const uint32_t (&r)[32],
                     const uint4 (&bias)[4], uint8_t* stage, int parity, const uint8_t* rsm) {
  const int lane = threadIdx.x & 31;
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t bw[4] = {bias[i].x, bias[i].y, bias[i].z, bias[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[i * 8 + 2 * k] = __uint_as_float(r[i * 8 + 2 * k]) + bf16lo(bw[k]);
      v[i * 8 + 2 * k + 1] = __uint_as_float(r[i * 8 + 2 * k + 1]) + bf16hi(bw[k]);
    }
  }
  if (EPI == EPI_SCORE) {
    if (col >= g.N) return false;  // a chunk past the last item: nothing to store
  } else if (EPI == EPI_SILU) {
    if (g.has_pre) {
      // the pre-activation X W^T + b through the first 2 KB of the warp's
      // buffer (16-bit, 64-byte swizzle), then SiLU through the second
      if (__shfl_sync(0xffffffffu, valid ? 1 : 0, 0) == 0) return false;
      if (lane == 0) bulk_wait_read<1>();  // the pre store before the last one has read it
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4 o;
        o.x = pack16(g.out_f16, v[k * 8 + 0], v[k * 8 + 1]);
        o.y = pack16(g.out_f16, v[k * 8 + 2], v[k * 8 + 3]);
        o.z = pack16(g.out_f16, v[k * 8 + 4], v[k * 8 + 5]);
        o.w = pack16(g.out_f16, v[k * 8 + 6], v[k * 8 + 7]);
        sts_u128(smem_u32(stage) + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4), o);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmO32, col, y0, stage);
        bulk_commit();
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = silu_accurate(v[i]);
  } else if (EPI == EPI_BIAS) {
    // bias only
  } else if (g.resid_kind == RESID_F32) {  // residual chunk staged by TMA, 128-byte swizzle
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 rr = lds_u128(smem_u32(rsm) + lane * 128 + ((k ^ (lane & 7)) << 4));
      v[4 * k + 0] += __uint_as_float(rr.x);
      v[4 * k + 1] += __uint_as_float(rr.y);
      v[4 * k + 2] += __uint_as_float(rr.z);
      v[4 * k + 3] += __uint_as_float(rr.w);
    }
  } else {  // 16-bit residual chunk staged by TMA, 64-byte swizzle
    const int f16 = g.resid_kind == RESID_F16;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 rr = lds_u128(smem_u32(rsm) + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4));
      const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        if (f16) {  // packed conversion of the pair
          const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&rw[m]));
          v[k * 8 + 2 * m] += p.x;
          v[k * 8 + 2 * m + 1] += p.y;
        } else {
          v[k * 8 + 2 * m] += bf16lo(rw[m]);
          v[k * 8 + 2 * m + 1] += bf16hi(rw[m]);
        }
      }
    }
  }
  if (__shfl_sync(0xffffffffu, valid ? 1 : 0, 0) == 0) return false;  // rows y0.. all invalid
  const bool both = ((EPI == EPI_RESID) && g.has_out32) || EPI == EPI_SCORE;
  if (both) {
    if (lane == 0) bulk_wait_read<0>();  // the warp's earlier stores have read the buffer
    __syncwarp();
    const uint32_t rowp = smem_u32(stage) + lane * 128;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      sts_u128(rowp + ((k ^ (lane & 7)) << 4),
               make_uint4(__float_as_uint(v[4 * k]), __float_as_uint(v[4 * k + 1]),
                          __float_as_uint(v[4 * k + 2]), __float_as_uint(v[4 * k + 3])));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmO32, col, y0, stage);
      bulk_commit();
    }
  }
  if (EPI != EPI_SCORE && g.has_out16) {
    // parity < 0: one 2 KB buffer (wait for the previous store to read it);
    // with a pre-activation store, the second 2 KB half
    const bool pre = EPI == EPI_SILU && g.has_pre;
    uint8_t* buf = stage + (pre ? 2048 : ((both || parity < 0) ? 0 : parity * 2048));
    if (lane == 0) {
      if ((both || parity < 0) && !pre) bulk_wait_read<0>();
      else bulk_wait_read<1>();
    }
    __syncwarp();
    const uint32_t rowp = smem_u32(buf) + lane * 64;
    const int f16 = g.out_f16;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint4 o;
      o.x = pack16(f16, v[k * 8 + 0], v[k * 8 + 1]);
      o.y = pack16(f16, v[k * 8 + 2], v[k * 8 + 3]);
      o.z = pack16(f16, v[k * 8 + 4], v[k * 8 + 5]);
      o.w = pack16(f16, v[k * 8 + 6], v[k * 8 + 7]);
      sts_u128(rowp + ((k ^ ((lane >> 1) & 3)) << 4), o);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmO16, col, y0, buf);
      bulk_commit();
    }
  }
  return true;
}

// EPI_FILTER: this lane's row, 32 columns from `col`: scores whose key is at
// most the row's threshold key are appended to the row's candidate list.
DEVI void gemm_filter_chunk(const GemmDev& g, int64_t row, bool valid, int col,
                            const uint32_t (&r)[32], uint32_t thr) {
  if (!valid || col >= g.N) return;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t key = desc_key(__uint_as_float(r[i]));
    if (key <= thr && col + i < g.N) {
      const int idx = atomicAdd(g.cand_cnt + row, 1);
      if (idx < g.cand_cap) {
        g.cand_key[row * g.cand_cap + idx] = key;
        g.cand_id[row * g.cand_cap + idx] = col + i;
      } else {
        *reinterpret_cast<volatile int*>(g.overflow) = 1;
      }
    }
  }
}

// MAJ: bit 0 = A is MN-major (stored [K, M] row-major), bit 1 = W is
// MN-major (stored [K, N] row-major); both arrive as 64 x 64 boxes.
template <int BN, int STAGES, int EPI, int COMPACT, int LNA, int MAJ>
__global__ void __launch_bounds__(GemmCfg<BN, STAGES, EPI, COMPACT, LNA>::THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmO16,
              const __grid_constant__ CUtensorMap tmO32, const __grid_constant__ CUtensorMap tmR,
              const __grid_constant__ CUtensorMap tmU, const GemmDev g) {
  using C = GemmCfg<BN, STAGES, EPI, COMPACT, LNA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* rbar = drain + 1;  // [8] residual chunk landed (per epilogue warp)
  uint64_t* afull = rbar + 8;  // [STAGES] LNA: the A tile has been turned into Z
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + STAGES);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
  int* s_go = reinterpret_cast<int*>(ab + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    *s_go = ((g.status == nullptr) || (*reinterpret_cast<volatile int*>(g.status) == 0)) &&
            (g.run_if == nullptr || *reinterpret_cast<volatile const int*>(g.run_if) != 0);
    ab->flag = 0;
    ab->limit_us = kWaitLimitUs;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      mbar_init(afull + s, kLnaThreads / 32);  // LNA: one arrival per A-building warp
    }
    mbar_init(tfull + 0, 1);
    mbar_init(tfull + 1, 1);
    mbar_init(tempty + 0, kEpiThreads / 32);
    mbar_init(tempty + 1, kEpiThreads / 32);
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(rbar + i, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  __syncthreads();
  if (!*s_go) return;

  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int64_t Mrows = g.M_cap;
  if (g.M_dev) {
    const int64_t m = *g.M_dev;
    Mrows = m < Mrows ? m : Mrows;
  }
  if (Mrows < 0) Mrows = 0;
  const int n_tiles = (g.N + BN - 1) / BN;  // the scores' last tile may be ragged
  const int m_tiles = (int)((Mrows + 127) / 128);
  const int mn_tiles = m_tiles * n_tiles;
  const int tiles = mn_tiles * g.splits;
  const int KB = (g.K + 63) / 64;
  // K blocks [kb_lo, kb_hi) of work unit t (split t / mn_tiles)
  auto kb_range = [&](int t_, int& lo, int& hi) {
    const int sp = t_ / mn_tiles;
    lo = sp * g.kb_split;
    hi = min(KB, lo + g.kb_split);
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mn = t % mn_tiles;
        const int mt = mn / n_tiles, nt = mn - (mn / n_tiles) * n_tiles;
        int kb_lo, kb_hi;
        kb_range(t, kb_lo, kb_hi);
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(empty + stage, ph ^ 1, ab, g.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(full + stage, C::STAGE_BYTES);
          if (LNA) {  // the normalised O (in A's place) and U; Z is formed in place
            tma_load_2d(sa, &tmA, kb * 64, mt * 128, full + stage);
            tma_load_2d(sa + C::A_BYTES, &tmU, kb * 64, mt * 128, full + stage);
          } else {
            if (MAJ & 1) {  // [K, M] source: two 64 (m) x 64 (k) boxes
              tma_load_2d(sa, &tmA, mt * 128, kb * 64, full + stage);
              tma_load_2d(sa + 8192, &tmA, mt * 128 + 64, kb * 64, full + stage);
            } else {
              tma_load_2d(sa, &tmA, kb * 64, mt * 128, full + stage);
            }
          }
          if (MAJ & 2) {  // [K, N] source: BN / 64 boxes of 64 (n) x 64 (k)
#pragma unroll
            for (int a = 0; a < BN / 64; ++a)
              tma_load_2d(sa + C::B_OFF + a * 8192, &tmB, g.n_off + nt * BN + a * 64, kb * 64,
                          full + stage);
          } else {
            tma_load_2d(sa + C::B_OFF, &tmB, kb * 64, g.n_off + nt * BN, full + stage);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (ph << stage);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {  // let every load already in flight land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) {
            AbortState tmp{0, kWaitLimitUs};
            mbar_wait(full + s, (last_par >> s) & 1u, &tmp, nullptr);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t IDESC = idesc_f16_f32(128, BN, MAJ & 1, (MAJ >> 1) & 1, g.ab_f16);
      int stage = 0, local = 0;
      uint32_t ph = 0;
      bool ok = true, issued_any = false;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
        int kb_lo, kb_hi;
        kb_range(t, kb_lo, kb_hi);
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait(tempty + acc, aph ^ 1, ab, g.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          // LNA: A holds Z once the epilogue warps have turned it (which they do
          // after the stage's loads landed)
          if (!mbar_wait(LNA ? afull + stage : full + stage, ph, ab, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::B_OFF;
          // K-major: the 16-wide K step is 32 bytes along a 128-byte row;
          // MN-major: 16 rows of 128 bytes, 64-element MN chunks 8 KB apart
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ss(d_tmem,
                          (MAJ & 1) ? sdesc_sw128(a0 + k * 2048, 8192, 1024)
                                    : sdesc_sw128(a0 + k * 32, 16, 1024),
                          (MAJ & 2) ? sdesc_sw128(b0 + k * 2048, 8192, 1024)
                                    : sdesc_sw128(b0 + k * 32, 16, 1024),
                          IDESC, (kb != kb_lo || k != 0) ? 1u : 0u);
          tc_commit(empty + stage);
          issued_any = true;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (ok) tc_commit(tfull + acc);
      }
      if (issued_any) {
        tc_commit(drain);  // completes once every MMA issued above has finished
        AbortState tmp{0, kWaitLimitUs};
        mbar_wait(drain, 0, &tmp, nullptr);
      }
    }
  } else if (warp < 2 + kEpiThreads / 32) {
    const int q = warp & 3;              // TMEM lane quarter this warp may read
    const int part = (warp - 2) >> 2;    // which half of the BN columns
    constexpr int CH = BN / 64;          // 32-column chunks per warp
    uint8_t* stage = smem + C::OUT_OFF + (warp - 2) * C::BUF;
    int local = 0, nchunk = 0;
    // residual: lane 0 has TMA bring the next 32 x 32 chunk into the warp's
    // buffer while the current one is computed and stored
    const bool rtma = (EPI == EPI_RESID);
    const uint32_t rbytes = g.resid_kind == RESID_F32 ? 4096u : 2048u;
    uint8_t* rbuf = smem + C::RES_OFF + (warp - 2) * C::BUF;
    uint64_t* rb = rbar + (warp - 2);
    uint32_t rpar = 0;
    bool r_pending = false;
    auto r_issue = [&](int t_, int c_) {  // (a residual is added only without split-K)
      const int mn_ = t_ % mn_tiles;
      const int mt_ = mn_ / n_tiles, nt_ = mn_ - (mn_ / n_tiles) * n_tiles;
      mbar_arrive_expect_tx(rb, rbytes);
      tma_load_2d(rbuf, &tmR, g.n_off + nt_ * BN + part * (BN / 2) + c_ * 32, mt_ * 128 + q * 32,
                  rb);
    };
    if (rtma && lane == 0 && (int)blockIdx.x < tiles) {
      r_issue(blockIdx.x, 0);
      r_pending = true;
    }
    // Drains the accumulator of tile t (this CTA's local-th) through the
    // epilogue and frees it for the MMAs.  Returns false if a wait gave up.
    auto epi_tile = [&](int t) -> bool {
      const int sp = t / mn_tiles, mn = t % mn_tiles;
      const int mt = mn / n_tiles, nt = mn - (mn / n_tiles) * n_tiles;
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      ++local;
      const int col0 = g.n_off + nt * BN + part * (BN / 2);
      const uint4* bptr = reinterpret_cast<const uint4*>(g.bias + col0);
      uint4 ba[4], bb[4];
      constexpr bool kNoBias = EPI == EPI_SCORE || EPI == EPI_FILTER;
#pragma unroll
      for (int i = 0; i < 4; ++i) ba[i] = kNoBias ? make_uint4(0, 0, 0, 0) : __ldg(bptr + i);
      if (!mbar_wait_warp(tfull + acc, aph, ab, g.status)) return false;
      tc_fence_after();
      const int64_t row = (int64_t)mt * 128 + q * 32 + lane;
      const bool valid = row < Mrows;
      const int y0 = (int)(sp * g.split_rows) + mt * 128 + q * 32;  // output row of lane 0
      const uint32_t thr = (EPI == EPI_FILTER && valid) ? desc_key(g.tau[row * g.tau_stride]) : 0u;
      const uint32_t tbase = tmem + acc * BN + part * (BN / 2) + ((uint32_t)(q * 32) << 16);
      uint32_t ra[32], rb_acc[32];
      // LNA kernels (more threads, fewer registers each) load one chunk at a
      // time; the others load the next chunk while the current one is stored
      constexpr bool kAhead = !LNA;
      tmem_ld32(tbase, ra);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        if (!kAhead && c > 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) ba[i] = kNoBias ? make_uint4(0, 0, 0, 0) : __ldg(bptr + c * 4 + i);
          tmem_ld32(tbase + c * 32, ra);
          tmem_ld_wait();
        }
        // the next chunk's accumulator and bias load while this chunk is stored
        if (kAhead && c + 1 < CH) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 bv = kNoBias ? make_uint4(0, 0, 0, 0) : __ldg(bptr + (c + 1) * 4 + i);
            if (c & 1) ba[i] = bv;
            else bb[i] = bv;
          }
          if (c & 1) tmem_ld32(tbase + (c + 1) * 32, ra);
          else tmem_ld32(tbase + (c + 1) * 32, rb_acc);
        }
        const uint8_t* rsm = nullptr;
        if (rtma) {
          if (!mbar_wait_warp(rb, rpar, ab, g.status)) {
            if (c + 1 < CH) tmem_ld_wait();
            return false;
          }
          rpar ^= 1;
          rsm = rbuf;
        }
        bool stored = false;
        if (EPI == EPI_FILTER) {
          if (c & 1) gemm_filter_chunk(g, row, valid, col0 + c * 32, rb_acc, thr);
          else gemm_filter_chunk(g, row, valid, col0 + c * 32, ra, thr);
        } else if (kAhead && (c & 1)) {
          stored = gemm_chunk<EPI>(g, &tmO16, &tmO32, row, valid, col0 + c * 32, y0, rb_acc, bb,
                                   stage, COMPACT ? -1 : (nchunk & 1), rsm);
        } else {
          stored = gemm_chunk<EPI>(g, &tmO16, &tmO32, row, valid, col0 + c * 32, y0, ra, ba,
                                   stage, COMPACT ? -1 : (nchunk & 1), rsm);
        }
        nchunk += stored ? 1 : 0;
        if (rtma) {
          __syncwarp();  // every lane has read the residual chunk
          if (lane == 0) {
            r_pending = false;
            int tn = t, cn = c + 1;
            if (cn == CH) {
              tn = t + (int)gridDim.x;
              cn = 0;
            }
            if (tn < tiles) {
              fence_proxy_async_smem();
              r_issue(tn, cn);
              r_pending = true;
            }
          }
        }
        if (kAhead && c + 1 < CH) tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
      return true;
    };

    for (int t = blockIdx.x; t < tiles; t += gridDim.x)
      if (!epi_tile(t)) break;
    if (lane == 0 && r_pending) {  // a residual load still in flight must land first
      AbortState tmp{0, kWaitLimitUs};
      mbar_wait(rb, rpar, &tmp, nullptr);
    }
    if (lane == 0) bulk_wait_all();  // every store has landed before the CTA exits
    __syncwarp();
  } else if (LNA) {
    // ------------------------------------------------ LNA: A = LayerNorm(O) * U
    // kLnaThreads / 32 warps turn the A tile of every K block into Z = ((O - mu) * rstd *
    // gamma + beta) * U, in place in shared memory, once TMA has brought the
    // tile of normalised O (in A's 128-byte swizzled K-major place) and the
    // matching U tile (same layout); the MMA thread waits for their arrivals
    // instead of TMA's.  O arrives normalised per (row, head): O = m + s * x,
    // so (O - mu) * rstd = a + b * x with each (row, head)'s coefficients
    // (a, b), computed before this launch (k_ln_coef) and fetched three K
    // blocks ahead of their use.  Thread tw takes the 16-byte chunk c = tw & 7
    // of rows (tw >> 3) + (kLnaThreads / 8) i, i < kLnaRows.  The transform runs in packed fp16
    // (two features per instruction): t = a + b x, z = (t gamma + beta) u,
    // each step rounded to fp16.
    const int tw = threadIdx.x - 64 - kEpiThreads;
    const int c = tw & 7;
    const int r0 = tw >> 3;
    const int K = g.K, H = g.ln_h;
    const int kb_head = g.ln_dv / 64;  // K blocks per head
    int stg = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int mt = (t % mn_tiles) / n_tiles, nt = (t % mn_tiles) % n_tiles;
      auto fetch_coef = [&](int kb_, uint32_t (&dst)[kLnaRows]) {
        const int head = min(kb_, KB - 1) / kb_head;
#pragma unroll
        for (int i = 0; i < kLnaRows; ++i) {
          const int64_t row = (int64_t)mt * 128 + r0 + (kLnaThreads / 8) * i;
          dst[i] = row < Mrows ? __ldg(g.ln_coef + row * H + head) : 0u;
        }
      };
      uint32_t cw0[kLnaRows], cw1[kLnaRows], cw2[kLnaRows];
      fetch_coef(0, cw0);
      fetch_coef(1, cw1);
      fetch_coef(2, cw2);
      uint4 gvn = __ldg(reinterpret_cast<const uint4*>(g.ln_gamma + c * 8));
      uint4 bvn = __ldg(reinterpret_cast<const uint4*>(g.ln_beta + c * 8));
      for (int kb = 0; kb < KB; ++kb) {
        const int col = kb * 64 + c * 8;
        __half2 gh[4], bh[4];
        {
          const uint32_t gw[4] = {gvn.x, gvn.y, gvn.z, gvn.w}, bw[4] = {bvn.x, bvn.y, bvn.z, bvn.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            gh[e] = __floats2half2_rn(bf16lo(gw[e]), bf16hi(gw[e]));
            bh[e] = __floats2half2_rn(bf16lo(bw[e]), bf16hi(bw[e]));
          }
        }
        uint32_t cw[kLnaRows];
#pragma unroll
        for (int i = 0; i < kLnaRows; ++i) {
          cw[i] = cw0[i];
          cw0[i] = cw1[i];
          cw1[i] = cw2[i];
        }
        fetch_coef(kb + 3, cw2);
        if (kb + 1 < KB) {
          gvn = __ldg(reinterpret_cast<const uint4*>(g.ln_gamma + col + 64));
          bvn = __ldg(reinterpret_cast<const uint4*>(g.ln_beta + col + 64));
        }
        // the normalised O and U of this stage have landed
        if (!mbar_wait_warp(full + stg, ph, ab, g.status)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + stg * C::STAGE_BYTES);
        const uint32_t su = sa + C::A_BYTES;
#pragma unroll
        for (int i = 0; i < kLnaRows; ++i) {
          const int r = r0 + (kLnaThreads / 8) * i;
          const uint32_t off = r * 128 + ((c ^ (r & 7)) << 4);
          uint4 xv = lds_u128(sa + off);
          const uint4 uv = lds_u128(su + off);
          const __half2 ab2 = *reinterpret_cast<const __half2*>(&cw[i]);
          const __half2 ca = __low2half2(ab2), cb = __high2half2(ab2);
          __half2* xh = reinterpret_cast<__half2*>(&xv);
          const __half2* uh = reinterpret_cast<const __half2*>(&uv);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            xh[e] = __hmul2(__hfma2(__hfma2(cb, xh[e], ca), gh[e], bh[e]), uh[e]);
          sts_u128(sa + off, xv);
          const int64_t row = (int64_t)mt * 128 + r;
          if (g.z_dbg && nt == 0 && row < Mrows)
            *reinterpret_cast<uint4*>(g.z_dbg + row * K + col) = xv;
        }
        fence_proxy_async_smem();  // the tensor cores read what these threads wrote
        __syncwarp();
        if (lane == 0) mbar_arrive(afull + stg);
        if (++stg == STAGES) {
          stg = 0;
          ph ^= 1;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int STAGES, int EPI, int COMPACT = 0, int LNA = 0, int MAJ = 0>
static cudaError_t launch_one(const CUtensorMap& ta, const CUtensorMap& tb,
                              const CUtensorMap& to16, const CUtensorMap& to32,
                              const CUtensorMap& tr, const GemmDev& gd, int grid, cudaStream_t s,
                              const CUtensorMap* tu_opt = nullptr) {
  const CUtensorMap& tu = tu_opt ? *tu_opt : ta;  // LNA only: the U tiles
  using C = GemmCfg<BN, STAGES, EPI, COMPACT, LNA>;
  static_assert(C::SMEM <= 232448, "shared memory per CTA");
  auto kfn = k_gemm_tc<BN, STAGES, EPI, COMPACT, LNA, MAJ>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM);
  if (e != cudaSuccess) return e;
  kfn<<<grid, C::THREADS, C::SMEM, s>>>(ta, tb, to16, to32, tr, tu, gd);
  return cudaGetLastError();
}

// ------------------------------------------------------------ CTA pairs
// The same product on clusters of two CTAs (one per SM) that share each
// 256 x 256 output tile through the pair MMA (cta_group::2): CTA r brings rows
// r*128.. of the A tile and W rows r*128.. of the tile's 256 into its own
// shared memory, so each CTA streams 32 KB per K block instead of the 48 KB a
// 128 x 256 tile of one CTA needs; rank 0 issues the MMAs (M = 256, N = 256),
// which leave each CTA's 128 output rows x 256 columns in its own tensor
// memory; both CTAs run the same epilogue warps on their half.
//   rank 0: counts both CTAs' bytes on its `full` barriers (the peer's loads
//           name them by cluster address); its MMA commits arrive on the
//           `empty` and `tfull` barriers of both CTAs (multicast commit);
//           both CTAs' epilogue warps arrive on rank 0's `tempty`.
// The plain-bias and SiLU epilogues (16-bit output, optionally the SiLU
// pre-activation) and the residual one with a 16-bit residual and output
// only (2 KB output and residual buffers per epilogue warp; each warp's next
// residual chunk arrives by TMA while the current one is finished);
// K-major operands.  Every wait is bounded; the two CTAs leave together
// through a bounded exchange of arrivals.
constexpr int kPairStages = 6;
template <int EPI>
struct PairCfg {
  static constexpr bool RES = EPI == EPI_RESID;
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;  // this CTA's 128 rows of A
  static constexpr uint32_t B_BYTES = 128 * 64 * 2;  // this CTA's 128 rows of W
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t BUF = RES ? 2048 : kStageBuf;  // per epilogue warp
  static constexpr uint32_t OUT_OFF = kPairStages * STAGE_BYTES;
  static constexpr uint32_t RES_OFF = OUT_OFF + (kEpiThreads / 32) * BUF;
  static constexpr uint32_t BAR_OFF = RES_OFF + (RES ? (kEpiThreads / 32) * 2048 : 0);
  static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
  static constexpr int THREADS = 64 + kEpiThreads;
};

template <int EPI>
__global__ void __launch_bounds__(PairCfg<EPI>::THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmO16,
                const __grid_constant__ CUtensorMap tmO32,
                const __grid_constant__ CUtensorMap tmR, const GemmDev g) {
  using C = PairCfg<EPI>;
  constexpr int S = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);  // [S], rank 0's in use
  uint64_t* empty = full + S;                                       // [S]
  uint64_t* tfull = empty + S;                                      // [2]
  uint64_t* tempty = tfull + 2;                                     // [2], rank 0's in use
  uint64_t* drain = tempty + 2;
  uint64_t* pdone = drain + 1;  // one arrival from each CTA at the end
  uint64_t* rbar = pdone + 1;   // [8] residual chunk landed (per epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 8);
  AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
  uint32_t* s_go = reinterpret_cast<uint32_t*>(ab + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  if (threadIdx.x == 0) {
    ab->flag = 0;
    ab->limit_us = kWaitLimitUs;
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(tfull + 0, 1);
    mbar_init(tfull + 1, 1);
    mbar_init(tempty + 0, 2 * (kEpiThreads / 32));
    mbar_init(tempty + 1, 2 * (kEpiThreads / 32));
    mbar_init(drain, 1);
    mbar_init(pdone, 2);
    for (int i = 0; i < 8; ++i) mbar_init(rbar + i, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised
  // rank 0 decides for the pair, so that both CTAs take the same path
  if (rank == 0 && threadIdx.x == 0) {
    const uint32_t go =
        ((g.status == nullptr) || (*reinterpret_cast<volatile int*>(g.status) == 0)) &&
        (g.run_if == nullptr || *reinterpret_cast<volatile const int*>(g.run_if) != 0);
    *s_go = go;
    st_cluster_u32(mapa_shared(smem_u32(s_go), 1), go);
  }
  cluster_sync_all();
  if (!*s_go) return;

  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int64_t Mrows = g.M_cap;
  if (g.M_dev) {
    const int64_t m = *g.M_dev;
    Mrows = m < Mrows ? m : Mrows;
  }
  if (Mrows < 0) Mrows = 0;
  const int n_tiles = g.N / 256;
  const int m_tiles = (int)((Mrows + 255) / 256);
  const int tiles = m_tiles * n_tiles;
  const int KB = g.K / 64;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
        const int mt = t / n_tiles, nt = t - (t / n_tiles) * n_tiles;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty + stage, ph ^ 1, ab, g.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(full + stage, 2 * C::STAGE_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(full + stage), 0);  // rank 0's barrier
          tma_load_2d_pair(sa, &tmA, kb * 64, mt * 256 + (int)rank * 128, fb);
          tma_load_2d_pair(sa + C::A_BYTES, &tmB, kb * 64, g.n_off + nt * 256 + (int)rank * 128,
                           fb);
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t IDESC = idesc_f16_f32(256, 256, 0, 0, g.ab_f16);
      int stage = 0, local = 0;
      uint32_t ph = 0;
      bool ok = true, issued_any = false;
      for (int t = pair; t < tiles && ok; t += npairs, ++local) {
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait_cluster(tempty + acc, aph ^ 1, ab, g.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * 256;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(full + stage, ph, ab, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16_ss_pair(d_tmem, sdesc_sw128(a0 + k * 32, 16, 1024),
                               sdesc_sw128(b0 + k * 32, 16, 1024), IDESC,
                               (kb != 0 || k != 0) ? 1u : 0u);
          tc_commit_pair(empty + stage, 0x3);
          issued_any = true;
          if (++stage == S) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (ok) tc_commit_pair(tfull + acc, 0x3);
      }
      if (issued_any) {
        tc_commit_pair(drain, 0x1);  // every MMA issued above has finished
        AbortState tmp{0, kWaitLimitUs};
        mbar_wait(drain, 0, &tmp, nullptr);
      }
    }
  } else {
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int part = (warp - 2) >> 2;  // which 128 of the 256 columns
    constexpr int CH = 4;              // 32-column chunks per warp
    uint8_t* stage = smem + C::OUT_OFF + (warp - 2) * C::BUF;
    int local = 0, nchunk = 0;
    // residual: lane 0 has TMA bring the next 32 x 32 chunk into the warp's
    // buffer while the current one is finished
    uint8_t* rbuf = smem + C::RES_OFF + (warp - 2) * 2048;
    uint64_t* rb = rbar + (warp - 2);
    uint32_t rpar = 0;
    bool r_pending = false;
    auto r_issue = [&](int t_, int c_) {
      const int mt_ = t_ / n_tiles, nt_ = t_ - (t_ / n_tiles) * n_tiles;
      mbar_arrive_expect_tx(rb, 2048u);
      tma_load_2d(rbuf, &tmR, g.n_off + nt_ * 256 + part * 128 + c_ * 32,
                  mt_ * 256 + (int)rank * 128 + q * 32, rb);
    };
    if (C::RES && lane == 0 && pair < tiles) {
      r_issue(pair, 0);
      r_pending = true;
    }
    bool alive = true;
    for (int t = pair; t < tiles && alive; t += npairs) {
      const int mt = t / n_tiles, nt = t - (t / n_tiles) * n_tiles;
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      ++local;
      const int col0 = g.n_off + nt * 256 + part * 128;
      const uint4* bptr = reinterpret_cast<const uint4*>(g.bias + col0);
      uint4 ba[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ba[i] = __ldg(bptr + i);
      if (!mbar_wait_warp(tfull + acc, aph, ab, g.status)) break;
      tc_fence_after();
      const int y0 = mt * 256 + (int)rank * 128 + q * 32;  // output row of lane 0
      const int64_t row = (int64_t)y0 + lane;
      const bool valid = row < Mrows;
      const uint32_t tbase = tmem + acc * 256 + part * 128 + ((uint32_t)(q * 32) << 16);
      uint32_t ra[32], rbv[32];
      tmem_ld32(tbase, ra);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        // the next chunk's accumulator and bias load while this one is stored
        if (c + 1 < CH) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 bv = __ldg(bptr + (c + 1) * 4 + i);
            if (c & 1) ba[i] = bv;
            else bb[i] = bv;
          }
          if (c & 1) tmem_ld32(tbase + (c + 1) * 32, ra);
          else tmem_ld32(tbase + (c + 1) * 32, rbv);
        }
        const uint8_t* rsm = nullptr;
        if (C::RES) {
          if (!mbar_wait_warp(rb, rpar, ab, g.status)) {
            if (c + 1 < CH) tmem_ld_wait();
            alive = false;
            break;
          }
          rpar ^= 1;
          rsm = rbuf;
        }
        bool stored;
        const int par = C::RES ? -1 : (nchunk & 1);
        if (c & 1)
          stored = gemm_chunk<EPI>(g, &tmO16, &tmO32, row, valid, col0 + c * 32, y0, rbv, bb,
                                   stage, par, rsm);
        else
          stored = gemm_chunk<EPI>(g, &tmO16, &tmO32, row, valid, col0 + c * 32, y0, ra, ba,
                                   stage, par, rsm);
        nchunk += stored ? 1 : 0;
        if (C::RES) {
          __syncwarp();  // every lane has read the residual chunk
          if (lane == 0) {
            r_pending = false;
            int tn = t, cn = c + 1;
            if (cn == CH) {
              tn = t + npairs;
              cn = 0;
            }
            if (tn < tiles) {
              fence_proxy_async_smem();
              r_issue(tn, cn);
              r_pending = true;
            }
          }
        }
        if (c + 1 < CH) tmem_ld_wait();
      }
      if (!alive) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(tempty + acc), 0));
    }
    if (lane == 0 && r_pending) {  // a residual load still in flight must land first
      AbortState tmp{0, kWaitLimitUs};
      mbar_wait(rb, rpar, &tmp, nullptr);
    }
    if (lane == 0) bulk_wait_all();  // every store has landed before the CTA exits
    __syncwarp();
  }
  // leave together: neither CTA exits while the other may still arrive on its
  // barriers or (rank 0's MMAs) read its shared memory
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive(pdone);
    mbar_arrive_cluster(mapa_shared(smem_u32(pdone), rank ^ 1u));
    AbortState tmp{0, 4 * kWaitLimitUs};
    mbar_wait(pdone, 0, &tmp, nullptr);
    // after a failed wait, loads already issued by either CTA may still be in
    // flight towards this CTA's shared memory: give them time to land
    if (g.status && *reinterpret_cast<volatile int*>(g.status) != 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 100000ull) __nanosleep(1000);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

template <int EPI>
static cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb,
                               const CUtensorMap& to16, const CUtensorMap& to32,
                               const CUtensorMap& tr, const GemmDev& gd, int pairs,
                               cudaStream_t s) {
  using C = PairCfg<EPI>;
  static_assert(C::SMEM <= 232448, "shared memory per CTA");
  auto kfn = k_gemm_pair<EPI>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kfn, ta, tb, to16, to32, tr, gd);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// How many CTA pairs of the pair kernel fit on the device at once (0 if the
// query fails): the persistent grid takes no more, so that no pair waits for
// another to finish.
template <int EPI>
static int pair_capacity() {
  static std::mutex mu;
  static std::map<int, int> cached;  // device -> clusters
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  const auto it = cached.find(dev);
  if (it != cached.end()) return it->second;
  using C = PairCfg<EPI>;
  auto kfn = k_gemm_pair<EPI>;
  int n = 0;
  if (ensure_smem_limit(reinterpret_cast<const void*>(kfn), C::SMEM) == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kfn), &cfg) !=
        cudaSuccess) {
      n = 0;
      (void)cudaGetLastError();  // the failed query's error, not a launch's
    }
  }
  cached[dev] = n;
  return n;
}

cudaError_t launch_gemm_tc(const GemmCall& c, cudaStream_t s, int kernel_id) {
  if (c.M_cap <= 0 || c.N <= 0) return cudaSuccess;
  if (c.N % 64 != 0 || c.K % 64 != 0) return cudaErrorInvalidValue;
  if (c.M_cap > (1ll << 31) - 256) return cudaErrorInvalidValue;
  const int sms = num_sms();
  const int64_t mt = (c.M_cap + 127) / 128;
  int BN = 64;
  if (c.N % 256 == 0 && mt * (c.N / 256) >= 2 * sms) BN = 256;
  else if (c.N % 128 == 0) BN = 128;
  CUtensorMap ta, tb, to16, to32, tr;
  const bool f16 = c.ab_f16 != 0;
  const bool lna = c.ln_x != nullptr;
  if (lna && (c.epi != EPI_RESID || !f16 || !c.ln_stats || !c.ln_coef || !c.ln_u || !c.ln_gamma ||
              !c.ln_beta || c.ln_h <= 0 || c.ln_dv % 64 != 0 || c.ln_h * c.ln_dv != c.K ||
              c.ld_u % 8 != 0))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tb, c.W, (uint64_t)(c.n_off + c.N), (uint64_t)c.K, (uint64_t)c.ldw * 2, 64,
                      (uint32_t)BN, f16))
    return cudaErrorInvalidValue;
  // LNA: A is the normalised O [M, K] (becomes Z in shared memory); U comes
  // from the first K columns of ln_u
  CUtensorMap tu;
  if (!encode_tmap_2d(&ta, lna ? c.ln_x : c.A, (uint64_t)c.M_cap, (uint64_t)c.K,
                      (uint64_t)(lna ? c.K : c.lda) * 2, 64, 128, f16))
    return cudaErrorInvalidValue;
  tu = ta;
  if (lna && !encode_tmap_2d(&tu, c.ln_u, (uint64_t)c.M_cap, (uint64_t)c.K, (uint64_t)c.ld_u * 2,
                             64, 128, true))
    return cudaErrorInvalidValue;
  // output maps over the whole [M_cap, ldo] matrix, 32 x 32 boxes; an unused
  // map is a copy of a valid one (never dereferenced)
  to16 = ta;
  to32 = ta;
  const CUtensorMapDataType t16 =
      c.out_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (c.out && !encode_tmap_2d_ex(&to16, c.out, (uint64_t)c.M_cap, (uint64_t)c.ldo,
                                  (uint64_t)c.ldo * 2, 32, 32, t16, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  if (c.out32 && !encode_tmap_2d_ex(&to32, c.out32, (uint64_t)c.M_cap, (uint64_t)c.ldo,
                                    (uint64_t)c.ldo * 4, 32, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // EPI_SILU's pre-activation output: a 16-bit matrix laid out like `out`
  if (c.out_pre && (c.epi != EPI_SILU || !c.out ||
                    !encode_tmap_2d_ex(&to32, c.out_pre, (uint64_t)c.M_cap, (uint64_t)c.ldo,
                                       (uint64_t)c.ldo * 2, 32, 32, t16,
                                       CU_TENSOR_MAP_SWIZZLE_64B)))
    return cudaErrorInvalidValue;
  // residual: [M_cap, n_off + N] with row stride ldr, 32 x 32 boxes (fp32 with
  // 128-byte swizzle, 16-bit with 64-byte swizzle)
  tr = ta;
  if (c.epi == EPI_RESID) {
    const bool r32 = c.resid_kind == RESID_F32;
    const CUtensorMapDataType rt = r32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : (c.resid_kind == RESID_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (!c.resid ||
        !encode_tmap_2d_ex(&tr, c.resid, (uint64_t)c.M_cap, (uint64_t)(c.n_off + c.N),
                           (uint64_t)c.ldr * (r32 ? 4 : 2), 32, 32, rt,
                           r32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  GemmDev gd{};  // value-initialised: optional fields (run_if, filter lists) stay null
  gd.M_cap = c.M_cap;
  gd.M_dev = c.M_dev;
  gd.N = c.N;
  gd.K = c.K;
  gd.n_off = c.n_off;
  gd.ab_f16 = c.ab_f16;
  gd.bias = static_cast<const __nv_bfloat16*>(c.bias);
  gd.has_out16 = c.out != nullptr;
  gd.out_f16 = c.out_f16;
  gd.has_out32 = (c.epi == EPI_RESID && c.out32 != nullptr);
  gd.resid = c.resid;
  gd.ldr = c.ldr;
  gd.resid_kind = c.resid_kind;
  gd.status = c.status;
  gd.ln_x = static_cast<const __half*>(c.ln_x);
  gd.ln_coef = c.ln_coef;
  gd.ln_u = static_cast<const __half*>(c.ln_u);
  gd.ld_u = c.ld_u;
  gd.ln_gamma = static_cast<const __nv_bfloat16*>(c.ln_gamma);
  gd.ln_beta = static_cast<const __nv_bfloat16*>(c.ln_beta);
  gd.ln_eps = c.ln_eps;
  gd.ln_h = c.ln_h;
  gd.ln_dv = c.ln_dv;
  gd.z_dbg = static_cast<__half*>(c.z_dbg);
  gd.splits = 1;
  gd.kb_split = (c.K + 63) / 64;
  gd.has_pre = c.out_pre != nullptr && c.epi == EPI_SILU;
  const int64_t tiles = mt * (c.N / BN);
  const int grid = (int)std::min<int64_t>(tiles, sms);
  if (lna) {  // each (row, head)'s LayerNorm coefficients first
    const cudaError_t e = launch_ln_coef(c.ln_stats, c.ln_h, c.ln_eps, c.ln_coef, c.M_cap, c.M_dev,
                                         c.status, s);
    if (e != cudaSuccess) return e;
  }
  // SiLU, plain-bias and (16-bit residual and output only) residual products
  // with 256-column tiles: CTA pairs
  const bool pair_res = c.epi == EPI_RESID && c.resid_kind != RESID_F32 && c.out32 == nullptr;
  if (!lna && (c.epi == EPI_SILU || c.epi == EPI_BIAS || pair_res) && BN == 256 &&
      gemm_pair_for(c.K)) {
    const int cap = c.epi == EPI_SILU   ? pair_capacity<EPI_SILU>()
                    : c.epi == EPI_BIAS ? pair_capacity<EPI_BIAS>()
                                        : pair_capacity<EPI_RESID>();
    if (cap > 0) {
      CUtensorMap tb2;  // W in 128-row boxes: each CTA of a pair brings half a tile
      if (!encode_tmap_2d(&tb2, c.W, (uint64_t)(c.n_off + c.N), (uint64_t)c.K,
                          (uint64_t)c.ldw * 2, 64, 128, f16))
        return cudaErrorInvalidValue;
      const int64_t ptiles = ((c.M_cap + 255) / 256) * (c.N / 256);
      const int pairs = (int)std::min<int64_t>(ptiles, cap);
      LaunchScope ls(kernel_id, s);
      if (c.epi == EPI_SILU) return launch_pair<EPI_SILU>(ta, tb2, to16, to32, tr, gd, pairs, s);
      if (c.epi == EPI_BIAS) return launch_pair<EPI_BIAS>(ta, tb2, to16, to32, tr, gd, pairs, s);
      return launch_pair<EPI_RESID>(ta, tb2, to16, to32, tr, gd, pairs, s);
    }
  }
  LaunchScope ls(kernel_id, s);
  if (c.epi == EPI_SILU) {
    if (BN == 256) return launch_one<256, 4, EPI_SILU>(ta, tb, to16, to32, tr, gd, grid, s);
    if (BN == 128) return launch_one<128, 6, EPI_SILU>(ta, tb, to16, to32, tr, gd, grid, s);
    return launch_one<64, 8, EPI_SILU>(ta, tb, to16, to32, tr, gd, grid, s);
  }
  if (c.epi == EPI_BIAS) {
    if (BN == 256) return launch_one<256, 4, EPI_BIAS>(ta, tb, to16, to32, tr, gd, grid, s);
    if (BN == 128) return launch_one<128, 6, EPI_BIAS>(ta, tb, to16, to32, tr, gd, grid, s);
    return launch_one<64, 8, EPI_BIAS>(ta, tb, to16, to32, tr, gd, grid, s);
  }
  if (lna) {  // f2 with LayerNorm * U formed in its A operand's shared memory
    if (BN == 256) {
      if (c.resid_kind != RESID_F32 && c.out32 == nullptr)
        return launch_one<256, 3, EPI_RESID, 1, 1>(ta, tb, to16, to32, tr, gd, grid, s, &tu);
      return launch_one<256, 2, EPI_RESID, 0, 1>(ta, tb, to16, to32, tr, gd, grid, s, &tu);
    }
    if (BN == 128) return launch_one<128, 3, EPI_RESID, 0, 1>(ta, tb, to16, to32, tr, gd, grid, s, &tu);
    return launch_one<64, 4, EPI_RESID, 0, 1>(ta, tb, to16, to32, tr, gd, grid, s, &tu);
  }
  // the residual buffers take one A/B stage's worth of shared memory
  if (BN == 256) {
    if (c.resid_kind != RESID_F32 && c.out32 == nullptr)
      return launch_one<256, 4, EPI_RESID, 1>(ta, tb, to16, to32, tr, gd, grid, s);
    return launch_one<256, 3, EPI_RESID>(ta, tb, to16, to32, tr, gd, grid, s);
  }
  if (BN == 128) return launch_one<128, 4, EPI_RESID>(ta, tb, to16, to32, tr, gd, grid, s);
  return launch_one<64, 6, EPI_RESID>(ta, tb, to16, to32, tr, gd, grid, s);
}

cudaError_t launch_gemm_scores(const void* A, int64_t lda, const void* W, int64_t ldw, int ab_f16,
                               int64_t M_cap, int64_t N, int K, float* out, int64_t ldo,
                               int* status, cudaStream_t s, int kernel_id, int64_t w_row_step,
                               const int* run_if) {
  if (M_cap <= 0 || N <= 0) return cudaSuccess;
  if (K % 64 != 0 || K <= 0 || ldo % 4 != 0 || ldo < N) return cudaErrorInvalidValue;
  if (M_cap > (1ll << 31) - 256 || N > (1ll << 31) - 256) return cudaErrorInvalidValue;
  constexpr int BN = 256;
  CUtensorMap ta, tb, to32;
  const bool f16 = ab_f16 != 0;
  if (!encode_tmap_2d(&ta, A, (uint64_t)M_cap, (uint64_t)K, (uint64_t)lda * 2, 64, 128, f16))
    return cudaErrorInvalidValue;
  // rows past N read as zeros; the output map's extent is N, so stores past
  // the last item are clipped.  w_row_step > 1 reads every w_row_step-th row
  // of W (a strided sample of the items) as the N rows.
  if (w_row_step < 1 ||
      !encode_tmap_2d(&tb, W, (uint64_t)N, (uint64_t)K, (uint64_t)(ldw * w_row_step) * 2, 64, BN,
                      f16))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d_ex(&to32, out, (uint64_t)M_cap, (uint64_t)N, (uint64_t)ldo * 4, 32, 32,
                         CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmDev gd{};
  gd.M_cap = M_cap;
  gd.M_dev = nullptr;
  gd.N = (int)N;
  gd.K = K;
  gd.n_off = 0;
  gd.ab_f16 = ab_f16;
  gd.bias = nullptr;
  gd.has_out16 = 0;
  gd.has_out32 = 1;
  gd.resid = nullptr;
  gd.status = status;
  gd.run_if = run_if;
  gd.splits = 1;
  gd.kb_split = K / 64;
  const int64_t tiles = ((M_cap + 127) / 128) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  LaunchScope ls(kernel_id, s);
  return launch_one<BN, 4, EPI_SCORE>(ta, tb, ta, to32, ta, gd, grid, s);
}

cudaError_t launch_gemm_filter(const void* A, int64_t lda, const void* W, int64_t ldw, int ab_f16,
                               int64_t M_cap, int64_t N, int K, const float* tau, int tau_stride,
                               uint32_t* cand_key, int32_t* cand_id, int* cnt, int cap,
                               int* overflow, int* status, cudaStream_t s, int kernel_id) {
  if (M_cap <= 0 || N <= 0) return cudaSuccess;
  if (K % 64 != 0 || K <= 0 || cap <= 0) return cudaErrorInvalidValue;
  if (M_cap > (1ll << 31) - 256 || N > (1ll << 31) - 256) return cudaErrorInvalidValue;
  constexpr int BN = 256;
  CUtensorMap ta, tb;
  const bool f16 = ab_f16 != 0;
  if (!encode_tmap_2d(&ta, A, (uint64_t)M_cap, (uint64_t)K, (uint64_t)lda * 2, 64, 128, f16))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tb, W, (uint64_t)N, (uint64_t)K, (uint64_t)ldw * 2, 64, BN, f16))
    return cudaErrorInvalidValue;
  GemmDev gd{};
  gd.M_cap = M_cap;
  gd.N = (int)N;
  gd.K = K;
  gd.ab_f16 = ab_f16;
  gd.status = status;
  gd.tau = tau;
  gd.tau_stride = tau_stride;
  gd.cand_key = cand_key;
  gd.cand_id = cand_id;
  gd.cand_cnt = cnt;
  gd.cand_cap = cap;
  gd.overflow = overflow;
  gd.splits = 1;
  gd.kb_split = K / 64;
  const int64_t tiles = ((M_cap + 127) / 128) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  LaunchScope ls(kernel_id, s);
  return launch_one<BN, 4, EPI_FILTER>(ta, tb, ta, ta, ta, gd, grid, s);
}

}  // namespace hstu

namespace hstu {

cudaError_t launch_gemm_grad(const GradGemm& c, cudaStream_t s, int kernel_id) {
  if (c.M <= 0 || c.N <= 0 || c.K <= 0) return cudaSuccess;
  if (c.M > (1ll << 31) - 256 || c.N > (1ll << 31) - 256 || c.K > (1ll << 31) - 256)
    return cudaErrorInvalidValue;
  if (c.splits < 1 || (c.resid && c.splits != 1) || c.ldo % 4 != 0) return cudaErrorInvalidValue;
  if (c.splits > 1 && c.split_rows < ((c.M + 127) / 128) * 128) return cudaErrorInvalidValue;
  if (!c.a_mn && c.K % 64 != 0) return cudaErrorInvalidValue;  // K-major A: whole 64-wide blocks
  if (!c.w_mn && c.K % 64 != 0) return cudaErrorInvalidValue;
  if (c.resid && (!c.zero_bias || c.N % 64 != 0)) return cudaErrorInvalidValue;
  constexpr int BN = 256;
  const bool f16 = c.ab_f16 != 0;
  CUtensorMap ta, tb, to32, to16, tr;
  // A: [M, K] (boxes 64 k x 128 m) or [K, M] (boxes 64 m x 64 k)
  if (c.a_mn ? !encode_tmap_2d(&ta, c.A, (uint64_t)c.K, (uint64_t)c.M, (uint64_t)c.lda * 2, 64,
                               64, f16)
             : !encode_tmap_2d(&ta, c.A, (uint64_t)c.M, (uint64_t)c.K, (uint64_t)c.lda * 2, 64,
                               128, f16))
    return cudaErrorInvalidValue;
  if (c.w_mn ? !encode_tmap_2d(&tb, c.W, (uint64_t)c.K, (uint64_t)c.N, (uint64_t)c.ldw * 2, 64,
                               64, f16)
             : !encode_tmap_2d(&tb, c.W, (uint64_t)c.N, (uint64_t)c.K, (uint64_t)c.ldw * 2, 64,
                               BN, f16))
    return cudaErrorInvalidValue;
  const int64_t rows_out = c.splits > 1 ? c.splits * c.split_rows : c.M;
  if (!encode_tmap_2d_ex(&to32, c.out, (uint64_t)rows_out, (uint64_t)c.N, (uint64_t)c.ldo * 4, 32,
                         32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  to16 = to32;
  tr = to32;
  if (c.resid) {
    if (!encode_tmap_2d_ex(&tr, c.resid, (uint64_t)c.M, (uint64_t)c.N, (uint64_t)c.ldo * 4, 32,
                           32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (c.out16 && !encode_tmap_2d_ex(&to16, c.out16, (uint64_t)c.M, (uint64_t)c.N,
                                      (uint64_t)c.ldo * 2, 32, 32,
                                      c.out16_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                      CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  const int KB = (int)((c.K + 63) / 64);
  const int splits = (int)std::min<int64_t>(c.splits, KB);
  const int kb_split = (KB + splits - 1) / splits;
  GemmDev gd{};
  gd.M_cap = c.M;
  gd.N = (int)c.N;
  gd.K = (int)c.K;
  gd.ab_f16 = c.ab_f16;
  gd.status = c.status;
  gd.splits = (KB + kb_split - 1) / kb_split;  // no empty split
  if (c.splits_used) *c.splits_used = gd.splits;
  gd.kb_split = kb_split;
  gd.split_rows = c.split_rows;
  const int64_t tiles = ((c.M + 127) / 128) * ((c.N + BN - 1) / BN) * gd.splits;
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  LaunchScope ls(kernel_id, s);
  if (c.resid) {  // out = resid + A W^T (+ a zero bias), fp32 and optionally 16-bit
    gd.bias = static_cast<const __nv_bfloat16*>(c.zero_bias);
    gd.has_out16 = c.out16 != nullptr;
    gd.out_f16 = c.out16_f16 ? 1 : 0;
    gd.has_out32 = 1;
    gd.resid = c.resid;
    gd.ldr = c.ldo;
    gd.resid_kind = RESID_F32;
    if (!c.a_mn && c.w_mn)
      return launch_one<256, 3, EPI_RESID, 0, 0, 2>(ta, tb, to16, to32, tr, gd, grid, s);
    return cudaErrorInvalidValue;
  }
  if (c.a_mn && c.w_mn) return launch_one<256, 4, EPI_SCORE, 0, 0, 3>(ta, tb, ta, to32, ta, gd, grid, s);
  if (c.w_mn) return launch_one<256, 4, EPI_SCORE, 0, 0, 2>(ta, tb, ta, to32, ta, gd, grid, s);
  if (c.a_mn) return launch_one<256, 4, EPI_SCORE, 0, 0, 1>(ta, tb, ta, to32, ta, gd, grid, s);
  return launch_one<256, 4, EPI_SCORE>(ta, tb, ta, to32, ta, gd, grid, s);
}

}  // namespace hstu

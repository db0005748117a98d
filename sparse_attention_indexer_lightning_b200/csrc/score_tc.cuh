// Lightning-indexer scoring on the sm_100a tensor cores: bf16 queries and
// keys, or (F8) fp8 e4m3 queries and keys.
//
// score(t, s) = sum_h w[t, h] * max(0, q[t, h] . k[s])   ("03 long context",
// section "The Architectural Answer: Read Less of the Past", stage 1; the
// GLM-shaped 32-head x 128-d form of "Latent Sparse Attention", "Where the
// time goes").
//
// Layout of the contraction (swap-AB): the MMA's M side is a tile of 128 keys
// (A, K-major, 128-byte swizzle, fed by TMA), the N side is QG queries x 32
// heads (B, K-major, TMA), K = d = 128 as 8 MMAs of K = 16.  The fp32
// accumulator lives in TMEM with one key per lane, so the epilogue thread that
// owns a key reads its 32 head sums with one tcgen05.ld and reduces the heads
// in registers: ReLU, multiply by w, add -- no shuffles.
//
// F8 (the indexer's FP8 GEMM, "03 long context" lecture, section "Sparsity
// Is a Systems Feature: The Blast Radius", kernel layer): A and B are e4m3
// codes, a 128-byte row per key or query head (one swizzle panel), K = 128
// as 4 kind::f8f6f4 MMAs of K = 32; the code products are exact and summed
// in fp32.  With non-negative scales the ReLU commutes with them: the host
// passes w * q_scale as the head weights and the epilogue multiplies each
// key's head sum by its scale.
//
// Roles (one persistent CTA per SM, contiguous runs of work units):
//   warp 0      TMA producer (keys every unit, the query tile on group change)
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2..   epilogue (4 warps for QG = 1, 16 for QG = 8: four per TMEM
//               lane quadrant, two of the group's 8 queries each)
// Pipelines: STAGES key buffers (full/empty mbarriers), BSLOTS query-tile slots,
// 2 TMEM accumulators so the epilogue of unit i overlaps the MMA of unit i+1.
// Every wait is bounded; a wait that runs out raises the library fault word
// and the CTA drains its copies and MMAs before it frees TMEM and exits.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

// F8: fp8 e4m3 queries and keys (kind::f8f6f4 MMAs, K = 32 each; a 128-byte
// row holds a whole key, so one swizzle panel); otherwise bf16 (two 64-wide
// panels per row, K = 16 per MMA).
template <int QG, bool FILTER = false, bool F8 = false>
struct TcCfg {
  static constexpr int BM = kTileKeys;             // keys per tile
  static constexpr int BN = QG * kHeads;           // queries x heads per MMA
  static constexpr int ESZ = F8 ? 1 : 2;           // bytes per element
  static constexpr int A_BYTES = BM * kDim * ESZ;  // 32 KB (bf16), 16 KB (fp8)
  static constexpr int A_HALF = BM * 128;          // one 128-byte swizzle panel of the tile
  static constexpr int B_BYTES = BN * kDim * ESZ;
  static constexpr int B_HALF = BN * 128;
  static constexpr int PANELS = kDim * ESZ / 128;  // 2 (bf16) or 1 (fp8)
  static constexpr int STAGES = (QG == 1) ? 6 : (F8 ? 4 : 3);
  // query-tile slots: 2 lets the next group's tile land during the current
  // group's last MMAs; 1 frees its space for key stages (the bf16 filter form,
  // whose candidate staging would otherwise leave room for 2 key stages: 3
  // stages and 1 slot measured faster)
  static constexpr int BSLOTS = (FILTER && !F8) ? 1 : 2;
  static constexpr int ACC = (QG == 1) ? 8 : 2;       // accumulator stages in TMEM
  static constexpr int ACC_COLS = BN < 32 ? 32 : BN;
  static constexpr int TMEM_COLS = (ACC * ACC_COLS <= 32) ? 32
                                   : (ACC * ACC_COLS <= 64) ? 64
                                   : (ACC * ACC_COLS <= 128) ? 128
                                   : (ACC * ACC_COLS <= 256) ? 256 : 512;
  // Epilogue warps come in sets of 4 (one per TMEM lane quadrant); the QG
  // queries of a group are split between the EPI_SETS warps of a quadrant.
  static constexpr int EPI_SETS = (QG == 1) ? 1 : 4;
  static constexpr int EPI_WARPS = 4 * EPI_SETS;
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr int Q_PER_EPI_WARP = (QG + EPI_SETS - 1) / EPI_SETS;
  static constexpr size_t SMEM_A = size_t(STAGES) * A_BYTES;
  static constexpr size_t SMEM_B = size_t(BSLOTS) * B_BYTES;
  static constexpr size_t SMEM_BAR = 512;
  static constexpr size_t SMEM_HIST = (QG == 1) ? kHistBins * 4 : 0;  // per-row selection histogram
  // filter form: each epilogue warp stages up to SBUF candidates per query
  static constexpr int SBUF = 64;
  static constexpr size_t SMEM_F = FILTER ? size_t(EPI_WARPS) * Q_PER_EPI_WARP * SBUF * 8 : 0;
  static constexpr size_t SMEM_BASE = 1024 /*align slack*/ + SMEM_A + SMEM_B + SMEM_BAR + SMEM_HIST + SMEM_F;
  // eight-query forms with room left: each epilogue warp keeps its queries'
  // head weights in shared memory (read per key tile from there instead of
  // through L1: fp8 scoring 912 -> 865 us per chunk)
  static constexpr size_t SMEM_W1 = size_t(EPI_WARPS) * Q_PER_EPI_WARP * kHeads * 4;
  static constexpr bool WSMEM = QG > 1 && SMEM_BASE + SMEM_W1 <= 232448;
  static constexpr size_t SMEM_W = WSMEM ? SMEM_W1 : 0;
  static constexpr size_t SMEM_TOTAL = SMEM_BASE + SMEM_W;
  static_assert(SMEM_TOTAL <= 232448, "shared memory budget");
  static_assert(ACC <= 8, "accumulator barriers");
};

struct TcBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t bfull[2];
  uint64_t bempty[2];
  uint64_t tfull[8];
  uint64_t tempty[8];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(TcBarriers) <= 512, "barrier block");

// Keys of the whole history query (b, t) may see: a precomputed count, or
// floor((q_pos + 1) / stride) capped at n_total (block-complete causal rule).
__device__ __forceinline__ int eligible_keys(const ScoreParams& p, int b, int t) {
  const int64_t row = static_cast<int64_t>(b) * p.T + t;
  if (p.lim_rows) return __ldg(p.lim_rows + row);
  const int64_t qp = __ldg(p.q_pos + row);
  int64_t e = qp < 0 ? 0 : (qp + 1) / p.stride;
  return static_cast<int>(e > p.n_total ? p.n_total : e);
}

// FILTER: the filter form of ScoreParams (p.out == nullptr), built as its own
// instantiation so the storing form keeps its registers.
template <int QG, bool FILTER, bool F8>
__global__ void __launch_bounds__(TcCfg<QG, FILTER, F8>::THREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                    const ScoreParams p) {
  using C = TcCfg<QG, FILTER, F8>;
  if (p.run_if != nullptr && *p.run_if == 0) return;  // a conditional launch with nothing to do
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::SMEM_A;
  TcBarriers* bars = reinterpret_cast<TcBarriers*>(smem + C::SMEM_A + C::SMEM_B);
  uint32_t* shist = reinterpret_cast<uint32_t*>(smem + C::SMEM_A + C::SMEM_B + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const bool use_hist = (QG == 1) && (p.hist != nullptr);
  if (use_hist)
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) shist[i] = 0;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int G = (p.T + QG - 1) / QG;
  const int NT = (p.N + C::BM - 1) / C::BM;
  const long long units = static_cast<long long>(p.B) * G * NT;
  const long long u_begin = units * blockIdx.x / gridDim.x;
  const long long u_end = units * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->bfull[s], 1);
      mbar_init(&bars->bempty[s], 1);
    }
    for (int s = 0; s < C::ACC; ++s) {
      mbar_init(&bars->tfull[s], 1);
      mbar_init(&bars->tempty[s], C::EPI_WARPS);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long prev_bg = -1;
      int bslot = C::BSLOTS - 1;
      uint32_t bphase[2] = {0, 0};
      int issued[8];
      uint32_t issued_par[8];
      for (int s = 0; s < 8; ++s) issued[s] = 0, issued_par[s] = 0;
      int b_issued[2] = {0, 0};
      uint32_t b_par[2] = {0, 0};
      bool ok = true;
      UnitPos up;
      up.init(u_begin, NT, G);
      for (long long u = u_begin; u < u_end && ok; ++u, up.next(NT, G)) {
        const int tile = up.tile, g = up.g, b = up.b;
        const long long bg = static_cast<long long>(b) * G + g;
        if (bg != prev_bg) {
          bslot = (bslot + 1 == C::BSLOTS) ? 0 : bslot + 1;
          if (!mbar_wait<false>(&bars->bempty[bslot], bphase[bslot] ^ 1, abort_flag)) { ok = false; break; }
          b_par[bslot] = bphase[bslot];
          b_issued[bslot] = 1;
          bphase[bslot] ^= 1;
          mbar_arrive_expect_tx(&bars->bfull[bslot], C::B_BYTES);
          const int qrow = (b * p.T + g * QG) * kHeads;
          uint8_t* dst = sB + bslot * C::B_BYTES;
          tma_load_2d(dst, &qmap, &bars->bfull[bslot], 0, qrow);
          if (C::PANELS == 2) tma_load_2d(dst + C::B_HALF, &qmap, &bars->bfull[bslot], 64, qrow);
          prev_bg = bg;
        }
        if (!mbar_wait<false>(&bars->empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->full[stage], C::A_BYTES);
        const int krow = b * p.N + tile * C::BM;
        uint8_t* dst = sA + stage * C::A_BYTES;
        tma_load_2d(dst, &kmap, &bars->full[stage], 0, krow);
        if (C::PANELS == 2) tma_load_2d(dst + C::A_HALF, &kmap, &bars->full[stage], 64, krow);
        issued[stage] = 1;
        issued_par[stage] = phase;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA goes away.
        for (int s = 0; s < C::STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&bars->full[s], issued_par[s]);
        for (int s = 0; s < 2; ++s)
          if (b_issued[s]) mbar_wait_drain(&bars->bfull[s], b_par[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop.  With one query per group (N = 32) the
    // MMAs are short and one elected lane of the converged warp issues them;
    // with eight (N = 256) the epilogue sets the pace and issuing from lane 0
    // alone measured faster.
    constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(C::BM, C::BN) : idesc_bf16_f32(C::BM, C::BN);
    constexpr bool ELECT = (QG == 1);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    long long prev_bg = -1;
    int bslot = C::BSLOTS - 1;
    uint32_t bphase[2] = {0, 0};
    const uint32_t a_base = smem_u32(sA);
    const uint32_t b_base = smem_u32(sB);
    UnitPos up;
    up.init(u_begin, NT, G);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, G)) {
      const long long bg = static_cast<long long>(up.b) * G + up.g;
      if (bg != prev_bg) {
        if (prev_bg >= 0) {
          if (ELECT) umma_commit_warp(&bars->bempty[bslot]);
          else if (lane == 0) umma_commit(&bars->bempty[bslot]);
        }
        bslot = (bslot + 1 == C::BSLOTS) ? 0 : bslot + 1;
        if (!warp_wait<false>(&bars->bfull[bslot], bphase[bslot], abort_flag)) break;
        bphase[bslot] ^= 1;
        prev_bg = bg;
      }
      if (!warp_wait<false>(&bars->tempty[acc], acc_phase ^ 1, abort_flag)) break;
      tc_fence_after();
      if (!warp_wait<false>(&bars->full[stage], phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t a_addr = a_base + stage * C::A_BYTES;
      const uint32_t b_addr = b_base + bslot * C::B_BYTES;
      const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
      // one MMA per 32 bytes of K: 16 bf16 or 32 e4m3 inside a 128-byte swizzle row
#pragma unroll
      for (int kk = 0; kk < 4 * C::PANELS; ++kk) {
        const uint32_t koff = (kk & 3) * 32;
        const uint64_t adesc = sw128_kmajor_desc(a_addr + (kk >> 2) * C::A_HALF + koff);
        const uint64_t bdesc = sw128_kmajor_desc(b_addr + (kk >> 2) * C::B_HALF + koff);
        if (F8) {
          if (lane == 0) umma_e4m3(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        } else if (ELECT) {
          umma_f16_warp(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        } else if (lane == 0) {
          umma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
      }
      if (ELECT) {
        umma_commit_warp(&bars->empty[stage]);
        umma_commit_warp(&bars->tfull[acc]);
      } else if (lane == 0) {
        umma_commit(&bars->empty[stage]);
        umma_commit(&bars->tfull[acc]);
      }
      __syncwarp();
      if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
    }
    // All MMAs the issuing lane started are complete once `drain` flips.
    if (ELECT) umma_commit_warp(&bars->drain);
    else if (lane == 0) umma_commit(&bars->drain);
    if (lane == 0) mbar_wait_drain(&bars->drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns the 32 keys of its TMEM lane quadrant and Q_PER_EPI_WARP
    // queries of the group.  One register buffer: a query's TMEM load, then
    // its reduction (a second buffer for overlapping the next load measured
    // slower: the registers it takes cost more than the overlap gives); the
    // accumulator is handed back to the MMA warp as soon as the unit's last
    // load has landed in registers.
    const int ew = warp - 2;                  // 0 .. EPI_WARPS-1
    const int quad = warp & 3;                // TMEM lane quadrant this warp may read
    const int qset = ew >> 2;                 // which share of the group's queries
    int acc = 0;
    uint32_t acc_phase = 0;
    HeadWeights wreg;                         // QG == 1: the group's one query's weights
    // Per-query data of the current group, derived once when the group changes
    // (consecutive units of a CTA walk the key tiles of one group):
    int limq[C::Q_PER_EPI_WARP];              // keys of this launch the query may see (<= N)
    float* orow[C::Q_PER_EPI_WARP];           // storing form: the query's row at this launch's key 0
    const float* wq[C::Q_PER_EPI_WARP];       // QG > 1: the query's head weights
    uint32_t thr[C::Q_PER_EPI_WARP];          // filter form: order code a key must reach
#pragma unroll
    for (int i = 0; i < C::Q_PER_EPI_WARP; ++i) limq[i] = 0, orow[i] = nullptr, wq[i] = nullptr, thr[i] = 0;
    constexpr bool filter = FILTER;
    // Filter form: each warp stages its queries' candidates in shared memory
    // and reserves global slots for a whole batch with one atomic.
    float* fbuf = reinterpret_cast<float*>(smem + C::SMEM_A + C::SMEM_B + C::SMEM_BAR + C::SMEM_HIST) +
                  static_cast<size_t>(ew) * C::Q_PER_EPI_WARP * C::SBUF * 2;
    float* wsh = reinterpret_cast<float*>(smem + C::SMEM_A + C::SMEM_B + C::SMEM_BAR + C::SMEM_HIST + C::SMEM_F) +
                 static_cast<size_t>(ew) * C::Q_PER_EPI_WARP * kHeads;   // WSMEM: this warp's queries' weights
    uint32_t fcnt[C::Q_PER_EPI_WARP];
    int64_t frow[C::Q_PER_EPI_WARP];
#pragma unroll
    for (int i = 0; i < C::Q_PER_EPI_WARP; ++i) fcnt[i] = 0, frow[i] = 0;
    auto flush_q = [&](int i) {                            // warp-uniform
      __syncwarp();
      uint32_t base = 0;
      if (lane == 0) base = atomicAdd(p.cand_cnt + frow[i], fcnt[i]);
      base = __shfl_sync(0xffffffffu, base, 0);
      const float* bv = fbuf + i * C::SBUF * 2;
      const int32_t* bl = reinterpret_cast<const int32_t*>(bv + C::SBUF);
      for (uint32_t e = lane; e < fcnt[i]; e += 32) {
        const uint32_t slot = base + e;
        if (slot < static_cast<uint32_t>(p.cand_cap)) {
          const int64_t at = frow[i] * p.ld_cand + slot;
          p.cand_val[at] = bv[e];
          p.cand_lab[at] = bl[e];
        } else {
          p.row_over[frow[i]] = 1;
          *p.any_over = 1;
        }
      }
      __syncwarp();
      fcnt[i] = 0;
    };
    auto flush_all = [&]() {
#pragma unroll
      for (int i = 0; i < C::Q_PER_EPI_WARP; ++i)
        if (fcnt[i]) flush_q(i);
    };
    UnitPos up;
    up.init(u_begin, NT, G);
    int nq = 0;                                            // queries of this warp in the current group
    int hb = 0;                                            // problem of the current group
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, G)) {
      const int tile = up.tile;
      const int n = tile * C::BM + quad * 32 + lane;       // key within this launch
      if (u == u_begin || tile == 0) {                     // units run (b, g, tile): a new group
        const int g = up.g, b = up.b;
        hb = b;
        if (filter) flush_all();                           // staged entries belong to the previous group
        // this warp's share of the QG columns blocks, cut by the group size
        // and by the last group's end
        nq = min(p.T - g * QG, QG) - qset * C::Q_PER_EPI_WARP;
        nq = nq < 0 ? 0 : (nq > C::Q_PER_EPI_WARP ? C::Q_PER_EPI_WARP : nq);
        int lim = p.N;
        if (p.n_valid) lim = min(lim, __ldg(p.n_valid + b));
        if (QG == 1) wreg.load(p.w + (static_cast<int64_t>(b) * p.T + g) * kHeads);
#pragma unroll
        for (int jq = 0; jq < C::Q_PER_EPI_WARP; ++jq) {
          if (jq < nq) {
            const int t = g * QG + qset * C::Q_PER_EPI_WARP + jq;
            const int64_t row = static_cast<int64_t>(b) * p.T + t;
            int lt = lim;
            if (p.lim_rows || p.q_pos) {
              // eligible keys of this query (whole history), relative to this launch
              const int rel = eligible_keys(p, b, t) - p.key_base;
              lt = rel < 0 ? 0 : (rel < lt ? rel : lt);
            }
            limq[jq] = lt;
            wq[jq] = p.w + row * kHeads;
            if (C::WSMEM) {                                // the group's weights, once per group
              __syncwarp();
              wsh[jq * kHeads + lane] = __ldg(wq[jq] + lane);
              __syncwarp();
              wq[jq] = wsh + jq * kHeads;
            }
            if (!filter) {
              orow[jq] = p.out + row * p.ld_out + p.out_col0;
            } else {
              // the row's threshold entry; a list with padding takes every eligible key
              const int64_t kth = row * p.ld_kth;
              thr[jq] = (p.kth_lab[kth] < 0) ? 0u : order_code(p.kth_val[kth]) + 1u;
              frow[jq] = row;
            }
          }
        }
      }
      float ks = 1.f;                                      // fp8: the key's scale, loaded ahead of the wait
      if (F8) ks = (n < p.N) ? __ldg(p.key_scale + static_cast<int64_t>(hb) * p.N + n) : 0.f;
      if (!warp_wait<false>(&bars->tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * C::ACC_COLS + qset * C::Q_PER_EPI_WARP * kHeads);
      uint32_t cur[32];
      if (nq == 0) {                                       // nothing to read: release now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->tempty[acc]);
      }
#pragma unroll
      for (int jq = 0; jq < C::Q_PER_EPI_WARP; ++jq) {
        if (jq < nq) {                                     // warp-uniform
          tmem_ld_32x32_nowait(tbase + static_cast<uint32_t>(jq * kHeads), cur);
          tmem_wait_ld(cur);
          if (jq + 1 == nq) {                              // the unit's last load is in: release
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[acc]);
          }
          float s;
          if (QG == 1) {
            s = head_reduce_w(cur, wreg);
          } else if (C::WSMEM) {
            HeadWeights hw;                                // from the warp's shared copy
            const ulonglong2* w2 = reinterpret_cast<const ulonglong2*>(wq[jq]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const ulonglong2 t2 = w2[i];
              hw.v[2 * i] = t2.x;
              hw.v[2 * i + 1] = t2.y;
            }
            s = head_reduce_w(cur, hw);
          } else {
            s = head_reduce(cur, wq[jq]);
          }
          if (F8) s *= ks;                                 // the key's scale (w holds w * q_scale)
          if (!filter) {
            if (n < p.N) {
              orow[jq][n] = (n < limq[jq]) ? s : neg_inf();
              if (use_hist && n < limq[jq]) atomicAdd(&shist[hist_bin(order_code(s))], 1u);
            }
          } else {
            const bool take = (n < limq[jq]) && order_code(s) >= thr[jq];
            const uint32_t bal = __ballot_sync(0xffffffffu, take);
            if (bal) {
              const uint32_t add = static_cast<uint32_t>(__popc(bal));
              if (fcnt[jq] + add > static_cast<uint32_t>(C::SBUF)) flush_q(jq);
              if (take) {
                const uint32_t off = fcnt[jq] + static_cast<uint32_t>(__popc(bal & ((1u << lane) - 1u)));
                float* bv = fbuf + jq * C::SBUF * 2;
                bv[off] = s;
                reinterpret_cast<int32_t*>(bv + C::SBUF)[off] = p.key_base + n;
              }
              fcnt[jq] += add;
            }
          }
        }
      }
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
      if (use_hist && (u + 1 == u_end || tile + 1 == NT)) {
        // the row (one query per sequence here) ends in this CTA: publish its counts
        role_barrier(1, C::EPI_WARPS * 32);
        flush_hist(shist, p.hist + static_cast<int64_t>(hb) * p.T * kHistBins, ew * 32 + lane, C::EPI_WARPS * 32);
        role_barrier(1, C::EPI_WARPS * 32);
      }
    }
    if (filter) flush_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int QG, bool FILTER, bool F8 = false>
static cudaError_t launch_tc(const CUtensorMap* kmap, const CUtensorMap* qmap, const ScoreParams& p, int num_sms,
                             cudaStream_t st) {
  using C = TcCfg<QG, FILTER, F8>;
  static std::atomic<uint64_t> attr_done{0};
  {
    const cudaError_t e = smem_limit_once(attr_done, reinterpret_cast<const void*>(&score_tc_kernel<QG, FILTER, F8>), C::SMEM_TOTAL);
    if (e != cudaSuccess) return e;
  }
  const int G = (p.T + QG - 1) / QG;
  const int NT = (p.N + C::BM - 1) / C::BM;
  const long long units = static_cast<long long>(p.B) * G * NT;
  if (units == 0) return cudaSuccess;
  const int grid = static_cast<int>(units < num_sms ? units : num_sms);
  score_tc_kernel<QG, FILTER, F8><<<grid, C::THREADS, C::SMEM_TOTAL, st>>>(*kmap, *qmap, p);
  return cudaGetLastError();
}

cudaError_t launch_score_tc(int qg, const CUtensorMap* kmap, const CUtensorMap* qmap, const ScoreParams& p,
                            int num_sms, cudaStream_t st) {
  const bool filter = p.out == nullptr;
  if (qg == 1) return filter ? launch_tc<1, true>(kmap, qmap, p, num_sms, st) : launch_tc<1, false>(kmap, qmap, p, num_sms, st);
  if (qg == 8) return filter ? launch_tc<8, true>(kmap, qmap, p, num_sms, st) : launch_tc<8, false>(kmap, qmap, p, num_sms, st);
  return cudaErrorInvalidValue;
}

// fp8 queries and keys, eight queries per group: p.w holds w * q_scale per
// (query, head) and p.key_scale the keys' scales.
cudaError_t launch_score_tc_f8(const CUtensorMap* kmap, const CUtensorMap* qmap, const ScoreParams& p, int num_sms,
                               cudaStream_t st) {
  const bool filter = p.out == nullptr;
  return filter ? launch_tc<8, true, true>(kmap, qmap, p, num_sms, st)
                : launch_tc<8, false, true>(kmap, qmap, p, num_sms, st);
}

}  // namespace lsi

// Indexer scoring of 8-bit keys with a per-key fp32 scale:
//   * int8 compact keys, scanned in order (the coarse pass of the two-stage
//     decode search, LeanSparse podcast transcript 07:12-07:34),
//   * fp8 e4m3 keys gathered by shortlist id (the exact re-rank, same
//     transcript 07:34-08:00; the 128 B key + 4 B scale entry of "03 long
//     context", "The Architectural Answer: Read Less of the Past").
//
//   score = sum_h w[h] * max(0, scale * (q[h] . code))
//
// One thread widens one key row to fp16 in registers (exact for both formats)
// and writes it to tensor memory with tcgen05.st; the MMA takes A (128 keys x
// 128) from tensor memory and B (the query's 32 heads, rescaled per head by a
// power of two and rounded to fp16, exact for every element within 2^28 of its
// head's largest) from shared memory, accumulating in fp32 with one key per
// TMEM lane.  The head weights carry the inverse powers of two, so the scores
// equal the bf16 formula.  Per 128 keys shared memory sees the 16 KB of raw
// rows written and read once and 8 KB of query-tile reads: the widened keys
// never pass through it.
//
// A unit is HALVES x 128 keys of one problem: 256 for contiguous keys (one
// pipeline hand-off per 32 KB; with 16 KB units the hand-offs alone held the
// stream to ~4.6 TB/s in a producer-only measurement, 32 KB units ran at
// ~6.1 TB/s), 128 for gathered rows.  Each 128-key half has its own TMEM lane
// block (A and D columns), so a unit is 2 x 8 MMAs.
//
// Roles (448 threads, one persistent CTA per SM):
//   warp 0      producer: raw rows (one 2-D TMA box with the 128-byte swizzle
//               when the keys are contiguous; one 128-byte bulk copy per row at
//               a 144-byte pitch when gathered), the rows' scales by cp.async
//               with their validity flags, and the query tile by TMA
//   warp 1      TMEM allocator; widens each new query tile to fp16 in place;
//               issues the MMAs through one elected lane
//   warps 2-9   two groups of four: thread = key row, 8-bit -> fp16 -> TMEM
//   warps 10-13 epilogue: scale, ReLU, head weights, head sum, store
// Both raw layouts make the row-per-thread 16-byte reads bank-conflict-free.
// All waits are bounded (see common.cuh).

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

template <int FMT, int HALVES>
struct Q8Cfg {
  static constexpr bool PQ = FMT == SRC_PQ;
  static constexpr int BM = kTileKeys;                  // keys per half (TMEM lanes)
  static constexpr int KPU = HALVES * BM;               // keys per unit
  static constexpr int BN = kHeads;                     // one query per problem
  static constexpr int ROW = PQ ? kPqSub : kDim;        // bytes per key row (8-bit codes / PQ codes)
  // gathered rows (HALVES == 1) land at a 144-byte pitch, contiguous ones as
  // 128-byte rows under the TMA's 128-byte swizzle (PQ: 32-byte rows, no
  // swizzle)
  static constexpr int PITCH = (HALVES == 1) ? ROW + 16 : ROW;
  static constexpr int RAW_BYTES = KPU * PITCH;         // 1024-multiple
  static constexpr int RS = (HALVES == 1 || PQ) ? 8 : 6;  // raw stages
  static constexpr int AS = 6 / HALVES;                 // widened stages in TMEM
  static constexpr int ACC = 4 / HALVES;                // accumulator stages in TMEM
  static constexpr int A_COLS = HALVES * (kDim / 2);    // two fp16 per 32-bit column
  static constexpr int D_COLS = HALVES * BN;
  static constexpr int A_COL0 = ACC * D_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SS = (HALVES == 1) ? 32 : 8;     // scale stages (the producer's lead over the epilogue)
  static constexpr int CVT_WARPS = 8;
  static constexpr int CVT_GROUPS = 2;
  static constexpr int CVT_GROUP_WARPS = CVT_WARPS / CVT_GROUPS;
  static constexpr int EPI_WARPS = 4;
  static constexpr int THREADS = (2 + CVT_WARPS + EPI_WARPS) * 32;
  static constexpr int B_BYTES = BN * kDim * 2;
  static constexpr int B_HALF = BN * 64 * 2;
  static constexpr size_t SMEM_RAW = size_t(RS) * RAW_BYTES;
  static constexpr size_t SMEM_B = size_t(2) * B_BYTES;
  static constexpr size_t S_BYTES = size_t(KPU) * 8;    // per key: fp32 scale + int flag
  static constexpr size_t SMEM_S = size_t(SS) * S_BYTES;
  static constexpr size_t SMEM_BAR = 1024;
  static constexpr size_t SMEM_CB = PQ ? size_t(kPqSub) * 256 * 8 : 0;  // PQ codebooks, fp16 [32][256][4]
  static constexpr size_t SMEM_TOTAL = 1024 + SMEM_RAW + SMEM_B + SMEM_S + SMEM_BAR + SMEM_CB;
  static_assert(HALVES == 1 || HALVES == 2, "128- or 256-key units");
  static_assert(RAW_BYTES % 1024 == 0, "swizzled stages need 1024-byte alignment");
  static_assert(A_COL0 + AS * A_COLS <= TMEM_COLS, "TMEM columns");
  static_assert(CVT_GROUP_WARPS == 4 && EPI_WARPS == 4, "one warp per TMEM lane quadrant");
  static_assert(RS <= 8 && AS <= 6 && ACC <= 4 && SS <= 32, "barrier arrays");
  static_assert(SMEM_TOTAL <= 232448, "shared memory budget");
};

struct Q8Barriers {
  uint64_t rfull[8];
  uint64_t rempty[8];
  uint64_t afull[6];
  uint64_t aempty[6];
  uint64_t bfull[2];
  uint64_t bempty[2];
  uint64_t tfull[4];
  uint64_t tempty[4];
  uint64_t sfull[32];
  uint64_t sempty[32];
  uint64_t drain;
  uint64_t cbfull;  // PQ codebooks landed
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Q8Barriers) <= 1024, "barrier block");

// Drain wait: bounded by time only (used after an abort and at the end).
__device__ __forceinline__ void q8_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > LSI_WAIT_LIMIT_NS) {
      atomicOr(&g_fault, FAULT_WAIT_TIMEOUT);
      return;
    }
  }
}

// 16 8-bit codes (one 16-byte chunk, element 0 in the low byte) -> 8 words of
// fp16 pairs, element 2w in the low half of word w.
template <int FMT>
__device__ __forceinline__ void widen16(const uint4& v, uint32_t* o) {
  if (FMT == SRC_INT8 || FMT == SRC_PQ) {
    i8x4_to_f16x4(v.x, o[0], o[1]);
    i8x4_to_f16x4(v.y, o[2], o[3]);
    i8x4_to_f16x4(v.z, o[4], o[5]);
    i8x4_to_f16x4(v.w, o[6], o[7]);
  } else {
    e4m3x4_to_f16x4(v.x, o[0], o[1]);
    e4m3x4_to_f16x4(v.y, o[2], o[3]);
    e4m3x4_to_f16x4(v.z, o[4], o[5]);
    e4m3x4_to_f16x4(v.w, o[6], o[7]);
  }
}

template <int FMT, int HALVES>
__global__ void __launch_bounds__(Q8Cfg<FMT, HALVES>::THREADS, 1)
    score_q8_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                    const CvtParams p) {
  using C = Q8Cfg<FMT, HALVES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sR = smem;
  uint8_t* sB = sR + C::SMEM_RAW;
  uint8_t* sS = sB + C::SMEM_B;
  Q8Barriers* bars = reinterpret_cast<Q8Barriers*>(sS + C::SMEM_S);
  uint8_t* sCB = sS + C::SMEM_S + C::SMEM_BAR;  // PQ codebooks
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NT = (p.N + C::KPU - 1) / C::KPU;
  const long long units = static_cast<long long>(p.B) * NT;
  const long long u_begin = units * blockIdx.x / gridDim.x;
  const long long u_end = units * (blockIdx.x + 1) / gridDim.x;
  const bool gathered = (HALVES == 1) && p.rows != nullptr;  // the launcher sends gathers to HALVES == 1

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::RS; ++s) {
      mbar_init(&bars->rfull[s], 1);
      mbar_init(&bars->rempty[s], C::CVT_GROUP_WARPS);
    }
    for (int s = 0; s < C::AS; ++s) {
      mbar_init(&bars->afull[s], C::CVT_GROUP_WARPS);
      mbar_init(&bars->aempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->bfull[s], 1);
      mbar_init(&bars->bempty[s], 1);
    }
    for (int s = 0; s < C::ACC; ++s) {
      mbar_init(&bars->tfull[s], 1);
      mbar_init(&bars->tempty[s], C::EPI_WARPS);
    }
    for (int s = 0; s < C::SS; ++s) {
      mbar_init(&bars->sfull[s], 32);  // every producer lane arrives (plus its cp.async arrivals)
      mbar_init(&bars->sempty[s], C::EPI_WARPS);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->cbfull, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&qmap);
    if (!gathered) tma_prefetch_desc(&kmap);
  }
  if (C::PQ && threadIdx.x == 0) {  // barrier init by this same thread above; the codebooks once per CTA
    mbar_arrive_expect_tx(&bars->cbfull, static_cast<uint32_t>(C::SMEM_CB));
    bulk_load(sCB, p.books, static_cast<uint32_t>(C::SMEM_CB), &bars->cbfull);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint8_t* keys = static_cast<const uint8_t*>(p.keys);
    int rs = 0, ss = 0;
    uint32_t rphase = 0, sphase = 0;
    int prev_b = -1;
    int bslot = 1;
    uint32_t bphase[2] = {0, 0};
    int issued[C::RS];
    uint32_t issued_par[C::RS];
#pragma unroll
    for (int s = 0; s < C::RS; ++s) issued[s] = 0, issued_par[s] = 0;
    int b_issued[2] = {0, 0};
    uint32_t b_par[2] = {0, 0};
    bool ok = true;
    int nvb = p.N;  // valid keys of the current problem (contiguous keys)
    auto load_rids = [&](int tb, int ttile, int32_t (&out)[4]) {
      const int jb = ttile * C::BM;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = jb + lane + 32 * i;
        out[i] = (j < p.N) ? __ldg(p.rows + static_cast<int64_t>(tb) * p.N + j) : -1;
      }
    };
    int32_t rid_next[4] = {-1, -1, -1, -1};
    UnitPos up;
    up.init(u_begin, NT, 1);
    if (gathered && u_begin < u_end) load_rids(up.b, up.tile, rid_next);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, 1)) {
      const int tile = up.tile;
      const int b = up.b;
      if (b != prev_b) {
        bslot ^= 1;
        if (!warp_wait(&bars->bempty[bslot], bphase[bslot] ^ 1, abort_flag)) { ok = false; break; }
        b_par[bslot] = bphase[bslot];
        b_issued[bslot] = 1;
        bphase[bslot] ^= 1;
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars->bfull[bslot], C::B_BYTES);
          const int qrow = static_cast<int>(static_cast<int64_t>(b) * p.q_row_stride);
          uint8_t* dst = sB + bslot * C::B_BYTES;
          tma_load_2d(dst, &qmap, &bars->bfull[bslot], 0, qrow);
          tma_load_2d(dst + C::B_HALF, &qmap, &bars->bfull[bslot], 64, qrow);
        }
        nvb = p.N;
        if (!gathered && p.n_valid) nvb = min(nvb, __ldg(p.n_valid + b));
        prev_b = b;
      }
      if (!warp_wait(&bars->rempty[rs], rphase ^ 1, abort_flag)) { ok = false; break; }
      if (!warp_wait(&bars->sempty[ss], sphase ^ 1, abort_flag)) { ok = false; break; }
      uint8_t* dst = sR + rs * C::RAW_BYTES;
      float* ssc = reinterpret_cast<float*>(sS + ss * C::S_BYTES);
      int* sok = reinterpret_cast<int*>(ssc + C::KPU);
      const int j0 = tile * C::KPU;
      if (!gathered) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars->rfull[rs], C::KPU * C::ROW);
#pragma unroll
          for (int h = 0; h < HALVES; ++h)
            tma_load_2d(dst + h * C::BM * C::ROW, &kmap, &bars->rfull[rs], 0, b * p.N + j0 + h * C::BM);
        }
#pragma unroll
        for (int i = 0; i < 4 * HALVES; ++i) {
          const int r = lane + 32 * i;
          const bool valid = j0 + r < nvb;
          sok[r] = valid ? 1 : 0;
          if (C::PQ) ssc[r] = 1.f;  // PQ keys carry no scale
          else if (valid) cp_async_4(ssc + r, p.scale + static_cast<int64_t>(b) * p.N + j0 + r);
        }
      } else {
        // lane l holds the row ids of rows l, l+32, l+64, l+96 (the next
        // unit's are read now, so their latency overlaps this unit's copies);
        // the rows move as 16-byte cp.async chunks, eight lanes per row, so a
        // warp instruction copies four whole rows
        int32_t rid[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) rid[i] = rid_next[i];
        if (u + 1 < u_end) {
          if (tile + 1 == NT) load_rids(b + 1, 0, rid_next);
          else load_rids(b, tile + 1, rid_next);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (rid[i] >= p.key_rows) {
            atomicOr(&g_fault, FAULT_BAD_INDEX);
            rid[i] = -1;
          }
        }
        const int chunk = lane & 7, sub = lane >> 3;
#pragma unroll
        for (int it = 0; it < C::BM / 4; ++it) {
          const int r = it * 4 + sub;
          const int32_t rr = __shfl_sync(0xffffffffu, rid[it >> 3], r & 31);
          if (rr >= 0)
            cp_async_16(dst + r * C::PITCH + chunk * 16,
                        keys + (static_cast<int64_t>(b) * p.key_stride + rr) * C::ROW + chunk * 16);
        }
        cp_async_mbar_arrive(&bars->rfull[rs]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->rfull[rs]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          sok[r] = rid[i] >= 0 ? 1 : 0;
          if (rid[i] >= 0) cp_async_4(ssc + r, p.scale + static_cast<int64_t>(b) * p.key_stride + rid[i]);
        }
      }
      cp_async_mbar_arrive(&bars->sfull[ss]);
      mbar_arrive(&bars->sfull[ss]);
      issued[rs] = 1;
      issued_par[rs] = rphase;
      if (++rs == C::RS) { rs = 0; rphase ^= 1; }
      if (++ss == C::SS) { ss = 0; sphase ^= 1; }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok && lane == 0) {
      for (int s = 0; s < C::RS; ++s)
        if (issued[s]) q8_wait_drain(&bars->rfull[s], issued_par[s]);
      for (int s = 0; s < 2; ++s)
        if (b_issued[s]) q8_wait_drain(&bars->bfull[s], b_par[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_f16_f32(C::BM, C::BN);
    int as = 0, acc = 0;
    uint32_t aphase = 0, acc_phase = 0;
    int prev_b = -1;
    int bslot = 1;
    uint32_t bphase[2] = {0, 0};
    const uint32_t b_base = smem_u32(sB);
    UnitPos up;
    up.init(u_begin, NT, 1);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, 1)) {
      const int b = up.b;
      if (b != prev_b) {
        if (prev_b >= 0) umma_commit_warp(&bars->bempty[bslot]);
        bslot ^= 1;
        // every lane observes the barrier itself: all of them read the tile next
        const bool okb = mbar_wait(&bars->bfull[bslot], bphase[bslot], abort_flag);
        if (!__all_sync(0xffffffffu, okb)) break;
        bphase[bslot] ^= 1;
        prev_b = b;
        q_tile_to_f16(sB + bslot * C::B_BYTES, C::B_HALF, lane);
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (!warp_wait(&bars->tempty[acc], acc_phase ^ 1, abort_flag)) break;
      tc_fence_after();
      if (!warp_wait(&bars->afull[as], aphase, abort_flag)) break;
      tc_fence_after();
      const uint32_t b_addr = b_base + bslot * C::B_BYTES;
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        const uint32_t d_tmem = tmem_base + acc * C::D_COLS + h * C::BN;
        const uint32_t a_tmem = tmem_base + C::A_COL0 + as * C::A_COLS + h * (kDim / 2);
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint64_t bdesc = sw128_kmajor_desc(b_addr + (kk >> 2) * C::B_HALF + (kk & 3) * 32);
          umma_f16_tmem_a_warp(d_tmem, a_tmem + kk * 8, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
      }
      umma_commit_warp(&bars->aempty[as]);
      umma_commit_warp(&bars->tfull[acc]);
      if (++as == C::AS) { as = 0; aphase ^= 1; }
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
    }
    umma_commit_warp(&bars->drain);
    if (lane == 0) q8_wait_drain(&bars->drain, 0);
    __syncwarp();
  } else if (warp < 2 + C::CVT_WARPS) {
    // ------------------------------------------------------------ widening
    // Group cg takes units cg, cg + 2, ...; warp w of the group owns TMEM lane
    // quadrant w & 3, and its thread `lane` owns key row 32 * (w & 3) + lane.
    const int cg = (warp - 2) / C::CVT_GROUP_WARPS;
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + C::A_COL0;
    const long long count = u_end - u_begin;
    bool cb_ok = true;
    if (C::PQ) cb_ok = warp_wait(&bars->cbfull, 0, abort_flag);
    for (long long i = cg; i < count && cb_ok; i += C::CVT_GROUPS) {
      const int rs = static_cast<int>(i % C::RS), as = static_cast<int>(i % C::AS);
      const uint32_t rphase = static_cast<uint32_t>((i / C::RS) & 1), aphase = static_cast<uint32_t>((i / C::AS) & 1);
      if (!warp_wait(&bars->rfull[rs], rphase, abort_flag)) break;
      if (!warp_wait(&bars->aempty[as], aphase ^ 1, abort_flag)) break;
      tc_fence_after();
      const uint8_t* raw = sR + rs * C::RAW_BYTES;
      // contiguous: 128-byte rows, 16-byte chunk c stored at c ^ (row & 7);
      // gathered: 144-byte pitch, chunks in order
      const int sw = gathered ? 0 : (row & 7);
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        const uint8_t* rowp = raw + (h * C::BM + row) * C::PITCH;
        if (C::PQ) {
          // 32 codes; sub-vector m is row code[m] of codebook m (4 fp16 = 8 bytes)
          const uint2* cb = reinterpret_cast<const uint2*>(sCB);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint4 cw = *reinterpret_cast<const uint4*>(rowp + part * 16);
            const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t code = (w4[c >> 2] >> (8 * (c & 3))) & 0xffu;
              const uint2 e = cb[(part * 16 + c) * 256 + code];
              o[2 * c] = e.x;
              o[2 * c + 1] = e.y;
            }
            tmem_st_32x32(t_row + as * C::A_COLS + h * (kDim / 2) + part * 32, o);
          }
        } else {
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            uint4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = *reinterpret_cast<const uint4*>(rowp + (((part * 4 + c) ^ sw) << 4));
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) widen16<FMT>(v[c], o + 8 * c);
            tmem_st_32x32(t_row + as * C::A_COLS + h * (kDim / 2) + part * 32, o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->rempty[rs]);
        mbar_arrive(&bars->afull[as]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int acc = 0, ss = 0;
    uint32_t acc_phase = 0, sphase = 0;
    int w_b = -1;
    HeadWeights wreg;
    UnitPos up;
    up.init(u_begin, NT, 1);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, 1)) {
      const int tile = up.tile;
      const int b = up.b;
      if (w_b != b) {
        // lane h: head h's weight times 2^-s_h, the inverse of the query tile's shift
        const uint16_t* qrow = p.q + (static_cast<int64_t>(b) * p.q_row_stride + lane) * kDim;
        const float wl = __ldg(p.w + static_cast<int64_t>(b) * kHeads + lane) * exp2i(-q_head_shift_global(qrow));
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wreg.v[i] = pack_f32x2(__shfl_sync(0xffffffffu, wl, 2 * i), __shfl_sync(0xffffffffu, wl, 2 * i + 1));
        w_b = b;
      }
      if (!warp_wait(&bars->sfull[ss], sphase, abort_flag)) break;
      const float* ssc = reinterpret_cast<const float*>(sS + ss * C::S_BYTES);
      float sc[HALVES];
      int valid[HALVES];
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        sc[h] = ssc[h * C::BM + row];
        valid[h] = reinterpret_cast<const int*>(ssc + C::KPU)[h * C::BM + row];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->sempty[ss]);
      if (++ss == C::SS) { ss = 0; sphase ^= 1; }
      if (!warp_wait(&bars->tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_d = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * C::D_COLS);
      uint32_t v0[32], v1[32];
      tmem_ld_32x32_nowait(t_d, v0);
      if (HALVES == 2) tmem_ld_32x32_nowait(t_d + C::BN, v1);
      tmem_wait_ld(v0);
      if (HALVES == 2) tmem_wait_ld(v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tempty[acc]);
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        const int j = tile * C::KPU + h * C::BM + row;
        if (j < p.N) {
          float s = neg_inf();
          if (valid[h]) {
            s = head_reduce_scaled(h == 0 ? v0 : v1, wreg, sc[h]);
            if (p.hist) atomicAdd(p.hist + static_cast<int64_t>(b) * kHistBins + hist_bin(order_code(s)), 1u);
          }
          p.out[static_cast<int64_t>(b) * p.N + j] = s;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int FMT, int HALVES>
static cudaError_t launch_q8(const CUtensorMap* qmap, const CUtensorMap* kmap, const CvtParams& p, int num_sms,
                             cudaStream_t st) {
  using C = Q8Cfg<FMT, HALVES>;
  static std::atomic<uint64_t> attr_done{0};
  {
    const cudaError_t e = smem_limit_once(attr_done, reinterpret_cast<const void*>(&score_q8_kernel<FMT, HALVES>), C::SMEM_TOTAL);
    if (e != cudaSuccess) return e;
  }
  const int NT = (p.N + C::KPU - 1) / C::KPU;
  const long long units = static_cast<long long>(p.B) * NT;
  if (units == 0) return cudaSuccess;
  const int grid = static_cast<int>(units < num_sms ? units : num_sms);
  score_q8_kernel<FMT, HALVES><<<grid, C::THREADS, C::SMEM_TOTAL, st>>>(*qmap, *kmap, p);
  return cudaGetLastError();
}

// Contiguous keys take 256-key units, gathered rows 128-key units.
cudaError_t launch_score_q8(const CUtensorMap* qmap, const CUtensorMap* kmap, const CvtParams& p, int num_sms,
                            cudaStream_t st) {
  const bool gathered = p.rows != nullptr;
  switch (p.fmt) {
    case SRC_INT8:
      return gathered ? launch_q8<SRC_INT8, 1>(qmap, kmap, p, num_sms, st)
                      : launch_q8<SRC_INT8, 2>(qmap, kmap, p, num_sms, st);
    case SRC_E4M3:
      return gathered ? launch_q8<SRC_E4M3, 1>(qmap, kmap, p, num_sms, st)
                      : launch_q8<SRC_E4M3, 2>(qmap, kmap, p, num_sms, st);
    case SRC_PQ:  // contiguous only
      return gathered ? cudaErrorInvalidValue : launch_q8<SRC_PQ, 2>(qmap, kmap, p, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lsi

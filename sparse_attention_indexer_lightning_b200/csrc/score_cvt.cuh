// Indexer scoring of keys that need converting before the tensor cores:
//   * int8 compact keys with a per-key fp32 scale (the coarse pass of the
//     two-stage decode search, LeanSparse podcast transcript 07:12-07:34),
//   * fp8 e4m3 keys with a per-key fp32 scale, gathered by shortlist id (the
//     exact re-rank, same transcript 07:34-08:00; the 128 B key + 4 B scale
//     entry of "03 long context", "The Architectural Answer: Read Less of the
//     Past"),
//   * bf16 keys gathered by position (the exact rescore after bucket
//     expansion, "Latent Sparse Attention", "The method, term by term").
//
//   score = sum_h w[h] * max(0, scale * (q[h] . code))
//
// Both 8-bit formats widen to fp16 exactly (int8 magnitudes <= 128; e4m3 is a
// subset of fp16), and the query tile is rescaled per head by a power of two
// (largest |q| into [2^14, 2^15)) and rounded to fp16 in shared memory, which
// is exact for every element within 2^28 of its head's largest; the head
// weights get the inverse power of two, so the contraction runs as an
// f16 x f16 -> fp32 tcgen05 MMA with one key per TMEM lane and the scores
// equal the bf16 formula.  Gathered bf16 keys use a bf16 x bf16 MMA.
//
// Roles (448 threads, one persistent CTA per SM):
//   warp 0      producer: 1-D bulk copies of raw rows (one copy per tile when
//               contiguous, one per row when gathered) + TMA of the query tile
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2-9   converters: raw rows -> bf16 in the 128-byte-swizzled K-major
//               layout the MMA descriptor expects
//   warps 10-13 epilogue: scale, ReLU, head weights, head sum, store (the next
//               unit's row ids and scales are loaded one unit ahead)
// All waits are bounded (see common.cuh).

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

template <int FMT>
struct CvtCfg {
  static constexpr int BM = kTileKeys;
  static constexpr int BN = kHeads;                       // one query per problem
  static constexpr int ROW_BYTES = (FMT == SRC_BF16) ? 256 : 128;
  static constexpr int RAW_BYTES = BM * ROW_BYTES;
  static constexpr int A_BYTES = BM * kDim * 2;
  static constexpr int A_HALF = BM * 64 * 2;
  static constexpr int B_BYTES = BN * kDim * 2;
  static constexpr int B_HALF = BN * 64 * 2;
  static constexpr int RS = (FMT == SRC_BF16) ? 3 : 6;   // raw stages
  static constexpr int AS = 3;                            // converted stages
  static constexpr int ACC = 8;  // accumulator stages in TMEM (32 columns each)
  static constexpr int TMEM_COLS = ACC * BN;
  static_assert(ACC <= 8 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation");
  static constexpr int CVT_WARPS = 8;
  static constexpr int CVT_GROUPS = 2;                       // tiles converted at once
  static constexpr int CVT_GROUP_WARPS = CVT_WARPS / CVT_GROUPS;
  static constexpr int EPI_WARPS = 4;
  static constexpr int THREADS = (2 + CVT_WARPS + EPI_WARPS) * 32;
  static constexpr size_t SMEM_RAW = size_t(RS) * RAW_BYTES;
  static constexpr size_t SMEM_A = size_t(AS) * A_BYTES;
  static constexpr size_t SMEM_B = size_t(2) * B_BYTES;
  static constexpr size_t SMEM_BAR = 512;
  static constexpr size_t SMEM_HIST = kHistBins * 4;
  static constexpr size_t SMEM_TOTAL = 1024 + SMEM_RAW + SMEM_A + SMEM_B + SMEM_BAR + SMEM_HIST;
  static_assert(SMEM_TOTAL <= 232448, "shared memory budget");
};

struct CvtBarriers {
  uint64_t rfull[8];
  uint64_t rempty[8];
  uint64_t afull[4];
  uint64_t aempty[4];
  uint64_t bfull[2];
  uint64_t bempty[2];
  uint64_t tfull[8];
  uint64_t tempty[8];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(CvtBarriers) <= 512, "barrier block");

__device__ __forceinline__ void cvt_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > LSI_WAIT_LIMIT_NS) {
      atomicOr(&g_fault, FAULT_WAIT_TIMEOUT);
      return;
    }
  }
}

// 4 signed bytes -> 4 bf16, exactly.  For a byte v = sign*128 + m (m < 128)
// the bf16 pattern 0x4300 | m is 128 + m, and 0x4300 | (v & 0x80) is 128 or
// 256; their bf16 difference m - sign*128 = v is representable, so the
// packed subtraction is exact.
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t t0 = __byte_perm(x, 0u, 0x4140);  // bytes 0,1 into the low byte of each half
  const uint32_t t1 = __byte_perm(x, 0u, 0x4342);  // bytes 2,3
  const uint32_t m0 = (t0 & 0x007F007Fu) | 0x43004300u, o0 = (t0 & 0x00800080u) | 0x43004300u;
  const uint32_t m1 = (t1 & 0x007F007Fu) | 0x43004300u, o1 = (t1 & 0x00800080u) | 0x43004300u;
  __nv_bfloat162 r0 = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&m0),
                              *reinterpret_cast<const __nv_bfloat162*>(&o0));
  __nv_bfloat162 r1 = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&m1),
                              *reinterpret_cast<const __nv_bfloat162*>(&o1));
  lo = *reinterpret_cast<uint32_t*>(&r0);
  hi = *reinterpret_cast<uint32_t*>(&r1);
}

// 2 e4m3 codes (low 16 bits of x, element 0 in the low byte) -> bf16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t x) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(x));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  const float2 f = __half22float2(h);
  __nv_bfloat162 r = __float22bfloat162_rn(f);
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
  lo = e4m3x2_to_bf16x2(x & 0xFFFFu);
  hi = e4m3x2_to_bf16x2(x >> 16);
}

template <int FMT>
__global__ void __launch_bounds__(CvtCfg<FMT>::THREADS, 1)
    score_cvt_kernel(const __grid_constant__ CUtensorMap qmap, const CvtParams p) {
  using C = CvtCfg<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sR = smem;
  uint8_t* sA = smem + C::SMEM_RAW;
  uint8_t* sB = sA + C::SMEM_A;
  CvtBarriers* bars = reinterpret_cast<CvtBarriers*>(sB + C::SMEM_B);
  uint32_t* shist = reinterpret_cast<uint32_t*>(sB + C::SMEM_B + C::SMEM_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const bool use_hist = p.hist != nullptr;
  if (use_hist)
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) shist[i] = 0;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NT = (p.N + C::BM - 1) / C::BM;
  const long long units = static_cast<long long>(p.B) * NT;
  const long long u_begin = units * blockIdx.x / gridDim.x;
  const long long u_end = units * (blockIdx.x + 1) / gridDim.x;
  const uint8_t* keys = static_cast<const uint8_t*>(p.keys);

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
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&qmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int rs = 0;
    uint32_t rphase = 0;
    int prev_b = -1;
    int bslot = 1;
    uint32_t bphase[2] = {0, 0};
    int issued[8];
    uint32_t issued_par[8];
    for (int s = 0; s < 8; ++s) issued[s] = 0, issued_par[s] = 0;
    int b_issued[2] = {0, 0};
    uint32_t b_par[2] = {0, 0};
    bool ok = true;
    // gathered form: row ids of a unit's tile (-1 past the end)
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
    if (p.rows != nullptr && u_begin < u_end) load_rids(up.b, up.tile, rid_next);
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
        prev_b = b;
      }
      if (!warp_wait(&bars->rempty[rs], rphase ^ 1, abort_flag)) { ok = false; break; }
      uint8_t* dst = sR + rs * C::RAW_BYTES;
      const int j0 = tile * C::BM;
      const int nrows = min(C::BM, p.N - j0);
      if (p.rows == nullptr) {
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(nrows) * C::ROW_BYTES;
          mbar_arrive_expect_tx(&bars->rfull[rs], bytes);
          const uint8_t* src = keys + (static_cast<int64_t>(b) * p.N + j0) * C::ROW_BYTES;
          bulk_load(dst, src, bytes, &bars->rfull[rs]);
        }
      } else {
        // gathered: lane l copies rows l, l+32, l+64, l+96 of the tile; the
        // row ids of the next unit are read now, so their latency overlaps
        // this unit's copies
        int32_t rid[4];
        int cnt = 0;
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
        // 16-byte cp.async chunks, ROW_BYTES / 16 lanes per row: one warp
        // instruction copies 512 contiguous-per-row bytes (a per-row bulk copy
        // each would queue 128 small copies on the TMA unit)
        constexpr int CPR = C::ROW_BYTES / 16;           // chunks per row
        constexpr int RPI = 32 / CPR;                    // rows per warp instruction
        const int chunk = lane % CPR, sub = lane / CPR;
#pragma unroll
        for (int it = 0; it < C::BM / RPI; ++it) {
          const int r = it * RPI + sub;
          const int32_t rr = __shfl_sync(0xffffffffu, rid[(it * RPI) >> 5], r & 31);  // row r's id: lane r % 32
          if (rr >= 0)
            cp_async_16(dst + r * C::ROW_BYTES + chunk * 16,
                        keys + (static_cast<int64_t>(b) * p.key_stride + rr) * C::ROW_BYTES + chunk * 16);
        }
        cp_async_mbar_arrive(&bars->rfull[rs]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->rfull[rs]);
        (void)cnt;
      }
      issued[rs] = 1;
      issued_par[rs] = rphase;
      if (++rs == C::RS) { rs = 0; rphase ^= 1; }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok && lane == 0) {
      for (int s = 0; s < C::RS; ++s)
        if (issued[s]) cvt_wait_drain(&bars->rfull[s], issued_par[s]);
      for (int s = 0; s < 2; ++s)
        if (b_issued[s]) cvt_wait_drain(&bars->bfull[s], b_par[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp follows the units: on a problem change its lanes turn the
    // new query tile into fp16 (8-bit keys); one elected lane issues the MMAs.
    constexpr bool F16 = FMT != SRC_BF16;
    constexpr uint32_t idesc = F16 ? idesc_f16_f32(C::BM, C::BN) : idesc_bf16_f32(C::BM, C::BN);
    int as = 0;
    uint32_t aphase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int prev_b = -1;
    int bslot = 1;
    uint32_t bphase[2] = {0, 0};
    const uint32_t a_base = smem_u32(sA);
    const uint32_t b_base = smem_u32(sB);
    UnitPos up;
    up.init(u_begin, NT, 1);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, 1)) {
      const int b = up.b;
      if (b != prev_b) {
        if (prev_b >= 0) umma_commit_warp(&bars->bempty[bslot]);
        bslot ^= 1;
        // every lane observes the barrier itself: all of them read the tile next
        const bool ok = mbar_wait(&bars->bfull[bslot], bphase[bslot], abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        bphase[bslot] ^= 1;
        prev_b = b;
        if (F16) {
          q_tile_to_f16(sB + bslot * C::B_BYTES, C::B_HALF, lane);
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      if (!warp_wait(&bars->tempty[acc], acc_phase ^ 1, abort_flag)) break;
      tc_fence_after();
      if (!warp_wait(&bars->afull[as], aphase, abort_flag)) break;
      tc_fence_after();
      {
        const uint32_t a_addr = a_base + as * C::A_BYTES;
        const uint32_t b_addr = b_base + bslot * C::B_BYTES;
        const uint32_t d_tmem = tmem_base + acc * C::BN;
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t adesc = sw128_kmajor_desc(a_addr + (kk >> 2) * C::A_HALF + koff);
          const uint64_t bdesc = sw128_kmajor_desc(b_addr + (kk >> 2) * C::B_HALF + koff);
          umma_f16_warp(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bars->aempty[as]);
        umma_commit_warp(&bars->tfull[acc]);
      }
      if (++as == C::AS) { as = 0; aphase ^= 1; }
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
    }
    umma_commit_warp(&bars->drain);
    if (lane == 0) cvt_wait_drain(&bars->drain, 0);
    __syncwarp();
  } else if (warp < 2 + C::CVT_WARPS) {
    // ------------------------------------------------------------ converters
    // CVT_GROUPS groups of warps take alternate units, so that many tiles are
    // widened at once; each group's threads share one tile.
    constexpr int CT = C::CVT_GROUP_WARPS * 32;
    const int cg = (warp - 2) / C::CVT_GROUP_WARPS;
    const int ct = threadIdx.x - 64 - cg * CT;  // 0 .. CT-1
    const long long count = u_end - u_begin;
    for (long long i = cg; i < count; i += C::CVT_GROUPS) {
      const int rs = static_cast<int>(i % C::RS), as = static_cast<int>(i % C::AS);
      const uint32_t rphase = static_cast<uint32_t>((i / C::RS) & 1), aphase = static_cast<uint32_t>((i / C::AS) & 1);
      if (!warp_wait(&bars->rfull[rs], rphase, abort_flag)) break;
      if (!warp_wait(&bars->aempty[as], aphase ^ 1, abort_flag)) break;
      const uint8_t* raw = sR + rs * C::RAW_BYTES;
      uint8_t* a = sA + as * C::A_BYTES;
      if (FMT == SRC_BF16) {
        constexpr int PER = (C::BM * 16) / CT;  // 16-byte chunks per thread
        uint4 v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int id = i * CT + ct;
          v[i] = *reinterpret_cast<const uint4*>(raw + (id >> 4) * 256 + (id & 15) * 16);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int id = i * CT + ct;
          const int row = id >> 4, cc = id & 15;
          const int panel = cc >> 3, j = cc & 7;
          *reinterpret_cast<uint4*>(a + panel * C::A_HALF + row * 128 + ((j ^ (row & 7)) << 4)) = v[i];
        }
      } else {
        // A warp takes 4 rows x 8 input chunks per step.  Within each group of
        // 8 lanes (one shared-memory wavefront) the even row's chunks 0-3 (or
        // 4-7) pair with the odd row's other half: the 16-byte reads cover all
        // 32 banks, and so do both widened stores, whose chunk indexes then
        // differ in parity under the row swizzle.
        constexpr int PER = (C::BM * 8) / CT;
        const int qg = (ct & 31) >> 3, rsel = (ct >> 2) & 1;
        const int row0 = (ct >> 5) * 4 + 2 * (qg >> 1) + rsel;
        const int cc = 4 * (rsel ^ (qg & 1)) + (ct & 3);
        uint4 v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i)
          v[i] = *reinterpret_cast<const uint4*>(raw + (row0 + i * (CT / 8)) * 128 + cc * 16);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int row = row0 + i * (CT / 8);
          uint4 o0, o1;
          if (FMT == SRC_INT8) {
            i8x4_to_f16x4(v[i].x, o0.x, o0.y);
            i8x4_to_f16x4(v[i].y, o0.z, o0.w);
            i8x4_to_f16x4(v[i].z, o1.x, o1.y);
            i8x4_to_f16x4(v[i].w, o1.z, o1.w);
          } else {
            e4m3x4_to_f16x4(v[i].x, o0.x, o0.y);
            e4m3x4_to_f16x4(v[i].y, o0.z, o0.w);
            e4m3x4_to_f16x4(v[i].z, o1.x, o1.y);
            e4m3x4_to_f16x4(v[i].w, o1.z, o1.w);
          }
          const int panel = cc >> 2;
          const int j0 = (cc & 3) * 2;
          uint8_t* rowp = a + panel * C::A_HALF + row * 128;
          *reinterpret_cast<uint4*>(rowp + ((j0 ^ (row & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(rowp + (((j0 + 1) ^ (row & 7)) << 4)) = o1;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->rempty[rs]);
        mbar_arrive(&bars->afull[as]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int EPI0 = (2 + C::CVT_WARPS) * 32;  // first epilogue thread
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    // what the epilogue needs from global memory besides TMEM, for one unit
    auto fetch = [&](int b, int tile, bool& valid, float& sc) {
      const int j = tile * C::BM + quad * 32 + lane;
      valid = false;
      sc = 1.f;
      if (j >= p.N) return;
      int64_t sidx;
      if (p.rows) {
        const int32_t r = __ldg(p.rows + static_cast<int64_t>(b) * p.N + j);
        valid = (r >= 0) && (r < p.key_rows);
        sidx = static_cast<int64_t>(b) * p.key_stride + (valid ? r : 0);
      } else {
        valid = (p.n_valid == nullptr) || (j < __ldg(p.n_valid + b));
        sidx = static_cast<int64_t>(b) * p.N + j;
      }
      if (FMT != SRC_BF16 && valid) sc = __ldg(p.scale + sidx);
    };
    bool nvalid = false;
    float nsc = 1.f;
    UnitPos up;
    up.init(u_begin, NT, 1);
    if (u_begin < u_end) fetch(up.b, up.tile, nvalid, nsc);
    int w_b = -1;
    HeadWeights wreg;
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, 1)) {
      const int tile = up.tile;
      const int b = up.b;
      const bool valid = nvalid;
      const float sc = nsc;
      if (u + 1 < u_end) {  // next unit's row id and scale are in flight while this unit waits and computes
        if (tile + 1 == NT) fetch(b + 1, 0, nvalid, nsc);
        else fetch(b, tile + 1, nvalid, nsc);
      }
      if (w_b != b) {  // head weights of this problem, kept in registers
        if (FMT != SRC_BF16) {
          // lane h: head h's weight times 2^-s_h, the inverse of the query tile's shift
          const uint16_t* qrow = p.q + (static_cast<int64_t>(b) * p.q_row_stride + lane) * kDim;
          const float wl = __ldg(p.w + static_cast<int64_t>(b) * kHeads + lane) * exp2i(-q_head_shift_global(qrow));
#pragma unroll
          for (int i = 0; i < 16; ++i)
            wreg.v[i] = pack_f32x2(__shfl_sync(0xffffffffu, wl, 2 * i), __shfl_sync(0xffffffffu, wl, 2 * i + 1));
        } else {
          wreg.load(p.w + static_cast<int64_t>(b) * kHeads);
        }
        w_b = b;
      }
      if (!warp_wait(&bars->tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int j = tile * C::BM + quad * 32 + lane;
      uint32_t v[32];
      tmem_ld_32x32_nowait(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * C::BN),
                           v);
      tmem_wait_ld(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tempty[acc]);
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
      const bool last_of_row = (u + 1 == u_end) || (tile + 1 == NT);
      if (j < p.N) {
        float s = neg_inf();
        if (valid) {
          s = (FMT == SRC_BF16) ? head_reduce_w(v, wreg) : head_reduce_scaled(v, wreg, sc);
          if (use_hist) atomicAdd(&shist[hist_bin(order_code(s))], 1u);
        }
        p.out[static_cast<int64_t>(b) * p.N + j] = s;
      }
      if (use_hist && last_of_row) {  // warp-uniform: every epilogue warp sees the same unit
        role_barrier(1, C::EPI_WARPS * 32);
        flush_hist(shist, p.hist + static_cast<int64_t>(b) * kHistBins, threadIdx.x - EPI0, C::EPI_WARPS * 32);
        role_barrier(1, C::EPI_WARPS * 32);
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

template <int FMT>
static cudaError_t launch_cvt(const CUtensorMap* qmap, const CvtParams& p, int num_sms, cudaStream_t st) {
  using C = CvtCfg<FMT>;
  static std::atomic<uint64_t> attr_done{0};
  {
    const cudaError_t e = smem_limit_once(attr_done, reinterpret_cast<const void*>(&score_cvt_kernel<FMT>), C::SMEM_TOTAL);
    if (e != cudaSuccess) return e;
  }
  const int NT = (p.N + C::BM - 1) / C::BM;
  const long long units = static_cast<long long>(p.B) * NT;
  if (units == 0) return cudaSuccess;
  const int grid = static_cast<int>(units < num_sms ? units : num_sms);
  score_cvt_kernel<FMT><<<grid, C::THREADS, C::SMEM_TOTAL, st>>>(*qmap, p);
  return cudaGetLastError();
}

cudaError_t launch_score_cvt(const CUtensorMap* qmap, const CvtParams& p, int num_sms, cudaStream_t st) {
  switch (p.fmt) {
    case SRC_INT8: return launch_cvt<SRC_INT8>(qmap, p, num_sms, st);
    case SRC_E4M3: return launch_cvt<SRC_E4M3>(qmap, p, num_sms, st);
    case SRC_BF16: return launch_cvt<SRC_BF16>(qmap, p, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lsi

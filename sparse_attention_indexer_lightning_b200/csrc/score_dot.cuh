// Single-dot bucket scores of the native LSA flat search on the sm_100a
// tensor cores ("Latent Sparse Attention", section "The method, term by
// term", step 5: a query scores a bucket by one dot product of its 64-d unit
// index query with the bucket's unit centroid; section "How LSA finds the
// keys": 64 dimensions per query against every centroid of the blocks
// before its own).
//
//   out[t][p] = sum_{d < 64} q[t][d] * c[p][d]      (bf16 inputs, fp32 sums)
//
// Layout (swap-AB as in the indexer scorer): the MMA's M side is a tile of
// 128 centroids (A, K-major: a 64-d bf16 row is one 128-byte swizzle row),
// the N side 256 queries (B), K = 64 as 4 MMAs of K = 16; the fp32
// accumulator lives in TMEM with one centroid per lane, and each epilogue
// thread stores its centroid's scores for 64 queries (one coalesced 128-byte
// row segment per query and warp).  Columns past a query's visible buckets
// are computed like the rest; the selection reads only the visible prefix.
//
// Roles (one persistent CTA per SM, contiguous runs of work units ordered
// query group, centroid tile):
//   warp 0      TMA producer (a centroid tile every unit, the query tile on group change)
//   warp 1      TMEM allocator + MMA issuer
//   warps 2..17 epilogue: 4 per TMEM lane quadrant, 64 queries each
// Every wait is bounded; a wait that runs out raises the library fault word.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

struct DotCfg {
  static constexpr int BM = kTileKeys;            // 128 centroids per tile
  static constexpr int QB = 256;                  // queries per group (MMA N)
  static constexpr int DIM = kLsaDim;             // 64
  static constexpr int A_BYTES = BM * DIM * 2;    // 16 KB
  static constexpr int B_BYTES = QB * DIM * 2;    // 32 KB
  static constexpr int STAGES = 4;
  static constexpr int ACC = 2;
  static constexpr int ACC_COLS = QB;
  static constexpr int EPI_SETS = 4;
  static constexpr int EPI_WARPS = 4 * EPI_SETS;
  static constexpr int COLS_PER_WARP = QB / EPI_SETS;   // 64
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr size_t SMEM_A = size_t(STAGES) * A_BYTES;
  static constexpr size_t SMEM_B = size_t(2) * B_BYTES;
  static constexpr size_t SMEM_BAR = 512;
  // filter form, per epilogue warp: its 64 queries' negated thresholds and
  // visible counts, its slot counters of their list segments, a copy of each
  // lane's 32 scores of a half (read back for the listed ones) and a queue of
  // QUEUE listed (score bits, bucket, column) entries
  static constexpr int QUEUE = 64;
  static constexpr size_t SMEM_FW = 64 * 4 * 3 + 32 * 32 * 4 + QUEUE * 4 * 3;
  static constexpr size_t SMEM_F = size_t(EPI_WARPS) * SMEM_FW;
  static constexpr size_t SMEM_TOTAL = 1024 /*align slack*/ + SMEM_A + SMEM_B + SMEM_BAR + SMEM_F;
  static_assert(SMEM_TOTAL <= 232448, "shared memory budget");
  static_assert(DIM * 2 == 128, "one 128-byte swizzle row per vector");
};

struct DotBarriers {
  uint64_t full[DotCfg::STAGES];
  uint64_t empty[DotCfg::STAGES];
  uint64_t bfull[2];
  uint64_t bempty[2];
  uint64_t tfull[DotCfg::ACC];
  uint64_t tempty[DotCfg::ACC];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(DotBarriers) <= DotCfg::SMEM_BAR, "barrier block");


// FILTER: instead of storing every score, append (score, bucket) to the
// query's candidate list when the bucket is visible and its score reaches the
// query's threshold (LSA's sampled threshold: "appends only those above it to
// a short list"); a list that runs out of room flags its row.
template <bool FILTER>
__global__ void __launch_bounds__(DotCfg::THREADS, 1)
    dot_tc_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap qmap,
                  const DotParams p) {
  using C = DotCfg;
  if (p.run_if != nullptr && *p.run_if == 0) return;  // a conditional launch with nothing to do
  int T = p.T;
  if (!FILTER && p.live_rows != nullptr) {            // rows past the live count are not scored
    const int live = *p.live_rows - p.live_base;
    T = live < 0 ? 0 : (live < T ? live : T);
    if (T == 0) return;
  }
  const int P = p.P;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::SMEM_A;
  DotBarriers* bars = reinterpret_cast<DotBarriers*>(smem + C::SMEM_A + C::SMEM_B);
  uint8_t* sfilt = smem + C::SMEM_A + C::SMEM_B + C::SMEM_BAR;
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = (T + C::QB - 1) / C::QB;
  const int NT = (P + C::BM - 1) / C::BM;
  const long long units = static_cast<long long>(G) * NT;
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
    tmem_alloc(&bars->tmem_base, C::ACC * C::ACC_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&cmap);
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
      int prev_g = -1;
      int bslot = 1;
      uint32_t bphase[2] = {0, 0};
      uint32_t issued_mask = 0, issued_par = 0;     // stages / slots with a copy in flight (bit s), its parity
      uint32_t b_issued = 0, b_par = 0;
      bool ok = true;
      UnitPos up;
      up.init(u_begin, NT, G);
      for (long long u = u_begin; u < u_end && ok; ++u, up.next(NT, G)) {
        const int tile = up.tile, g = up.g;
        if (g != prev_g) {
          bslot ^= 1;
          if (!mbar_wait(&bars->bempty[bslot], bphase[bslot] ^ 1, abort_flag)) { ok = false; break; }
          b_issued |= 1u << bslot;
          b_par = (b_par & ~(1u << bslot)) | (bphase[bslot] << bslot);
          bphase[bslot] ^= 1;
          mbar_arrive_expect_tx(&bars->bfull[bslot], C::B_BYTES);
          tma_load_2d(sB + bslot * C::B_BYTES, &qmap, &bars->bfull[bslot], 0, g * C::QB);
          prev_g = g;
        }
        if (!mbar_wait(&bars->empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->full[stage], C::A_BYTES);
        tma_load_2d(sA + stage * C::A_BYTES, &cmap, &bars->full[stage], 0, tile * C::BM);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA goes away.
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask >> s & 1u) mbar_wait_drain(&bars->full[s], issued_par >> s & 1u);
        for (int s = 0; s < 2; ++s)
          if (b_issued >> s & 1u) mbar_wait_drain(&bars->bfull[s], b_par >> s & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(C::BM, C::QB);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int prev_g = -1;
    int bslot = 1;
    uint32_t bphase[2] = {0, 0};
    const uint32_t a_base = smem_u32(sA);
    const uint32_t b_base = smem_u32(sB);
    UnitPos up;
    up.init(u_begin, NT, G);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, G)) {
      if (up.g != prev_g) {
        if (prev_g >= 0 && lane == 0) umma_commit(&bars->bempty[bslot]);
        bslot ^= 1;
        if (!warp_wait(&bars->bfull[bslot], bphase[bslot], abort_flag)) break;
        bphase[bslot] ^= 1;
        prev_g = up.g;
      }
      if (!warp_wait(&bars->tempty[acc], acc_phase ^ 1, abort_flag)) break;
      tc_fence_after();
      if (!warp_wait(&bars->full[stage], phase, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_addr = a_base + stage * C::A_BYTES;
        const uint32_t b_addr = b_base + bslot * C::B_BYTES;
        const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
#pragma unroll
        for (int kk = 0; kk < C::DIM / 16; ++kk) {   // 16 bf16 = 32 B inside the 128-byte swizzle row
          const uint64_t adesc = sw128_kmajor_desc(a_addr + kk * 32);
          const uint64_t bdesc = sw128_kmajor_desc(b_addr + kk * 32);
          umma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->empty[stage]);
        umma_commit(&bars->tfull[acc]);
      }
      __syncwarp();
      if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
    }
    // All MMAs the issuing lane started are complete once `drain` flips.
    if (lane == 0) {
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;                // TMEM lane quadrant this warp may read
    const int cset = ew >> 2;                 // queries [64 * cset, 64 * cset + 64) of the group
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    // filter form: the warp's 64 queries' negated thresholds and visible
    // counts in shared memory (reloaded when the group changes; a query past the end
    // sees nothing), vis_min the smallest count; the warp appends to its own
    // quarter (by lane quadrant) of this CTA's segment of each row's list,
    // with slot counters in shared memory that no other warp touches, written
    // out when the group changes and at the end.
    float* thr_s = reinterpret_cast<float*>(sfilt + (warp - 2) * C::SMEM_FW);
    int* vis_s = reinterpret_cast<int*>(thr_s + 64);
    uint32_t* cnt_s = reinterpret_cast<uint32_t*>(vis_s + 64);
    // lane l's scores at row l (128 bytes), 16-byte chunk q stored at chunk
    // q ^ (l & 7) so that the 32 lanes' 16-byte stores spread over the banks
    uint4* spill = reinterpret_cast<uint4*>(cnt_s + 64) + lane * 8;
    uint32_t* q_val = reinterpret_cast<uint32_t*>(reinterpret_cast<uint4*>(cnt_s + 64) + 32 * 8);
    int32_t* q_pc = reinterpret_cast<int32_t*>(q_val + C::QUEUE);
    int32_t* q_col = q_pc + C::QUEUE;
    int qn = 0;                               // queued entries (warp-uniform)
    int vis_min = 0;
    LsaSeg seg{0, 0, 0};
    int64_t sub_off = 0;
    uint32_t sub_len = 0;
    int cur_t0 = -1;                          // the rows whose counters are live
    // the queued entries take their slots (one shared atomic each, up to 32
    // at a time) and go to the current group's list segments
    auto drain = [&](int t0d) {
      __syncwarp();
      for (int e = lane; e < qn; e += 32) {
        const int c = q_col[e];
        const int t = t0d + c;
        const uint32_t slot = atomicAdd(&cnt_s[c], 1u);
        if (slot < sub_len) {
          p.cand_list[static_cast<int64_t>(t) * p.ld_cand + sub_off + slot] =
              make_uint2(q_val[e], static_cast<uint32_t>(q_pc[e]));
        } else {
          p.row_over[t] = 1;
          *p.any_over = 1;
        }
      }
      qn = 0;
      __syncwarp();
    };
    auto flush = [&](int t0f) {
      drain(t0f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0f + 32 * h + lane;
        if (t < T && seg.j < p.nseg)
          p.cand_cnt[(static_cast<int64_t>(t) * p.nseg + seg.j) * 4 + quad] = cnt_s[32 * h + lane];
      }
    };
    UnitPos up;
    up.init(u_begin, NT, G);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, G)) {
      const int pc = up.tile * C::BM + quad * 32 + lane;     // this thread's centroid
      const int t0 = up.g * C::QB + cset * C::COLS_PER_WARP;
      if (FILTER && (u == u_begin || up.tile == 0)) {
        if (cur_t0 >= 0) flush(cur_t0);
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = t0 + 32 * h + lane;
          // negated; a zero threshold (either sign) becomes +0, so that a
          // score of -0 or +0 sums to +0 and is listed, as the top-k's keys
          // (which give -0 and +0 one code) require
          const float th = (t < T) ? p.tau[static_cast<int64_t>(t) * p.ld_tau] : 0.f;
          thr_s[32 * h + lane] = (th == 0.f) ? 0.f : -th;
          vis_s[32 * h + lane] = (t < T) ? p.vis[t] : 0;
          cnt_s[32 * h + lane] = 0;
        }
        vis_min = min(vis_s[lane], vis_s[32 + lane]);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) vis_min = min(vis_min, __shfl_xor_sync(0xffffffffu, vis_min, d));
        seg = lsa_segment(units, static_cast<int>(gridDim.x), NT, up.g, static_cast<int>(blockIdx.x), p.cap2,
                          p.slack);
        if (seg.j >= p.nseg) seg.len = 0;     // no counter for it: every listed pair flags its row
        sub_len = static_cast<uint32_t>(seg.len / 4);
        sub_off = seg.off + static_cast<int64_t>(quad) * sub_len;
        cur_t0 = t0;
        __syncwarp();
      }
      if (!warp_wait(&bars->tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t col = tmem_base + lane_off + static_cast<uint32_t>(acc * C::ACC_COLS + cset * C::COLS_PER_WARP);
      const int nt = min(C::COLS_PER_WARP, T - t0);          // queries of this warp that exist
      auto release = [&]() {                                  // the accumulator is read: hand it back
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->tempty[acc]);
        if (++acc == C::ACC) { acc = 0; acc_phase ^= 1; }
      };
      if (!FILTER) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32_nowait(col, v0);
        tmem_ld_32x32_nowait(col + 32, v1);
        tmem_wait_ld(v0);
        tmem_wait_ld(v1);
        release();
        if (pc < P && nt > 0) {
          float* o = p.out + static_cast<int64_t>(t0) * p.ld_out + pc;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nt) o[static_cast<int64_t>(j) * p.ld_out] = __uint_as_float(v0[j]);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (32 + j < nt) o[static_cast<int64_t>(32 + j) * p.ld_out] = __uint_as_float(v1[j]);
        }
      } else {
        // One 32-column half at a time: this lane's listed columns as a bit
        // mask.  A score is listed when it is visible and not below its
        // column's threshold in the top-k's key order: the sign bit of
        // fl(score + (-threshold)) (one rounding, so it is set exactly when
        // score < threshold; -0 and +0 equal; a NaN score is listed too,
        // which changes nothing since the top-k ranks it last; a -inf
        // threshold lists every visible bucket).  The
        // sums go two at a time through the packed fp32 adder, their sign
        // bits are shifted into four 8-bit words (column 4 * i + r at bit
        // 8 * r + 7 - i of the combined word); a tile below every column's
        // visible count skips the count.
        const bool all_visible = up.tile * C::BM + C::BM <= vis_min;
        const float4* nthr4 = reinterpret_cast<const float4*>(thr_s);
        const int4* vis4 = reinterpret_cast<const int4*>(vis_s);
        uint32_t v[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_ld_32x32_nowait(col + 32 * h, v);
          tmem_wait_ld(v);
          if (h == 1) release();
          uint32_t neg[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 nt = nthr4[8 * h + i];
            uint64_t d01, d23;
            asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d01)
                : "l"(pack_f32x2(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]))),
                  "l"(pack_f32x2(nt.x, nt.y)));
            asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d23)
                : "l"(pack_f32x2(__uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]))),
                  "l"(pack_f32x2(nt.z, nt.w)));
            float e0, e1, e2, e3;
            unpack_f32x2(d01, e0, e1);
            unpack_f32x2(d23, e2, e3);
            neg[0] = __funnelshift_l(__float_as_uint(e0), neg[0], 1);
            neg[1] = __funnelshift_l(__float_as_uint(e1), neg[1], 1);
            neg[2] = __funnelshift_l(__float_as_uint(e2), neg[2], 1);
            neg[3] = __funnelshift_l(__float_as_uint(e3), neg[3], 1);
          }
          uint32_t mask = ~(neg[0] | (neg[1] << 8) | (neg[2] << 16) | (neg[3] << 24));
          if (!all_visible) {                           // visible: pc - vis < 0
            uint32_t vis_neg[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int4 vv = vis4[8 * h + i];
              vis_neg[0] = __funnelshift_l(static_cast<uint32_t>(pc - vv.x), vis_neg[0], 1);
              vis_neg[1] = __funnelshift_l(static_cast<uint32_t>(pc - vv.y), vis_neg[1], 1);
              vis_neg[2] = __funnelshift_l(static_cast<uint32_t>(pc - vv.z), vis_neg[2], 1);
              vis_neg[3] = __funnelshift_l(static_cast<uint32_t>(pc - vv.w), vis_neg[3], 1);
            }
            mask &= vis_neg[0] | (vis_neg[1] << 8) | (vis_neg[2] << 16) | (vis_neg[3] << 24);
          }
          // listed pairs: each lane's next one per round, queued in lane
          // order (a round rarely repeats: few lanes list two in a half)
          if (__any_sync(0xffffffffu, mask != 0)) {
            if (mask) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                spill[q ^ (lane & 7)] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            while (true) {
              const uint32_t bal = __ballot_sync(0xffffffffu, mask != 0);
              if (bal == 0) break;
              const int n = __popc(bal);
              if (qn + n > C::QUEUE) drain(t0);
              if (mask) {
                const int bit = __ffs(mask) - 1;
                mask &= mask - 1;
                const int j = 4 * (7 - (bit & 7)) + (bit >> 3);
                const int e = qn + __popc(bal & ((1u << lane) - 1u));
                q_val[e] = reinterpret_cast<const uint32_t*>(spill + ((j >> 2) ^ (lane & 7)))[j & 3];
                q_pc[e] = pc;
                q_col[e] = 32 * h + j;
              }
              qn += n;
            }
            if (qn >= C::QUEUE / 2) drain(t0);
          }
        }
      }
    }
    if (FILTER && cur_t0 >= 0) flush(cur_t0);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::ACC * C::ACC_COLS);
  }
}

template <bool FILTER>
static cudaError_t launch_dot(const CUtensorMap* cmap, const CUtensorMap* qmap, const DotParams& p, int num_sms,
                              cudaStream_t st) {
  using C = DotCfg;
  static std::atomic<uint64_t> attr_done{0};
  {
    const cudaError_t e = smem_limit_once(attr_done, reinterpret_cast<const void*>(&dot_tc_kernel<FILTER>), C::SMEM_TOTAL);
    if (e != cudaSuccess) return e;
  }
  const int grid = dot_tc_grid(p.T, p.P, num_sms);
  if (grid == 0) return cudaSuccess;
  if (FILTER) {                            // the segments must fit the counters and the rows
    const long long units = static_cast<long long>((p.T + C::QB - 1) / C::QB) * ((p.P + C::BM - 1) / C::BM);
    const int NT = (p.P + C::BM - 1) / C::BM;
    if (lsa_max_segments(units, grid, NT) > p.nseg ||
        p.cap2 + static_cast<long long>(p.slack) * p.nseg > p.ld_cand)
      return cudaErrorInvalidValue;
  }
  dot_tc_kernel<FILTER><<<grid, C::THREADS, C::SMEM_TOTAL, st>>>(*cmap, *qmap, p);
  return cudaGetLastError();
}

int dot_tc_grid(int T, int P, int num_sms) {
  const long long units = static_cast<long long>((T + DotCfg::QB - 1) / DotCfg::QB) * ((P + DotCfg::BM - 1) / DotCfg::BM);
  return static_cast<int>(units < num_sms ? units : num_sms);
}

cudaError_t launch_dot_tc(const CUtensorMap* cmap, const CUtensorMap* qmap, const DotParams& p, int num_sms,
                          cudaStream_t st) {
  return p.out == nullptr ? launch_dot<true>(cmap, qmap, p, num_sms, st) : launch_dot<false>(cmap, qmap, p, num_sms, st);
}

// After the filtered scan, one CTA per row: the row's segments (one per CTA
// of the scan that scored it) are
// packed into one list of up to `cap` entries (nv[t] of them).  A row falls
// back to full scoring when a segment ran over (flagged in the scan), the
// list would exceed cap, or it holds fewer than min(top_p, visible) buckets.
__global__ void __launch_bounds__(256)
    lsa_compact_kernel(const uint2* __restrict__ slist, const uint32_t* __restrict__ cnt, int64_t ld_cand, int nseg,
                       int cap2, int slack, int grid, int NT, long long units, const int32_t* __restrict__ vis,
                       int top_p, int cap, float* __restrict__ cval, int32_t* __restrict__ clab,
                       int32_t* __restrict__ nv, int32_t* __restrict__ row_over, int* __restrict__ any_over) {
  __shared__ int offs[1025];
  __shared__ int64_t soff[1024];
  __shared__ int wsum[8];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const int g = t / DotCfg::QB;
  const int c0 = lsa_first_cta(units, grid, NT, g);
  const int nsub = 4 * nseg;                  // segment j's quarter q is sub-segment 4 * j + q
  // exclusive scan of the sub-segment counts (nsub <= 1024: 4 per thread);
  // a count past its sub-segment's length was flagged by the scan
  int c4[4];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sidx = tid * 4 + i;
    const int j = sidx >> 2, q = sidx & 3;
    c4[i] = 0;
    if (sidx < nsub && c0 + j < grid) {
      const LsaSeg sg = lsa_segment(units, grid, NT, g, c0 + j, cap2, slack);
      const int sub_len = sg.len / 4;
      soff[sidx] = sg.off + static_cast<int64_t>(q) * sub_len;
      c4[i] = static_cast<int>(min(cnt[static_cast<int64_t>(t) * nsub + sidx], static_cast<uint32_t>(sub_len)));
    }
    mine += c4[i];
  }
  int incl = mine;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < wid; ++w) run += wsum[w];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sidx = tid * 4 + i;
    if (sidx < nsub) offs[sidx] = run;
    run += c4[i];
  }
  if (tid == 255) offs[nsub] = run;
  __syncthreads();
  const int total = offs[nsub];
  const int need = min(top_p, vis[t]);
  if (tid == 0) {
    nv[t] = min(total, cap);
    if (total > cap || total < need) {
      row_over[t] = 1;
      *any_over = 1;
    }
  }
  if (total > cap) return;
  // output entry o comes from the sub-segment s with offs[s] <= o < offs[s + 1]
  for (int o = tid; o < total; o += 256) {
    int lo = 0, hi = nsub;                      // offs[lo] <= o < offs[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs[mid] <= o) lo = mid;
      else hi = mid;
    }
    const uint2 e = slist[static_cast<int64_t>(t) * ld_cand + soff[lo] + (o - offs[lo])];
    cval[static_cast<int64_t>(t) * cap + o] = __uint_as_float(e.x);
    clab[static_cast<int64_t>(t) * cap + o] = static_cast<int32_t>(e.y);
  }
}

// The rows the sampled threshold missed, in ascending order: list[0, count),
// -1 after (one CTA); run[c] = 1 when chunk c (list entries [c * rows,
// (c + 1) * rows)) holds any, for c < n_chunks.
__global__ void __launch_bounds__(1024)
    lsa_flag_list_kernel(const int32_t* __restrict__ row_over, int T, int rows, int n_chunks,
                         int32_t* __restrict__ list, int32_t* __restrict__ count, int32_t* __restrict__ run) {
  __shared__ int wsum[32];
  __shared__ int base_s;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) base_s = 0;
  __syncthreads();
  for (int t0 = 0; t0 < T; t0 += 1024) {
    const int t = t0 + tid;
    const int f = (t < T && row_over[t] != 0) ? 1 : 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[wid] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      before += (w < wid) ? wsum[w] : 0;
      total += wsum[w];
    }
    const int base = base_s;
    if (f) list[base + before + __popc(bal & ((1u << lane) - 1u))] = t;
    __syncthreads();                            // every thread has read base_s and wsum
    if (tid == 0) base_s = base + total;
    __syncthreads();
  }
  const int n = base_s;
  for (int i = n + tid; i < T; i += 1024) list[i] = -1;
  if (tid == 0) *count = n;
  for (int c = tid; c < n_chunks; c += 1024) run[c] = (static_cast<long long>(c) * rows < n) ? 1 : 0;
}

// The missed rows' index queries and visible counts, in list order, into
// qbuf [T][64] and vbuf [T] (zeros past the count).
__global__ void lsa_gather_rows_kernel(const int32_t* __restrict__ list, const int32_t* __restrict__ count, int T,
                                       const uint16_t* __restrict__ q, const int32_t* __restrict__ vis,
                                       const int* __restrict__ run_if, uint16_t* __restrict__ qbuf,
                                       int32_t* __restrict__ vbuf) {
  if (*run_if == 0) return;
  const int n = *count;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;   // one 16-byte piece: row i / 8, piece i % 8
  if (i >= T * 8) return;
  const int r = i >> 3, piece = i & 7;
  const bool live = r < n;
  const int t = live ? list[r] : 0;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (live) v = reinterpret_cast<const uint4*>(q + static_cast<int64_t>(t) * kLsaDim)[piece];
  reinterpret_cast<uint4*>(qbuf + static_cast<int64_t>(r) * kLsaDim)[piece] = v;
  if (piece == 0) vbuf[r] = live ? vis[t] : 0;
}

// Visible buckets of each query (causal block visibility: the buckets of the
// complete blocks before the query's own block) and the LSA read list
// ("Latent Sparse Attention", section "The method, term by term", steps 5-6):
//   row t of keys_out: the sinks below the window, then the window
//   [block_start(t), t], then the long-range keys of the picked buckets read
//   best first, members that fall in the sinks or the window skipped, until
//   `budget` are held (the last bucket cut short); -1 after the end; n_out[t]
//   the row's length.  Bucket members are stored in ascending position order.
// The sample scores for the thresholds are the tensor-core scorer's, over the
// buckets 0, stride, 2*stride, ...; n_samp[t] counts those below row t's
// visible count.
__global__ void lsa_visible_kernel(const int64_t* __restrict__ q_pos, int T, int block_keys, int bpb, int P,
                                   int stride, int32_t* __restrict__ vis, int32_t* __restrict__ n_samp) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int64_t qp = q_pos[t] < 0 ? 0 : q_pos[t];
  const int64_t v = (qp / block_keys) * bpb;
  const int32_t vv = static_cast<int32_t>(v < P ? v : P);
  vis[t] = vv;
  if (n_samp) n_samp[t] = (vv + stride - 1) / stride;   // sampled buckets below the visible count
}

__device__ __forceinline__ int lower_bound_i32(const int32_t* __restrict__ a, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// One CTA of 256 threads per query: the picked buckets are taken 1024 at a
// time (4 per thread, every load of a round in flight together), their kept
// member counts scanned across the block, and the round's members copied by
// the whole block (output slot q from the bucket whose start is the last one
// at or below q), so that the stores are coalesced.
constexpr int kExpandThreads = 256;
constexpr int kExpandItems = 4;

__global__ void __launch_bounds__(kExpandThreads)
    lsa_expand_kernel(const int32_t* __restrict__ picked, const int64_t* __restrict__ q_pos, int T, int top_p,
                      const int32_t* __restrict__ off, const int32_t* __restrict__ mem, int P, int block_keys,
                      int n_sink, int budget, int32_t* __restrict__ keys_out, int row_len,
                      int32_t* __restrict__ n_out) {
  constexpr int kItems = kExpandThreads * kExpandItems;       // buckets per round
  __shared__ int warp_sum[kExpandThreads / 32];
  __shared__ int round_total;
  __shared__ int s_start[kItems + 1];                          // a round's output start of each bucket
  __shared__ int s_src[kItems];                                // and where its members begin in mem
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const int64_t qp = q_pos[t] < 0 ? 0 : q_pos[t];
  const int64_t wstart = (qp / block_keys) * block_keys;
  const int64_t sink_end = n_sink < wstart ? n_sink : wstart;   // sinks inside the window belong to it
  const int n_win = static_cast<int>(qp - wstart + 1);
  int32_t* out = keys_out + static_cast<int64_t>(t) * row_len;
  for (int j = tid; j < sink_end; j += kExpandThreads) out[j] = j;
  for (int j = tid; j < n_win; j += kExpandThreads) out[sink_end + j] = static_cast<int32_t>(wstart + j);
  int32_t* lr = out + sink_end + n_win;
  const int32_t* pk = picked + static_cast<int64_t>(t) * top_p;
  int base = 0;
  for (int r0 = 0; r0 < top_p && base < budget; r0 += kExpandThreads * kExpandItems) {
    int o[kExpandItems], lo[kExpandItems], sz[kExpandItems];
    int mine = 0;
#pragma unroll
    for (int i = 0; i < kExpandItems; ++i) {
      const int j = r0 + tid * kExpandItems + i;
      const int32_t pb = (j < top_p) ? pk[j] : -1;
      o[i] = 0, lo[i] = 0, sz[i] = 0;
      if (pb >= 0 && pb < P) {
        o[i] = off[pb];
        const int n = max(0, off[pb + 1] - o[i]);
        // members below the sinks' end / before the window; members are
        // ascending, so a bucket whose first member clears the sinks and whose
        // last precedes the window (every bucket outside block 0) needs no search
        if (n > 0) {
          const int32_t first = mem[o[i]], last = mem[o[i] + n - 1];
          lo[i] = (first >= n_sink) ? 0 : lower_bound_i32(mem + o[i], n, n_sink);
          // (a bucket of the query's own block 0 can put the window's start
          // below the sinks' end: nothing of it is kept then)
          sz[i] = max(0, ((last < wstart) ? n : lower_bound_i32(mem + o[i], n, wstart)) - lo[i]);
        }
      }
      mine += sz[i];
    }
    // exclusive scan of the per-thread counts across the block
    int incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) warp_sum[wid] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kExpandThreads / 32; ++w) {
      const int v = warp_sum[w];
      before += (w < wid) ? v : 0;
      total += v;
    }
    int start = before + incl - mine;
#pragma unroll
    for (int i = 0; i < kExpandItems; ++i) {
      s_start[tid * kExpandItems + i] = start;
      s_src[tid * kExpandItems + i] = o[i] + lo[i];
      start += sz[i];
    }
    if (tid == 0) {
      round_total = total;
      s_start[kItems] = total;
    }
    __syncthreads();
    // the round's members, block-wide: output q comes from the last bucket
    // whose start is <= q (empty buckets share their successor's start)
    const int take = min(total, budget - base);
    for (int q = tid; q < take; q += kExpandThreads) {
      int a = 0, b = kItems;                          // s_start[a] <= q < s_start[b]
      while (b - a > 1) {
        const int mid = (a + b) >> 1;
        if (s_start[mid] <= q) a = mid;
        else b = mid;
      }
      lr[base + q] = mem[s_src[a] + (q - s_start[a])];
    }
    __syncthreads();                                   // the tables are reused by the next round
    base += round_total;
  }
  const int n_lr = base < budget ? base : budget;
  const int used = static_cast<int>(sink_end) + n_win + n_lr;
  for (int j = used + tid; j < row_len; j += kExpandThreads) out[j] = -1;
  if (tid == 0) n_out[t] = used;
}

cudaError_t launch_lsa_visible(const int64_t* q_pos, int T, int block_keys, int bpb, int P, int stride, int32_t* vis,
                               int32_t* n_samp, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_visible_kernel<<<(T + 255) / 256, 256, 0, st>>>(q_pos, T, block_keys, bpb, P, stride, vis, n_samp);
  return cudaGetLastError();
}

cudaError_t launch_lsa_compact(const uint2* slist, const uint32_t* cnt, const DotParams& fp, int grid,
                               const int32_t* vis, int T, int top_p, int cap, float* cval, int32_t* clab, int32_t* nv,
                               int32_t* row_over, int* any_over, cudaStream_t st) {
  if (T == 0 || grid == 0) return cudaSuccess;
  if (4 * fp.nseg > 1024) return cudaErrorInvalidValue;
  const int NT = (fp.P + DotCfg::BM - 1) / DotCfg::BM;
  const long long units = static_cast<long long>((T + DotCfg::QB - 1) / DotCfg::QB) * NT;
  lsa_compact_kernel<<<T, 256, 0, st>>>(slist, cnt, fp.ld_cand, fp.nseg, fp.cap2, fp.slack, grid, NT, units, vis,
                                        top_p, cap, cval, clab, nv, row_over, any_over);
  return cudaGetLastError();
}

cudaError_t launch_lsa_flag_list(const int32_t* row_over, int T, int rows, int n_chunks, int32_t* list,
                                 int32_t* count, int32_t* run, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_flag_list_kernel<<<1, 1024, 0, st>>>(row_over, T, rows, n_chunks, list, count, run);
  return cudaGetLastError();
}

cudaError_t launch_lsa_gather_rows(const int32_t* list, const int32_t* count, int T, const uint16_t* q,
                                   const int32_t* vis, const int* run_if, uint16_t* qbuf, int32_t* vbuf,
                                   cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_gather_rows_kernel<<<(T * 8 + 255) / 256, 256, 0, st>>>(list, count, T, q, vis, run_if, qbuf, vbuf);
  return cudaGetLastError();
}

cudaError_t launch_lsa_expand(const int32_t* picked, const int64_t* q_pos, int T, int top_p, const int32_t* off,
                              const int32_t* mem, int P, int block_keys, int n_sink, int budget, int32_t* keys_out,
                              int row_len, int32_t* n_out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_expand_kernel<<<T, kExpandThreads, 0, st>>>(picked, q_pos, T, top_p, off, mem, P, block_keys, n_sink, budget,
                                                  keys_out, row_len, n_out);
  return cudaGetLastError();
}

}  // namespace lsi

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
  // filter form, per epilogue warp: each column's ballot and list base (64 x
  // 2 words) and each lane's listed (score, column) pairs (LIST per lane)
  static constexpr int LIST = 16;
  static constexpr size_t SMEM_COL = 64 * 2 * 4;
  static constexpr size_t SMEM_LST = 32 * LIST * 8;
  static constexpr size_t SMEM_F = size_t(EPI_WARPS) * (SMEM_COL + SMEM_LST);
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
  const int T = p.T, P = p.P;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    // filter form: lane l holds the threshold and visible count of the warp's
    // queries t0 + l and t0 + 32 + l (reloaded when the group changes; a query
    // past the end sees nothing), vis_min the smallest of the 64 counts
    float thr_a = 0.f, thr_b = 0.f;
    int vis_a = 0, vis_b = 0, vis_min = 0;
    UnitPos up;
    up.init(u_begin, NT, G);
    for (long long u = u_begin; u < u_end; ++u, up.next(NT, G)) {
      const int pc = up.tile * C::BM + quad * 32 + lane;     // this thread's centroid
      const int t0 = up.g * C::QB + cset * C::COLS_PER_WARP;
      if (FILTER && (u == u_begin || up.tile == 0)) {
        const int ta = t0 + lane, tb = t0 + 32 + lane;
        thr_a = (ta < T) ? p.tau[static_cast<int64_t>(ta) * p.ld_tau] : 0.f;
        thr_b = (tb < T) ? p.tau[static_cast<int64_t>(tb) * p.ld_tau] : 0.f;
        vis_a = (ta < T) ? p.vis[ta] : 0;
        vis_b = (tb < T) ? p.vis[tb] : 0;
        vis_min = min(vis_a, vis_b);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) vis_min = min(vis_min, __shfl_xor_sync(0xffffffffu, vis_min, d));
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
        // Pass 1: one ballot per query column (lane j keeps the ballots of
        // columns j and 32 + j); each lane notes its listed (score, column)
        // pairs in shared memory.  Pass 2: every lane reserves its two
        // columns' slots with one atomic each, all in flight together, and
        // publishes ballot and base.  Pass 3: each lane writes its own pairs.
        uint32_t* scol = reinterpret_cast<uint32_t*>(sfilt + (warp - 2) * (C::SMEM_COL + C::SMEM_LST));
        uint2* slst = reinterpret_cast<uint2*>(sfilt + (warp - 2) * (C::SMEM_COL + C::SMEM_LST) + C::SMEM_COL) +
                      lane * C::LIST;
        uint32_t bal_a = 0, bal_b = 0;
        int nl = 0;                                     // this lane's listed pairs
        // one 32-column half at a time, so only 32 scores are live in registers.
        // Listed: visible and score >= threshold (as floats: -0 equals +0, a
        // NaN is never listed, a -inf threshold lists every visible bucket).
        // A tile below every column's visible count skips the per-column count.
        const bool all_visible = up.tile * C::BM + C::BM <= vis_min;
        uint32_t v[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_ld_32x32_nowait(col + 32 * h, v);
          tmem_wait_ld(v);
          if (h == 1) release();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float thr = __shfl_sync(0xffffffffu, h ? thr_b : thr_a, j);
            const uint32_t sv = v[j];
            bool take = __uint_as_float(sv) >= thr;
            if (!all_visible) {                          // warp-uniform: every lane takes part in the shuffle
              const int vis = __shfl_sync(0xffffffffu, h ? vis_b : vis_a, j);
              take = take && (pc < vis);
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, take);
            if (lane == j) {
              if (h) bal_b = bal;
              else bal_a = bal;
            }
            if (take) {
              if (nl < C::LIST) slst[nl] = make_uint2(sv, static_cast<uint32_t>(32 * h + j));
              ++nl;
            }
          }
        }
        uint32_t base_a = 0, base_b = 0;
        // each CTA appends to its own segment of a row's list (few atomics per address)
        if (bal_a)
          base_a = atomicAdd(p.cand_cnt + static_cast<int64_t>(t0 + lane) * p.nseg + blockIdx.x,
                             static_cast<uint32_t>(__popc(bal_a)));
        if (bal_b)
          base_b = atomicAdd(p.cand_cnt + static_cast<int64_t>(t0 + 32 + lane) * p.nseg + blockIdx.x,
                             static_cast<uint32_t>(__popc(bal_b)));
        scol[lane] = bal_a;
        scol[32 + lane] = bal_b;
        scol[64 + lane] = base_a;
        scol[96 + lane] = base_b;
        __syncwarp();
        const uint32_t below = (1u << lane) - 1u;
        for (int e = 0; e < nl && e < C::LIST; ++e) {
          const uint2 pr = slst[e];
          const int c = static_cast<int>(pr.y);
          const int t = t0 + c;
          const uint32_t slot = scol[64 + c] + static_cast<uint32_t>(__popc(scol[c] & below));
          if (slot < static_cast<uint32_t>(p.seg)) {
            const int64_t at = (static_cast<int64_t>(t) * p.nseg + blockIdx.x) * p.seg + slot;
            p.cand_val[at] = __uint_as_float(pr.x);
            p.cand_lab[at] = pc;
          } else {
            p.row_over[t] = 1;
            *p.any_over = 1;
          }
        }
        if (nl > C::LIST) {
          // more listed pairs than the lane's buffer holds: rescan for the
          // columns it could not note and send those rows to the fallback
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = 32 * h + j;
              if (((h ? scol[32 + j] : scol[j]) >> lane) & 1u) {
                bool noted = false;
                for (int e = 0; e < C::LIST; ++e) noted |= (static_cast<int>(slst[e].y) == c);
                if (!noted) {
                  p.row_over[t0 + c] = 1;
                  *p.any_over = 1;
                }
              }
            }
          }
        }
        __syncwarp();                                   // the warp's shared area is reused next unit
      }
    }
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
  if (FILTER && grid > p.nseg) return cudaErrorInvalidValue;   // one list segment per CTA
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

// Visible buckets of each query (causal block visibility: the buckets of the
// complete blocks before the query's own block) and the LSA read list
// ("Latent Sparse Attention", section "The method, term by term", steps 5-6):
//   row t of keys_out: the sinks below the window, then the window
//   [block_start(t), t], then the long-range keys of the picked buckets read
//   best first, members that fall in the sinks or the window skipped, until
//   `budget` are held (the last bucket cut short); -1 after the end; n_out[t]
//   the row's length.  Bucket members are stored in ascending position order.
// Sample scores for the thresholds: row t scores the buckets 0, stride,
// 2*stride, ... below its visible count (the same positions for every row, so
// the sampled centroids stay in L2): ss[t][i] = q[t] . c[i * stride].
__global__ void lsa_sample_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ c, int T, int n_samp,
                                  int stride, float* __restrict__ ss) {
  const int t = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  __shared__ float qs[kLsaDim];
  if (threadIdx.x < kLsaDim) qs[threadIdx.x] = __uint_as_float(static_cast<uint32_t>(q[t * kLsaDim + threadIdx.x]) << 16);
  __syncthreads();
  if (i >= n_samp) return;
  const uint4* row = reinterpret_cast<const uint4*>(c + static_cast<int64_t>(i) * stride * kLsaDim);
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < kLsaDim / 8; ++v) {
    const uint4 x = __ldg(row + v);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(w[e] << 16), qs[8 * v + 2 * e], acc);
      acc = fmaf(__uint_as_float(w[e] & 0xffff0000u), qs[8 * v + 2 * e + 1], acc);
    }
  }
  ss[static_cast<int64_t>(t) * n_samp + i] = acc;
}

// After the filtered scan, one CTA per row: the row's per-CTA segments are
// packed into one list of up to `cap` entries (nv[t] of them).  A row falls
// back to full scoring when a segment ran over (flagged in the scan), the
// list would exceed cap, or it holds fewer than min(top_p, visible) buckets.
__global__ void __launch_bounds__(256)
    lsa_compact_kernel(const float* __restrict__ sval, const int32_t* __restrict__ slab,
                       const uint32_t* __restrict__ cnt, int nseg, int seg, const int32_t* __restrict__ vis, int top_p,
                       int cap, float* __restrict__ cval, int32_t* __restrict__ clab, int32_t* __restrict__ nv,
                       int32_t* __restrict__ row_over, int* __restrict__ any_over) {
  __shared__ int offs[1025];
  __shared__ int wsum[8];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  // exclusive scan of the segment counts (nseg <= 1024: 4 per thread)
  int c4[4];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = tid * 4 + i;
    c4[i] = (c < nseg) ? static_cast<int>(min(cnt[static_cast<int64_t>(t) * nseg + c], static_cast<uint32_t>(seg))) : 0;
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
    const int c = tid * 4 + i;
    if (c < nseg) offs[c] = run;
    run += c4[i];
  }
  if (tid == 255) offs[nseg] = run;
  __syncthreads();
  const int total = offs[nseg];
  const int need = min(top_p, vis[t]);
  if (tid == 0) {
    nv[t] = min(total, cap);
    if (total > cap || total < need) {
      row_over[t] = 1;
      *any_over = 1;
    }
  }
  if (total > cap) return;
  // output entry o comes from the segment c with offs[c] <= o < offs[c + 1]
  for (int o = tid; o < total; o += 256) {
    int lo = 0, hi = nseg;                      // offs[lo] <= o < offs[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs[mid] <= o) lo = mid;
      else hi = mid;
    }
    const int64_t src = (static_cast<int64_t>(t) * nseg + lo) * seg + (o - offs[lo]);
    cval[static_cast<int64_t>(t) * cap + o] = sval[src];
    clab[static_cast<int64_t>(t) * cap + o] = slab[src];
  }
}

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
// member counts scanned across the block, and each thread copies its own
// buckets' members to their offsets.
constexpr int kExpandThreads = 256;
constexpr int kExpandItems = 4;

__global__ void __launch_bounds__(kExpandThreads)
    lsa_expand_kernel(const int32_t* __restrict__ picked, const int64_t* __restrict__ q_pos, int T, int top_p,
                      const int32_t* __restrict__ off, const int32_t* __restrict__ mem, int P, int block_keys,
                      int n_sink, int budget, int32_t* __restrict__ keys_out, int row_len,
                      int32_t* __restrict__ n_out) {
  __shared__ int warp_sum[kExpandThreads / 32];
  __shared__ int round_total;
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
          sz[i] = ((last < wstart) ? n : lower_bound_i32(mem + o[i], n, wstart)) - lo[i];
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
    int start = base + before + incl - mine;
#pragma unroll
    for (int i = 0; i < kExpandItems; ++i) {
      for (int m = 0; m < sz[i] && start + m < budget; ++m) lr[start + m] = mem[o[i] + lo[i] + m];
      start += sz[i];
    }
    if (tid == 0) round_total = total;
    __syncthreads();                                   // warp_sum is reused by the next round
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

cudaError_t launch_lsa_sample(const uint16_t* q, const uint16_t* c, int T, int n_samp, int stride, float* ss,
                              cudaStream_t st) {
  if (T == 0 || n_samp == 0) return cudaSuccess;
  lsa_sample_kernel<<<dim3((n_samp + 255) / 256, T), 256, 0, st>>>(q, c, T, n_samp, stride, ss);
  return cudaGetLastError();
}

cudaError_t launch_lsa_compact(const float* sval, const int32_t* slab, const uint32_t* cnt, int nseg, int seg,
                               const int32_t* vis, int T, int top_p, int cap, float* cval, int32_t* clab, int32_t* nv,
                               int32_t* row_over, int* any_over, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (nseg > 1024) return cudaErrorInvalidValue;
  lsa_compact_kernel<<<T, 256, 0, st>>>(sval, slab, cnt, nseg, seg, vis, top_p, cap, cval, clab, nv, row_over,
                                        any_over);
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

// Sparse main attention on the tensor cores (tcgen05): the same operation as
// sparse_attn.cuh -- stage 2 of DSA ("03 long context", section "The
// Architectural Answer: Read Less of the Past") in the absorbed MLA form
// ("Derivation 6": one 576-element latent row is every head's key, its first
// 512 elements the value) -- for groups of 128 heads and at most 512 selected
// slots per query, the indexer's k.
//
// Per query the work is two dense contractions: logits S = Q . C^T (128 heads
// x 576 by 576 x k) and the output O = P . V (128 x k by k x 512).  One CTA
// per (query, 128-head group, half of the value columns): both CTAs of a
// query compute S; each keeps 256 output columns (the fp32 output of all 512
// columns is 128 lanes x 512 columns, the whole tensor memory).
//
//  1. S is accumulated over the 9 panels of 64 elements of the 576: for panel
//     p a stage holds the query's 128 x 64 panel (16 KB, by TMA) and panel p
//     of every selected row (up to 512 x 128 B, gathered by 128 threads with
//     16-byte cp.async copies straight into the 128-byte-swizzled layout; each
//     thread fences its landed copies for the tensor core's proxy before it
//     arrives), two stages in flight; per 16-element step one or two MMAs
//     (M = 128 heads, N = up to 256 rows) add into S, tensor-memory columns
//     [0, 512);
//  2. (the gather threads then fetch the value rows for step 4);
//  3. 128 threads, one per head (TMEM lane), read their S row: the row max
//     over the valid slots, then p = exp(scale * s - max), the exact fp32 sum
//     l, and p rounded to bf16, packed two per column into columns
//     [0, k / 2) (each thread rewrites only S values it has already read);
//  4. the rows are gathered again, 64 rows x this CTA's 4 value panels per
//     chunk, four chunks in flight, and O (columns [256, 512)) accumulates
//     P . V with P as the
//     tensor-memory A operand and V read as an MN-major B operand from the
//     same swizzled staging (a K-major SW128 panel of rows is, byte for byte,
//     an MN-major SW128 panel of values);
//  5. each thread divides its head's 256 outputs by the sum of its rounded
//     weights (so the weights sum to 1) and stores them; lse = max + log l.
//
// Slots that are unused (-1), outside the shard, or past k read the query's
// first valid row and weigh 0 (masked before the exponential); a query with
// no valid slot writes zeros and lse = -inf.  Every wait is bounded; a wait
// that runs out raises the library fault word and the CTA drains its copies
// and MMAs before it frees tensor memory.
//
// Precision: logits and sums are fp32 over exact bf16 products; the weights
// enter the value contraction rounded to bf16 (relative 2^-9 each), so an
// output is within 2^-8 of the largest selected value magnitude of the fp64
// result, and lse within fp32 rounding.

#pragma once

#include "common.cuh"
#include "sparse_attn.cuh"

namespace lsi {

constexpr int kTcHeads = 128;                         // heads per CTA: the MMA's M
constexpr int kTcMaxK = 512;                          // slots per query
constexpr int kTcPanels = kAttnLatent / 64;           // 9 panels of 64 elements
constexpr int kTcVPanels = kAttnValue / 2 / 64;       // 4: a CTA's half of the value columns
constexpr int kTcChunkC = 64;                         // slots per value chunk
constexpr int kTcQPanel = kTcHeads * 128;             // 16 KB: one 64-element panel of the 128 heads
constexpr int kTcStage = kTcQPanel + kTcMaxK * 128;   // 80 KB: a query panel + that panel of 512 rows
constexpr int kTcCBuf = kTcVPanels * kTcChunkC * 128; // 32 KB: 64 rows x 4 value panels
constexpr int kTcCSlots = 4;                          // value chunks in flight (inside the stages' space)
constexpr int kTcThreads = 10 * 32;                   // query loader, MMA, 4 softmax / epilogue, 4 gather warps
constexpr int kTcGather = 128;                        // gather threads (warps 6-9)
constexpr int kTcOCol = 256;                          // TMEM column of the output accumulator
static_assert(kTcCSlots * kTcCBuf <= 2 * kTcStage, "value chunks fit the stages' space");
static_assert(kTcMaxK / 2 <= kTcOCol, "the packed weights stay below the output columns");

struct AttnTcBars {
  uint64_t afull[2];    // logit stages: query panel by TMA + the gather threads' arrivals
  uint64_t aempty[2];
  uint64_t cfull[kTcCSlots];
  uint64_t cempty[kTcCSlots];
  uint64_t sfull;
  uint64_t pfull;
  uint64_t ofull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int first_slot;   // lowest valid slot (kTcMaxK: none)
  int n_valid;
  uint32_t valid[kTcMaxK / 32];   // bit s: slot s weighs
};

// Shared memory: two logit stages (the value chunks reuse their space once
// the logits are done), slot -> row ids, barriers.
constexpr size_t kTcOffIds = 2 * size_t(kTcStage);
constexpr size_t kTcOffBars = kTcOffIds + kTcMaxK * sizeof(int32_t);
constexpr size_t kTcSmem = 1024 /*align slack*/ + kTcOffBars + 256;
static_assert(sizeof(AttnTcBars) <= 256, "barrier block");
static_assert(kTcSmem <= 232448, "shared memory budget");
constexpr float kLog2e = 1.4426950408889634f;

// grid: T * (H / 128) * 2 CTAs; CTA b: value half b & 1, head group (b >> 1) % (H / 128),
// query (b >> 1) / (H / 128).  qmap: the query rows [T * H][576] bf16, box 64 x 128, with
// the 128-byte swizzle; latent: the rows [n_rows][576] bf16, 16-byte aligned.
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const uint16_t* __restrict__ latent,
                          const int32_t* __restrict__ idx, const int64_t* __restrict__ row_off, int H, int k,
                          int64_t n_rows, float scale, int foreign_ok, float* __restrict__ out,
                          float* __restrict__ lse) {
  extern __shared__ uint8_t attn_tc_raw[];
  uint8_t* smem = smem_align1024(attn_tc_raw);
  int32_t* ids = reinterpret_cast<int32_t*>(smem + kTcOffIds);
  AttnTcBars* bars = reinterpret_cast<AttnTcBars*>(smem + kTcOffBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int HG = H / kTcHeads;
  const int vh = blockIdx.x & 1;
  const int grp = blockIdx.x >> 1;
  const int hg = grp % HG;
  const int t = grp / HG;
  const int h0 = hg * kTcHeads;
  // rows staged per logit panel (a multiple of 16: the MMAs' N), and value chunks
  const int R = (k > kTcMaxK / 2) ? kTcMaxK : ((k + 15) & ~15);
  const int NS = R < kTcMaxK / 2 ? R : kTcMaxK / 2;   // N of one logit MMA
  const int nC = (k + kTcChunkC - 1) / kTcChunkC;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->afull[b], 1 + kTcGather);
      mbar_init(&bars->aempty[b], 1);
    }
    for (int b = 0; b < kTcCSlots; ++b) {
      mbar_init(&bars->cfull[b], kTcGather);
      mbar_init(&bars->cempty[b], 1);
    }
    mbar_init(&bars->sfull, 1);
    mbar_init(&bars->pfull, 4);
    mbar_init(&bars->ofull, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    bars->first_slot = kTcMaxK;
    bars->n_valid = 0;
    for (int i = 0; i < kTcMaxK / 32; ++i) bars->valid[i] = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&qmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  // slot -> latent row (-1: weighs nothing), by the 128 softmax threads
  if (warp >= 2 && warp < 6) {
    const int64_t off = row_off ? __ldg(row_off + t) : 0;
    for (int s = threadIdx.x - 64; s < kTcMaxK; s += 128) {
      int32_t id = -1;
      if (s < k) {
        const int32_t v = __ldg(idx + static_cast<int64_t>(t) * k + s);
        if (v >= 0) {
          const int64_t r = off + v;
          if (r >= 0 && r < n_rows) {
            id = static_cast<int32_t>(r);
          } else if (!foreign_ok) {
            atomicOr(&g_fault, FAULT_BAD_INDEX);       // never read: the slot weighs nothing
          }
        }
      }
      ids[s] = id;
      if (id >= 0) {
        atomicMin(&bars->first_slot, s);
        atomicAdd(&bars->n_valid, 1);
        atomicOr(&bars->valid[s >> 5], 1u << (s & 31));
      }
    }
  }
  __syncthreads();
  const int n_valid = bars->n_valid;
  const int32_t fallback = n_valid > 0 ? ids[bars->first_slot] : 0;

  if (n_valid > 0 && warp == 0) {
    // ------------------------------------------------------------ query panels
    if (lane == 0) {
      const int qrow = t * H + h0;
      bool ok = true;
      for (int pnl = 0; pnl < kTcPanels && ok; ++pnl) {
        const int st = pnl & 1;
        const uint32_t ph = (pnl >> 1) & 1;
        if (!mbar_wait(&bars->aempty[st], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->afull[st], kTcQPanel);
        tma_load_2d(smem + st * kTcStage, &qmap, &bars->afull[st], 64 * pnl, qrow);
      }
    }
  } else if (n_valid > 0 && warp >= 6) {
    // ------------------------------------------------------------ row gather
    // Each item's copies are one cp.async group, completed (waited, fenced for
    // the async proxy, arrived) after the next item's copies are issued.
    const int g = threadIdx.x - 6 * 32;                // 0 .. 127
    bool ok = true;
    for (int pnl = 0; pnl < kTcPanels && ok; ++pnl) {
      const int st = pnl & 1;
      const uint32_t ph = (pnl >> 1) & 1;
      // one lane per warp waits (128 spinning threads would crowd shared memory)
      if (!warp_wait(&bars->aempty[st], ph ^ 1, abort_flag)) { ok = false; break; }
      uint8_t* rows = smem + st * kTcStage + kTcQPanel;
      for (int e = g; e < R * 8; e += kTcGather) {     // R rows x 8 16-byte pieces of panel pnl
        const int row = e >> 3, c16 = e & 7;
        const int32_t id = ids[row] >= 0 ? ids[row] : fallback;
        cp_async_16(rows + row * 128 + ((c16 ^ (row & 7)) << 4),
                    latent + static_cast<int64_t>(id) * kAttnLatent + pnl * 64 + c16 * 8);
      }
      cp_async_commit();
      if (pnl > 0) {
        cp_async_wait_group<1>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->afull[st ^ 1]);
      }
    }
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    if (ok) mbar_arrive(&bars->afull[(kTcPanels - 1) & 1]);
    // the value rows, once the logit stages are free
    if (ok) ok = warp_wait(&bars->sfull, 0, abort_flag);
    for (int c = 0; c < nC && ok; ++c) {
      const int st = c % kTcCSlots;
      const uint32_t ph = (c / kTcCSlots) & 1;
      if (!warp_wait(&bars->cempty[st], ph ^ 1, abort_flag)) { ok = false; break; }
      uint8_t* buf = smem + st * kTcCBuf;
      for (int e = g; e < kTcChunkC * 32; e += kTcGather) {  // 64 rows x this CTA's 4 value panels x 8
        const int row = e >> 5, j = e & 31;
        const int pnl = j >> 3, c16 = j & 7;
        const int sl = kTcChunkC * c + row;
        const int32_t id = ids[sl] >= 0 ? ids[sl] : fallback;
        cp_async_16(buf + pnl * (kTcChunkC * 128) + row * 128 + ((c16 ^ (row & 7)) << 4),
                    latent + static_cast<int64_t>(id) * kAttnLatent + (kTcVPanels * vh + pnl) * 64 + c16 * 8);
      }
      cp_async_commit();
      if (c > 0) {
        cp_async_wait_group<1>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->cfull[(c - 1) % kTcCSlots]);
      }
    }
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    if (ok) mbar_arrive(&bars->cfull[(nC - 1) % kTcCSlots]);
  } else if (n_valid > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = idesc_bf16_f32(kTcHeads, NS);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kTcHeads, kTcVPanels * 64) | (1u << 16);  // B MN-major
    const uint32_t base = smem_u32(smem);
    bool ok = true;
    for (int pnl = 0; pnl < kTcPanels && ok; ++pnl) {
      const int st = pnl & 1;
      const uint32_t ph = (pnl >> 1) & 1;
      if (!warp_wait(&bars->afull[st], ph, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t qa = base + st * kTcStage, ra = qa + kTcQPanel;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adesc = sw128_kmajor_desc(qa + kk * 32);
        for (int h = 0; h * NS < R; ++h) {
          const uint64_t bdesc = sw128_kmajor_desc(ra + h * (NS * 128) + kk * 32);
          umma_f16_warp(tmem_base + h * NS, adesc, bdesc, idesc_s, (pnl | kk) ? 1u : 0u);
        }
      }
      umma_commit_warp(&bars->aempty[st]);
    }
    if (ok) umma_commit_warp(&bars->sfull);
    if (ok) ok = warp_wait(&bars->pfull, 0, abort_flag);
    tc_fence_after();
    for (int c = 0; c < nC && ok; ++c) {
      const int st = c % kTcCSlots;
      const uint32_t ph = (c / kTcCSlots) & 1;
      if (!warp_wait(&bars->cfull[st], ph, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t bb = base + st * kTcCBuf;
#pragma unroll
      for (int s = 0; s < kTcChunkC / 16; ++s) {
        // 16 rows = two 8-row atoms along K; the 4 value panels 64 rows x 128 B apart along N
        const uint64_t bdesc = sw128_mnmajor_desc(bb + s * 2048, kTcChunkC * 128);
        const uint32_t a_tmem = tmem_base + (kTcChunkC * c + 16 * s) / 2;
        umma_f16_tmem_a_warp(tmem_base + kTcOCol, a_tmem, bdesc, idesc_o, (c | s) ? 1u : 0u);
      }
      umma_commit_warp(&bars->cempty[st]);
    }
    if (ok) umma_commit_warp(&bars->ofull);
    // all MMAs this warp started are complete once `drain` flips
    umma_commit_warp(&bars->drain);
    if (lane == 0) mbar_wait_drain(&bars->drain, 0);
    __syncwarp();
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int head = quad * 32 + lane;                 // TMEM lane = head of the group
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const int64_t orow = (static_cast<int64_t>(t) * H + h0 + head) * kAttnValue + kTcVPanels * 64 * vh;
    if (n_valid == 0) {
      float4* o4 = reinterpret_cast<float4*>(out + orow);
      for (int j = 0; j < kTcVPanels * 16; ++j) o4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (vh == 0 && lse) lse[static_cast<int64_t>(t) * H + h0 + head] = neg_inf();
    } else if (warp_wait(&bars->sfull, 0, abort_flag)) {
      tc_fence_after();
      // pass 1: the row max of the logits (in log2 units) over the valid slots
      const float sl2 = scale * kLog2e;
      float m = neg_inf();
      for (int c = 0; c * 32 < R; ++c) {
        uint32_t v[32];
        tmem_ld_32x32_nowait(trow + 32 * c, v);
        const uint32_t mb = bars->valid[c];            // slots >= k are never valid
        tmem_wait_ld(v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if ((mb >> j) & 1u) m = fmaxf(m, sl2 * __uint_as_float(v[j]));
      }
      // pass 2: weights, their exact sum, and the bf16 weights packed in place
      float lp[4] = {0.f, 0.f, 0.f, 0.f}, ltp[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
      for (int c = 0; c < nC; ++c) {
        uint32_t va[32], vb[32], pw[32];
        tmem_ld_32x32_nowait(trow + kTcChunkC * c, va);
        tmem_ld_32x32_nowait(trow + kTcChunkC * c + 32, vb);
        const uint32_t ma = bars->valid[2 * c], mbb = bars->valid[2 * c + 1];
        tmem_wait_ld(va);
        tmem_wait_ld(vb);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint32_t x0 = e < 16 ? va[2 * e] : vb[2 * e - 32];
          const uint32_t x1 = e < 16 ? va[2 * e + 1] : vb[2 * e - 31];
          const uint32_t w = e < 16 ? ma : mbb;
          const int bit = (2 * e) & 31;
          const float p0 = ((w >> bit) & 1u) ? exp2f(fmaf(sl2, __uint_as_float(x0), -m)) : 0.f;
          const float p1 = ((w >> (bit + 1)) & 1u) ? exp2f(fmaf(sl2, __uint_as_float(x1), -m)) : 0.f;
          lp[e & 3] += p0 + p1;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          ltp[e & 3] += __bfloat162float(pb.x) + __bfloat162float(pb.y);
          pw[e] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        tmem_st_32x32(trow + (kTcChunkC / 2) * c, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pfull);
      const float l = (lp[0] + lp[1]) + (lp[2] + lp[3]);
      const float lt = (ltp[0] + ltp[1]) + (ltp[2] + ltp[3]);
      if (warp_wait(&bars->ofull, 0, abort_flag)) {
        tc_fence_after();
        const float inv = 1.f / lt;                    // lt >= the largest weight, 1, rounded
        float4* o4 = reinterpret_cast<float4*>(out + orow);
        for (int j = 0; j < kTcVPanels * 2; ++j) {
          uint32_t v[32];
          tmem_ld_32x32_nowait(trow + kTcOCol + 32 * j, v);
          tmem_wait_ld(v);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            o4[8 * j + e] = make_float4(__uint_as_float(v[4 * e]) * inv, __uint_as_float(v[4 * e + 1]) * inv,
                                        __uint_as_float(v[4 * e + 2]) * inv, __uint_as_float(v[4 * e + 3]) * inv);
        }
        if (vh == 0 && lse) lse[static_cast<int64_t>(t) * H + h0 + head] = (m + log2f(l)) * 0.6931471805599453f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

cudaError_t launch_sparse_attn_tc(const CUtensorMap* qmap, const uint16_t* latent, const int32_t* idx,
                                  const int64_t* row_off, int T, int H, int k, int64_t n_rows, float scale,
                                  int foreign_ok, float* out, float* lse, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  static std::atomic<uint64_t> attr_done{0};
  {
    const cudaError_t e =
        smem_limit_once(attr_done, reinterpret_cast<const void*>(&sparse_attn_tc_kernel), kTcSmem);
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = static_cast<int64_t>(T) * (H / kTcHeads) * 2;
  sparse_attn_tc_kernel<<<static_cast<unsigned>(blocks), kTcThreads, kTcSmem, st>>>(
      *qmap, latent, idx, row_off, H, k, n_rows, scale, foreign_ok, out, lse);
  return cudaGetLastError();
}

}  // namespace lsi

// Sparse main attention over the selected latent rows: stage 2 of DSA ("03
// long context", section "The Architectural Answer: Read Less of the Past"),
// in the absorbed MLA form where one cached latent row of 576 bf16 elements
// (512 latent + 64 rotary; "Derivation 6" of the same lecture) is the key of
// every query head and its first 512 elements are the value.  For query t and
// head h over the selected rows S_t:
//
//   logit(s) = scale * q[t,h,:] . c[s,:],   lse = log sum_s exp(logit(s)),
//   o[t,h,:] = sum_s exp(logit(s) - lse) * c[s,:512]
//
// One CTA per (query, group of 8 heads), 256 threads, on the CUDA cores.  The
// selection streams through in chunks of 64 slots, each row gathered once
// (its first 512 elements serve as the value from the same staged copy), with
// the online-softmax recurrence per head (running max m and sum l; a chunk
// that raises m rescales what was accumulated by exp(m_old - m_new)):
//
//  1. the chunk's row ids (slot -> idx + row offset; -1 or out of range ->
//     none; out of range is flagged unless the caller holds one shard of the
//     rows), double-buffered so the next chunk's ids and rows can be fetched
//     while this one is computed;
//  2. logits: rows staged with a 289-word stride (32 consecutive rows start on
//     32 different banks); warp p takes dimensions 72p .. 72p + 71 (its query
//     loads are broadcasts) and its lane g rows g and g + 32, for all 8 heads;
//     the eight partial sums are added in a fixed order;
//  3. softmax step, warp h for head h: chunk max, new running max, rescale
//     factor, weights exp(logit - m), running sum;
//  4. values: thread i of each half of the CTA owns output columns 2i, 2i + 1,
//     256 + 2i, 257 + 2i of all 8 heads, rescales them, and adds its parity's
//     rows (the lower half the even rows, the upper half the odd ones),
//     reading a row's 8 weights as two 16-byte broadcasts; the halves' sums
//     meet in shared memory at the end.
//
// Rows are gathered a chunk ahead into registers, so the next chunk's loads
// are in flight while the current one is computed.  Unused slots stage zeros
// and weigh 0.  Shared memory does not depend on k.

#pragma once

#include "common.cuh"

namespace lsi {

constexpr int kAttnLatent = 576;                    // elements of a latent row (the key)
constexpr int kAttnValue = 512;                     // leading elements that are the value
constexpr int kAttnHeads = 8;                       // heads per CTA
constexpr int kAttnChunk = 64;                      // selected rows staged per step
constexpr int kAttnThreads = 256;
constexpr int kAttnMaxK = 1 << 16;                  // slots per query (the selection streams through)
constexpr int kAttnRowWords = kAttnLatent / 2 + 1;  // 289 words: row r starts on bank r mod 32
constexpr int kAttnParts = kAttnThreads / 32;       // dimension slices, one per warp
constexpr int kAttnSlice = kAttnLatent / kAttnParts;  // 72 dimensions per partial dot product
constexpr int kAttnHalf = kAttnThreads / 2;         // threads per half (value pass)
static_assert(kAttnValue / 2 == 2 * kAttnHalf, "two column pairs per thread of each half");
static_assert(kAttnChunk == 64, "a lane scores staged rows g and g + 32 and the softmax takes two per lane");
static_assert(kAttnSlice % 2 == 0, "slices of whole bf16 pairs");
static_assert(kAttnThreads / 32 == kAttnHeads, "one warp per head in the softmax step");
static_assert(kAttnHalf * kAttnHeads * 4 <= kAttnParts * kAttnHeads * kAttnChunk,
              "the upper half's sums fit the partial-sum buffer");

// Shared memory layout in 4-byte words, the same for every k:
//   [0, OffRows)         query heads, fp32 [d][h]
//   [OffRows, OffPart)   staged rows, 289 words each
//   [OffPart, OffW)      partial sums [slice][row][h], at the end the halves' exchange
//   [OffW, OffIds)       the chunk's logits, then its weights [row][h]
//   [OffIds, OffStat)    row ids of two chunks
//   [OffStat, Words)     rescale factors [h], then 1 / sums [h]
constexpr int kAttnOffRows = kAttnLatent * kAttnHeads;
constexpr int kAttnOffPart = kAttnOffRows + kAttnChunk * kAttnRowWords;
constexpr int kAttnOffW = kAttnOffPart + kAttnParts * kAttnChunk * kAttnHeads;
constexpr int kAttnOffIds = kAttnOffW + kAttnChunk * kAttnHeads;
constexpr int kAttnOffStat = kAttnOffIds + 2 * kAttnChunk;
constexpr int kAttnWords = kAttnOffStat + 2 * kAttnHeads;
static_assert(kAttnOffW % 4 == 0 && kAttnOffPart % 4 == 0, "float4 access to the weights and the exchange");

__host__ __device__ constexpr size_t attn_smem_bytes() { return 4 * static_cast<size_t>(kAttnWords); }

__device__ __forceinline__ float attn_bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float attn_bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// acc = a * b + acc on both fp32 halves of the pairs: two fused multiply-adds,
// each rounded once (the packed form halves the FMA instructions issued).
__device__ __forceinline__ void attn_fma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ float attn_warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float attn_warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One thread's share of a chunk of 64 rows (the whole 576-element rows), held
// in registers between the global loads and the shared-memory stores.
struct AttnChunk {
  static constexpr int kVecs = kAttnLatent / 8;                         // 16-byte loads per row
  static constexpr int kPer = kAttnChunk * kVecs / kAttnThreads;        // loads per thread
  static_assert(kAttnChunk * kVecs % kAttnThreads == 0, "whole loads per thread");
  uint4 v[kPer];
};

// Row ids of slots c0 .. c0 + 63 of query t (threads 0..63, one slot each).
__device__ __forceinline__ void attn_resolve(int32_t* ids, const int32_t* __restrict__ idx, int t, int k, int c0,
                                             int64_t off, int64_t n_rows, int foreign_ok) {
  const int i = threadIdx.x;
  if (i >= kAttnChunk) return;
  int32_t id = -1;
  if (c0 + i < k) {
    const int32_t s = idx[static_cast<int64_t>(t) * k + c0 + i];
    if (s >= 0) {
      const int64_t r = off + s;
      if (r >= 0 && r < n_rows)
        id = static_cast<int32_t>(r);
      else if (!foreign_ok)
        atomicOr(&g_fault, FAULT_BAD_INDEX);          // never read: the slot stays unused
    }
  }
  ids[i] = id;
}

// Gather the chunk's rows (an unused slot gives zeros).
__device__ __forceinline__ void attn_fetch(AttnChunk& c, const int32_t* ids, const uint16_t* __restrict__ latent) {
#pragma unroll
  for (int m = 0; m < AttnChunk::kPer; ++m) {
    const int i = threadIdx.x + m * kAttnThreads;
    const int r = i / AttnChunk::kVecs;
    const int v = i - r * AttnChunk::kVecs;
    const int32_t id = ids[r];
    c.v[m] = make_uint4(0u, 0u, 0u, 0u);
    if (id >= 0) c.v[m] = __ldg(reinterpret_cast<const uint4*>(latent + static_cast<int64_t>(id) * kAttnLatent) + v);
  }
}

// Store a fetched chunk into shared memory, a row every 289 words.
__device__ __forceinline__ void attn_put(const AttnChunk& c, uint32_t* rows) {
#pragma unroll
  for (int m = 0; m < AttnChunk::kPer; ++m) {
    const int i = threadIdx.x + m * kAttnThreads;
    const int r = i / AttnChunk::kVecs;
    const int v = i - r * AttnChunk::kVecs;
    uint32_t* dst = rows + r * kAttnRowWords + 4 * v;
    dst[0] = c.v[m].x;
    dst[1] = c.v[m].y;
    dst[2] = c.v[m].z;
    dst[3] = c.v[m].w;
  }
}

// grid: T * (H / 8) CTAs, CTA b = (query b / (H / 8), head group b % (H / 8)).
__global__ void __launch_bounds__(kAttnThreads)
    sparse_attn_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ latent,
                       const int32_t* __restrict__ idx, const int64_t* __restrict__ row_off, int H, int k,
                       int64_t n_rows, float scale, int foreign_ok, float* __restrict__ out,
                       float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char attn_smem[];
  float* qs = reinterpret_cast<float*>(attn_smem);
  uint32_t* rows = reinterpret_cast<uint32_t*>(qs + kAttnOffRows);
  float* part = qs + kAttnOffPart;
  float* wts = qs + kAttnOffW;
  int32_t* ids = reinterpret_cast<int32_t*>(qs + kAttnOffIds);
  float* stat = qs + kAttnOffStat;                    // [0, 8): rescale factors, [8, 16): 1 / sums

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int groups = H / kAttnHeads;
  const int t = blockIdx.x / groups;
  const int h0 = (blockIdx.x - t * groups) * kAttnHeads;
  const int64_t off = row_off ? row_off[t] : 0;
  const int nchunks = (k + kAttnChunk - 1) / kAttnChunk;

  const uint16_t* qt = q + (static_cast<int64_t>(t) * H + h0) * kAttnLatent;
  for (int i = tid; i < kAttnHeads * kAttnLatent; i += kAttnThreads) {
    const int hh = i / kAttnLatent;
    const int d = i - hh * kAttnLatent;
    qs[d * kAttnHeads + hh] = __uint_as_float(static_cast<uint32_t>(qt[i]) << 16);
  }
  attn_resolve(ids, idx, t, k, 0, off, n_rows, foreign_ok);
  __syncthreads();
  AttnChunk next;
  attn_fetch(next, ids, latent);

  const int g = lane;                                 // logits: staged rows g and g + 32
  const int sl = warp;                                // logits: this warp's dimension slice
  const int cg = tid & (kAttnHalf - 1);               // values: columns 2cg, 2cg + 1, 256 + 2cg, 257 + 2cg
  const int half = tid / kAttnHalf;                   // values: rows of this parity
  float m_run = -INFINITY;                            // softmax state of head `warp` (same in every lane)
  float l_run = 0.f;
  uint64_t o[kAttnHeads / 2][4];                      // head pair (2i, 2i + 1) of this thread's 4 columns
#pragma unroll
  for (int i = 0; i < kAttnHeads / 2; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0ull;

  for (int c = 0; c < nchunks; ++c) {
    const int32_t* cid = ids + (c & 1) * kAttnChunk;
    attn_put(next, rows);
    if (c + 1 < nchunks)
      attn_resolve(ids + ((c + 1) & 1) * kAttnChunk, idx, t, k, (c + 1) * kAttnChunk, off, n_rows, foreign_ok);
    __syncthreads();
    if (c + 1 < nchunks) attn_fetch(next, ids + ((c + 1) & 1) * kAttnChunk, latent);   // in flight during the math

    // 2. logits (accumulators hold the head pairs (2i, 2i + 1) of rows g and g + 32)
    {
      uint64_t a0[kAttnHeads / 2], a1[kAttnHeads / 2];
#pragma unroll
      for (int i = 0; i < kAttnHeads / 2; ++i) a0[i] = a1[i] = 0ull;
      const uint32_t* r0 = rows + g * kAttnRowWords + sl * (kAttnSlice / 2);
      const uint32_t* r1 = r0 + 32 * kAttnRowWords;
      const uint64_t* qq = reinterpret_cast<const uint64_t*>(qs + sl * kAttnSlice * kAttnHeads);
#pragma unroll 2
      for (int w = 0; w < kAttnSlice / 2; ++w) {
        const uint32_t x = r0[w];
        const uint32_t y = r1[w];
        const uint64_t x0 = pack_f32x2(attn_bf16_lo(x), attn_bf16_lo(x));
        const uint64_t x1 = pack_f32x2(attn_bf16_hi(x), attn_bf16_hi(x));
        const uint64_t y0 = pack_f32x2(attn_bf16_lo(y), attn_bf16_lo(y));
        const uint64_t y1 = pack_f32x2(attn_bf16_hi(y), attn_bf16_hi(y));
        const uint64_t* q0 = qq + w * kAttnHeads;       // dimension 2w: 4 head pairs, then dimension 2w + 1
#pragma unroll
        for (int i = 0; i < kAttnHeads / 2; ++i) {
          const uint64_t qa = q0[i];
          const uint64_t qb = q0[kAttnHeads / 2 + i];
          attn_fma2(a0[i], qa, x0);
          attn_fma2(a0[i], qb, x1);
          attn_fma2(a1[i], qa, y0);
          attn_fma2(a1[i], qb, y1);
        }
      }
      float* p0 = part + (sl * kAttnChunk + g) * kAttnHeads;
      float* p1 = p0 + 32 * kAttnHeads;
#pragma unroll
      for (int i = 0; i < kAttnHeads / 2; ++i) {
        unpack_f32x2(a0[i], p0[2 * i], p0[2 * i + 1]);
        unpack_f32x2(a1[i], p1[2 * i], p1[2 * i + 1]);
      }
    }
    __syncthreads();
    for (int i = tid; i < kAttnHeads * kAttnChunk; i += kAttnThreads) {
      const int j = i / kAttnHeads;
      const int hh = i - j * kAttnHeads;
      float s = part[j * kAttnHeads + hh];
#pragma unroll
      for (int sp = 1; sp < kAttnParts; ++sp) s += part[(sp * kAttnChunk + j) * kAttnHeads + hh];
      wts[j * kAttnHeads + hh] = cid[j] >= 0 ? s * scale : -INFINITY;
    }
    __syncthreads();

    // 3. softmax step for head `warp` (every lane takes slots lane and lane + 32)
    {
      const float x0 = wts[lane * kAttnHeads + warp];
      const float x1 = wts[(lane + 32) * kAttnHeads + warp];
      const float m_new = fmaxf(m_run, attn_warp_max(fmaxf(x0, x1)));
      const float alpha = (m_new == -INFINITY) ? 1.f : expf(m_run - m_new);   // exp(-inf) = 0 on the first rows
      const float e0 = (x0 == -INFINITY) ? 0.f : expf(x0 - m_new);
      const float e1 = (x1 == -INFINITY) ? 0.f : expf(x1 - m_new);
      wts[lane * kAttnHeads + warp] = e0;
      wts[(lane + 32) * kAttnHeads + warp] = e1;
      l_run = l_run * alpha + attn_warp_sum(e0 + e1);
      m_run = m_new;
      if (lane == 0) stat[warp] = alpha;
    }
    __syncthreads();

    // 4. values
#pragma unroll
    for (int i = 0; i < kAttnHeads / 2; ++i) {
      const float al0 = stat[2 * i];
      const float al1 = stat[2 * i + 1];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float lo, hi;
        unpack_f32x2(o[i][cc], lo, hi);
        o[i][cc] = pack_f32x2(lo * al0, hi * al1);
      }
    }
    for (int j = half; j < kAttnChunk; j += 2) {
      const uint32_t xa = rows[j * kAttnRowWords + cg];
      const uint32_t xb = rows[j * kAttnRowWords + kAttnHalf + cg];
      const uint64_t v[4] = {pack_f32x2(attn_bf16_lo(xa), attn_bf16_lo(xa)),
                             pack_f32x2(attn_bf16_hi(xa), attn_bf16_hi(xa)),
                             pack_f32x2(attn_bf16_lo(xb), attn_bf16_lo(xb)),
                             pack_f32x2(attn_bf16_hi(xb), attn_bf16_hi(xb))};
      const ulonglong2* pj = reinterpret_cast<const ulonglong2*>(wts + j * kAttnHeads);   // 32-byte aligned
      const ulonglong2 pa = pj[0];                    // head pairs (0, 1) and (2, 3)
      const ulonglong2 pb = pj[1];                    // head pairs (4, 5) and (6, 7)
      const uint64_t p[kAttnHeads / 2] = {pa.x, pa.y, pb.x, pb.y};
#pragma unroll
      for (int i = 0; i < kAttnHeads / 2; ++i) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) attn_fma2(o[i][cc], p[i], v[cc]);
      }
    }
    __syncthreads();                                  // rows, weights and factors are rewritten next chunk
  }

  if (lane == 0) {
    stat[kAttnHeads + warp] = l_run > 0.f ? 1.f / l_run : 0.f;
    if (lse) lse[static_cast<int64_t>(t) * H + h0 + warp] = l_run > 0.f ? m_run + logf(l_run) : -INFINITY;
  }
  // the upper half's sums go through shared memory (the partial-sum buffer is free) to the lower half
  float oh[kAttnHeads][4];                            // the pairs split per head
#pragma unroll
  for (int i = 0; i < kAttnHeads / 2; ++i) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) unpack_f32x2(o[i][cc], oh[2 * i][cc], oh[2 * i + 1][cc]);
  }
  float4* xfer = reinterpret_cast<float4*>(part) + cg;   // head hh at xfer[hh * 128]
  if (half == 1) {
#pragma unroll
    for (int hh = 0; hh < kAttnHeads; ++hh)
      xfer[hh * kAttnHalf] = make_float4(oh[hh][0], oh[hh][1], oh[hh][2], oh[hh][3]);
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int hh = 0; hh < kAttnHeads; ++hh) {
      const float4 u = xfer[hh * kAttnHalf];
      const float il = stat[kAttnHeads + hh];
      float* dst = out + (static_cast<int64_t>(t) * H + h0 + hh) * kAttnValue;
      *reinterpret_cast<float2*>(dst + 2 * cg) = make_float2((oh[hh][0] + u.x) * il, (oh[hh][1] + u.y) * il);
      *reinterpret_cast<float2*>(dst + 2 * kAttnHalf + 2 * cg) =
          make_float2((oh[hh][2] + u.z) * il, (oh[hh][3] + u.w) * il);
    }
  }
}

cudaError_t launch_sparse_attn(const uint16_t* q, const uint16_t* latent, const int32_t* idx, const int64_t* row_off,
                               int T, int H, int k, int64_t n_rows, float scale, int foreign_ok, float* out, float* lse,
                               cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const size_t smem = attn_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t blocks = static_cast<int64_t>(T) * (H / kAttnHeads);
  sparse_attn_kernel<<<static_cast<unsigned>(blocks), kAttnThreads, smem, st>>>(q, latent, idx, row_off, H, k, n_rows,
                                                                                  scale, foreign_ok, out, lse);
  return cudaGetLastError();
}

// Combine of S partial attentions of the same queries over disjoint row sets
// (the online-softmax rule): with m = max_s lse_s and w_s = exp(lse_s - m),
// o = sum_s w_s o_s / sum_s w_s and lse = m + log sum_s w_s.  One thread per
// (query, head, pair of output columns); a part with lse = -inf weighs 0, and
// all parts empty give o = 0, lse = -inf.
__global__ void __launch_bounds__(256)
    attn_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int S, int64_t rows,
                      int d_v, float* __restrict__ o, float* __restrict__ lse) {
  const int pairs = d_v / 2;
  const int64_t n = rows * pairs;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / pairs;
    const int c = static_cast<int>(i - r * pairs) * 2;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, lse_parts[s * rows + r]);
    float den = 0.f, a0 = 0.f, a1 = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float ls = lse_parts[s * rows + r];
        if (ls == -INFINITY) continue;
        const float w = expf(ls - m);
        const float2 v = *reinterpret_cast<const float2*>(o_parts + (s * rows + r) * d_v + c);
        den += w;
        a0 = fmaf(w, v.x, a0);
        a1 = fmaf(w, v.y, a1);
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    *reinterpret_cast<float2*>(o + r * d_v + c) = make_float2(a0 * inv, a1 * inv);
    if (c == 0 && lse) lse[r] = den > 0.f ? m + logf(den) : -INFINITY;
  }
}

cudaError_t launch_attn_merge(const float* o_parts, const float* lse_parts, int S, int64_t rows, int d_v, float* o,
                              float* lse, int num_sms, cudaStream_t st) {
  const int64_t n = rows * (d_v / 2);
  if (n == 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256;
  const int blocks = static_cast<int>(want < 8LL * num_sms ? want : 8LL * num_sms);
  attn_merge_kernel<<<blocks, 256, 0, st>>>(o_parts, lse_parts, S, rows, d_v, o, lse);
  return cudaGetLastError();
}

}  // namespace lsi

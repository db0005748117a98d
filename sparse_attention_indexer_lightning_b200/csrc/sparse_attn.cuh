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
// One CTA per (query, group of 8 heads), 256 threads, on the CUDA cores:
//
//  1. the CTA's row ids (slot -> idx + row offset; -1 or out of range -> none;
//     out of range is flagged unless the caller holds one shard of the rows)
//     and its 8 query heads (fp32, [dimension][head]) go to shared memory;
//  2. logits: the selected rows are staged 64 at a time (a row per 289-word
//     stride, so 32 consecutive rows start on 32 different banks); warp p
//     takes dimensions 72p .. 72p + 71 (its query loads are broadcasts) and
//     its lane g rows g and g + 32, for all 8 heads; the eight partial sums
//     are added in a fixed order; logits are kept slot-major ([slot][head]);
//  3. softmax: warp h takes head h: max, exp(logit - max), sum, 1 / sum, lse;
//  4. values: the value parts are staged again, 64 rows at a time, densely
//     (256 words a row); thread i of each half owns output columns 4i .. 4i + 3
//     of all 8 heads, the lower half takes the even rows and the upper half
//     the odd ones, reading a row's 8 weights as two 16-byte broadcasts; the
//     two halves' sums are added at the end.
//
// The selection sits in shared memory in full (k <= 2048 slots), so the
// softmax is exact in two passes, with no running rescale.  Unused slots
// stage zeros and weigh 0.  Rows are gathered a chunk ahead into registers
// (the next chunk's loads are in flight while the current one is computed;
// the value pass's first chunk while the softmax runs).

#pragma once

#include "common.cuh"

namespace lsi {

constexpr int kAttnLatent = 576;                    // elements of a latent row (the key)
constexpr int kAttnValue = 512;                     // leading elements that are the value
constexpr int kAttnHeads = 8;                       // heads per CTA
constexpr int kAttnChunk = 64;                      // selected rows staged per pass
constexpr int kAttnThreads = 256;
constexpr int kAttnMaxK = 2048;
constexpr int kAttnRowWords = kAttnLatent / 2 + 1;  // 289 words: row r starts on bank r mod 32
constexpr int kAttnParts = kAttnThreads / 32;      // dimension slices, one per warp
constexpr int kAttnSlice = kAttnLatent / kAttnParts;  // 72 dimensions per partial dot product
static_assert(kAttnValue / 4 == kAttnThreads / 2, "four value columns per thread of each half");
static_assert(kAttnThreads / 2 * 4 * kAttnHeads <= kAttnParts * kAttnHeads * kAttnChunk,
              "the upper half's sums fit the partial-sum buffer");
static_assert(kAttnChunk == 64, "a lane scores staged rows g and g + 32");
static_assert(kAttnSlice % 2 == 0, "slices of whole bf16 pairs");
static_assert(kAttnThreads / 32 == kAttnHeads, "one warp per head in the softmax");
static_assert((kAttnLatent * kAttnHeads + kAttnChunk * kAttnRowWords + kAttnParts * kAttnHeads * kAttnChunk) % 4 == 0,
              "the weights start on a 16-byte boundary (float4 reads)");

__host__ __device__ constexpr int attn_kpad(int k) { return (k + kAttnChunk - 1) / kAttnChunk * kAttnChunk; }

// Dynamic shared memory of one CTA for k slots (4-byte words throughout).
__host__ __device__ constexpr size_t attn_smem_bytes(int k) {
  return 4 * (static_cast<size_t>(kAttnLatent) * kAttnHeads      // query heads [d][h]
              + static_cast<size_t>(kAttnChunk) * kAttnRowWords  // staged rows
              + kAttnParts * kAttnHeads * kAttnChunk              // partial dot products [slice][row][h]
              + static_cast<size_t>(kAttnHeads) * attn_kpad(k)    // logits, then weights [slot][h]
              + attn_kpad(k)                                      // row ids [slot]
              + kAttnHeads);                                      // 1 / sum of weights [h]
}

__device__ __forceinline__ float attn_bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float attn_bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float attn_warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float attn_warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One thread's share of a chunk of 64 staged rows, `WORDS` 32-bit words
// (bf16 pairs) of each, held in registers between the global loads and the
// shared-memory stores, so that the next chunk's gather is in flight while
// the current one is computed.
template <int WORDS>
struct AttnChunk {
  static constexpr int kVecs = WORDS / 4;                               // 16-byte loads per row
  static constexpr int kPer = kAttnChunk * kVecs / kAttnThreads;        // loads per thread
  static_assert(kAttnChunk * kVecs % kAttnThreads == 0, "whole loads per thread");
  uint4 v[kPer];
};

// Gather rows of slots c0 .. c0 + 63 (an unused slot gives zeros).
template <int WORDS>
__device__ __forceinline__ void attn_fetch(AttnChunk<WORDS>& c, const int32_t* ids, int c0,
                                           const uint16_t* __restrict__ latent) {
#pragma unroll
  for (int m = 0; m < AttnChunk<WORDS>::kPer; ++m) {
    const int i = threadIdx.x + m * kAttnThreads;
    const int r = i / AttnChunk<WORDS>::kVecs;
    const int v = i - r * AttnChunk<WORDS>::kVecs;
    const int32_t id = ids[c0 + r];
    c.v[m] = make_uint4(0u, 0u, 0u, 0u);
    if (id >= 0) c.v[m] = __ldg(reinterpret_cast<const uint4*>(latent + static_cast<int64_t>(id) * kAttnLatent) + v);
  }
}

// Store a fetched chunk into shared memory, a row every `stride` words.
template <int WORDS>
__device__ __forceinline__ void attn_put(const AttnChunk<WORDS>& c, uint32_t* rows, int stride) {
#pragma unroll
  for (int m = 0; m < AttnChunk<WORDS>::kPer; ++m) {
    const int i = threadIdx.x + m * kAttnThreads;
    const int r = i / AttnChunk<WORDS>::kVecs;
    const int v = i - r * AttnChunk<WORDS>::kVecs;
    uint32_t* dst = rows + r * stride + 4 * v;
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
  const int kp = attn_kpad(k);
  float* qs = reinterpret_cast<float*>(attn_smem);
  uint32_t* rows = reinterpret_cast<uint32_t*>(qs + kAttnLatent * kAttnHeads);
  float* part = reinterpret_cast<float*>(rows + kAttnChunk * kAttnRowWords);
  float* sc = part + kAttnParts * kAttnHeads * kAttnChunk;
  int32_t* ids = reinterpret_cast<int32_t*>(sc + kAttnHeads * kp);
  float* inv_l = reinterpret_cast<float*>(ids + kp);

  const int tid = threadIdx.x;
  const int groups = H / kAttnHeads;
  const int t = blockIdx.x / groups;
  const int h0 = (blockIdx.x - t * groups) * kAttnHeads;
  const int64_t off = row_off ? row_off[t] : 0;

  // 1. row ids and query heads
  for (int i = tid; i < kp; i += kAttnThreads) {
    int32_t id = -1;
    if (i < k) {
      const int32_t s = idx[static_cast<int64_t>(t) * k + i];
      if (s >= 0) {
        const int64_t r = off + s;
        if (r >= 0 && r < n_rows)
          id = static_cast<int32_t>(r);
        else if (!foreign_ok)
          atomicOr(&g_fault, FAULT_BAD_INDEX);      // never read: the slot stays unused
      }
    }
    ids[i] = id;
  }
  const uint16_t* qt = q + (static_cast<int64_t>(t) * H + h0) * kAttnLatent;
  for (int i = tid; i < kAttnHeads * kAttnLatent; i += kAttnThreads) {
    const int hh = i / kAttnLatent;
    const int d = i - hh * kAttnLatent;
    qs[d * kAttnHeads + hh] = __uint_as_float(static_cast<uint32_t>(qt[i]) << 16);
  }
  __syncthreads();

  // 2. logits
  const int g = tid & 31;                             // staged rows g and g + 32
  const int sl = tid >> 5;                            // dimension slice of this warp
  {
    AttnChunk<kAttnLatent / 2> next;
    attn_fetch(next, ids, 0, latent);
    for (int c0 = 0; c0 < kp; c0 += kAttnChunk) {
      attn_put(next, rows, kAttnRowWords);
      __syncthreads();
      if (c0 + kAttnChunk < kp) attn_fetch(next, ids, c0 + kAttnChunk, latent);   // in flight during the math
      float a0[kAttnHeads], a1[kAttnHeads];
#pragma unroll
      for (int hh = 0; hh < kAttnHeads; ++hh) a0[hh] = a1[hh] = 0.f;
      const uint32_t* r0 = rows + g * kAttnRowWords + sl * (kAttnSlice / 2);
      const uint32_t* r1 = r0 + 32 * kAttnRowWords;
      const float* qq = qs + sl * kAttnSlice * kAttnHeads;
#pragma unroll 2
      for (int w = 0; w < kAttnSlice / 2; ++w) {
        const uint32_t x = r0[w];
        const uint32_t y = r1[w];
        const float x0 = attn_bf16_lo(x);
        const float x1 = attn_bf16_hi(x);
        const float y0 = attn_bf16_lo(y);
        const float y1 = attn_bf16_hi(y);
        const float* q0 = qq + 2 * w * kAttnHeads;
#pragma unroll
        for (int hh = 0; hh < kAttnHeads; ++hh) {
          const float qa = q0[hh];
          const float qb = q0[kAttnHeads + hh];
          a0[hh] = fmaf(x1, qb, fmaf(x0, qa, a0[hh]));
          a1[hh] = fmaf(y1, qb, fmaf(y0, qa, a1[hh]));
        }
      }
      float* p0 = part + (sl * kAttnChunk + g) * kAttnHeads;
      float* p1 = p0 + 32 * kAttnHeads;
#pragma unroll
      for (int hh = 0; hh < kAttnHeads; ++hh) {
        p0[hh] = a0[hh];
        p1[hh] = a1[hh];
      }
      __syncthreads();
      for (int i = tid; i < kAttnHeads * kAttnChunk; i += kAttnThreads) {
        const int j = i / kAttnHeads;
        const int hh = i - j * kAttnHeads;
        float s = part[j * kAttnHeads + hh];
#pragma unroll
        for (int sp = 1; sp < kAttnParts; ++sp) s += part[(sp * kAttnChunk + j) * kAttnHeads + hh];
        sc[(c0 + j) * kAttnHeads + hh] = ids[c0 + j] >= 0 ? s * scale : -INFINITY;
      }
      __syncthreads();
    }
  }

  // the value pass's first gather overlaps the softmax
  constexpr int kValWords = kAttnValue / 2;           // dense staging: row j at word 256 j (8-byte aligned)
  AttnChunk<kValWords> vnext;
  attn_fetch(vnext, ids, 0, latent);

  // 3. softmax, one warp per head (kp is a multiple of 32: every lane loops alike)
  {
    const int warp = tid >> 5;
    const int lane = tid & 31;
    float* sh = sc + warp;                          // head `warp` of slot j at sh[j * 8]
    float m = -INFINITY;
    for (int j = lane; j < kp; j += 32) m = fmaxf(m, sh[j * kAttnHeads]);
    m = attn_warp_max(m);
    float l = 0.f;
    for (int j = lane; j < kp; j += 32) {
      const float x = sh[j * kAttnHeads];
      const float e = (x == -INFINITY) ? 0.f : expf(x - m);
      sh[j * kAttnHeads] = e;
      l += e;
    }
    l = attn_warp_sum(l);
    if (lane == 0) {
      inv_l[warp] = l > 0.f ? 1.f / l : 0.f;
      if (lse) lse[static_cast<int64_t>(t) * H + h0 + warp] = l > 0.f ? m + logf(l) : -INFINITY;
    }
  }
  __syncthreads();

  // 4. values
  const int cg = tid & (kAttnThreads / 2 - 1);        // columns 4 cg .. 4 cg + 3
  const int half = tid / (kAttnThreads / 2);          // rows of this parity
  float o[kAttnHeads][4];
#pragma unroll
  for (int hh = 0; hh < kAttnHeads; ++hh) o[hh][0] = o[hh][1] = o[hh][2] = o[hh][3] = 0.f;
  for (int c0 = 0; c0 < kp; c0 += kAttnChunk) {
    attn_put(vnext, rows, kValWords);
    __syncthreads();
    if (c0 + kAttnChunk < kp) attn_fetch(vnext, ids, c0 + kAttnChunk, latent);
    for (int j = half; j < kAttnChunk; j += 2) {
      const uint2 x = *reinterpret_cast<const uint2*>(rows + j * kValWords + 2 * cg);
      const float v0 = attn_bf16_lo(x.x);
      const float v1 = attn_bf16_hi(x.x);
      const float v2 = attn_bf16_lo(x.y);
      const float v3 = attn_bf16_hi(x.y);
      const float4* pj = reinterpret_cast<const float4*>(sc + (c0 + j) * kAttnHeads);   // 32-byte aligned
      const float4 pa = pj[0];
      const float4 pb = pj[1];
      const float p[kAttnHeads] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int hh = 0; hh < kAttnHeads; ++hh) {
        o[hh][0] = fmaf(p[hh], v0, o[hh][0]);
        o[hh][1] = fmaf(p[hh], v1, o[hh][1]);
        o[hh][2] = fmaf(p[hh], v2, o[hh][2]);
        o[hh][3] = fmaf(p[hh], v3, o[hh][3]);
      }
    }
    __syncthreads();
  }
  // the odd rows' sums go through shared memory (the partial-sum buffer is free) to the even rows' threads
  float4* xfer = reinterpret_cast<float4*>(part) + cg;   // head hh at xfer[hh * 128]
  if (half == 1) {
#pragma unroll
    for (int hh = 0; hh < kAttnHeads; ++hh)
      xfer[hh * (kAttnThreads / 2)] = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int hh = 0; hh < kAttnHeads; ++hh) {
      const float4 u = xfer[hh * (kAttnThreads / 2)];
      const float il = inv_l[hh];
      float* dst = out + (static_cast<int64_t>(t) * H + h0 + hh) * kAttnValue + 4 * cg;
      *reinterpret_cast<float4*>(dst) =
          make_float4((o[hh][0] + u.x) * il, (o[hh][1] + u.y) * il, (o[hh][2] + u.z) * il, (o[hh][3] + u.w) * il);
    }
  }
}

cudaError_t launch_sparse_attn(const uint16_t* q, const uint16_t* latent, const int32_t* idx, const int64_t* row_off,
                               int T, int H, int k, int64_t n_rows, float scale, int foreign_ok, float* out, float* lse,
                               cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const size_t smem = attn_smem_bytes(k);
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

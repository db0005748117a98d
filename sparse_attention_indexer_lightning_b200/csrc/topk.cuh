// Exact row-wise top-k by (score desc, position asc).
//
// Selection order follows the packed-key radix select of "Latent Sparse
// Attention", section "What the kernels do about the top-p": the score's bits
// sit above the inverted id in one 64-bit key, so the largest keys are the
// highest scores with ties going to the lower id.  Scores are first mapped to
// an order-preserving 32-bit code (-0.0 and +0.0 share a code; NaN gets code
// 0, below -inf), so the 64-bit keys of a row are all distinct and the k-th
// largest key is a unique threshold.
//
// One CTA of 1024 threads per row:
//   1. MSB-first radix select over the 64-bit keys, 8 bits per pass, with a
//      shared-memory histogram; it stops as soon as every key sharing the
//      current prefix is wanted (normally after the 4 passes over the score
//      bits -- the id bits are only visited when scores tie at the cut).
//   2. One pass collects the keys >= threshold (exactly k of them).
//   3. Bitonic sort of the k keys in shared memory, descending, so the output
//      is in the canonical order.
// Values are written as bit copies of the input.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t order_code(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN ranks below -inf
  if (b == 0x80000000u) b = 0u;                     // -0.0 ties +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct TopkShared {
  unsigned long long key[kMaxTopK];
  uint32_t col[kMaxTopK];
  uint32_t hist[256];
  uint32_t digit, need, done, total, cnt;
};

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = p.scores + static_cast<int64_t>(r) * p.ld;
  const int32_t* lab = p.labels ? p.labels + static_cast<int64_t>(r) * p.ld_labels : nullptr;
  int n = p.N;
  if (p.n_valid) n = max(0, min(n, p.n_valid[r]));

  unsigned long long prefix = 0ull;
  int kk = 0;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      uint32_t label = static_cast<uint32_t>(i);
      if (lab) {
        const int32_t l = lab[i];
        if (l < 0) continue;
        label = static_cast<uint32_t>(l);
      }
      const unsigned long long key =
          (static_cast<unsigned long long>(order_code(row[i])) << 32) | static_cast<uint32_t>(~label);
      if (pass == 0 || (key >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (highest bins first)
      const int lane = tid;
      // read before the shuffles below, which every lane must pass before any
      // lane rewrites sh.need
      const uint32_t prev_need = sh.need;
      uint32_t c[8];
      uint32_t lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sh.hist[255 - 8 * lane - j];
        lsum += c[j];
      }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
      uint32_t want;
      if (pass == 0) {
        want = min(static_cast<uint32_t>(p.k), total);
        if (lane == 0) sh.total = total;
      } else {
        want = prev_need;
      }
      uint32_t cum = incl - lsum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (want > 0 && cum < want && cum + c[j] >= want) {
          sh.digit = 255 - 8 * lane - j;
          sh.need = want - cum;
          sh.done = (c[j] == want - cum) ? 1u : 0u;
        }
        cum += c[j];
      }
      if (want == 0 && lane == 0) {
        sh.done = 1u;
        sh.need = 0u;
        sh.digit = 0u;
      }
    }
    __syncthreads();
    if (pass == 0) kk = static_cast<int>(min(static_cast<uint32_t>(p.k), sh.total));
    if (kk == 0) break;
    prefix |= static_cast<unsigned long long>(sh.digit) << shift;
    const uint32_t done = sh.done;
    __syncthreads();  // everyone has read digit/need/done before the next pass rewrites them
    if (done) break;
  }
  if (kk > 0) {
    if (tid == 0) sh.cnt = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      uint32_t label = static_cast<uint32_t>(i);
      if (lab) {
        const int32_t l = lab[i];
        if (l < 0) continue;
        label = static_cast<uint32_t>(l);
      }
      const unsigned long long key =
          (static_cast<unsigned long long>(order_code(row[i])) << 32) | static_cast<uint32_t>(~label);
      if (key >= prefix) {
        const uint32_t slot = atomicAdd(&sh.cnt, 1u);
        if (slot < static_cast<uint32_t>(kMaxTopK)) {
          sh.key[slot] = key;
          sh.col[slot] = static_cast<uint32_t>(i);
        }
      }
    }
    __syncthreads();
    int P2 = 1;
    while (P2 < kk) P2 <<= 1;
    for (int i = kk + tid; i < P2; i += kTopkThreads) {
      sh.key[i] = 0ull;
      sh.col[i] = 0u;
    }
    __syncthreads();
    for (int size = 2; size <= P2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (P2 >> 1); i += kTopkThreads) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool desc = (lo & size) == 0;
          const unsigned long long a = sh.key[lo], b = sh.key[hi];
          if (desc ? (a < b) : (a > b)) {
            sh.key[lo] = b;
            sh.key[hi] = a;
            const uint32_t t = sh.col[lo];
            sh.col[lo] = sh.col[hi];
            sh.col[hi] = t;
          }
        }
        __syncthreads();
      }
    }
  }
  int32_t* io = p.idx_out + static_cast<int64_t>(r) * p.ld_out;
  float* vo = p.val_out ? p.val_out + static_cast<int64_t>(r) * p.ld_out : nullptr;
  for (int j = tid; j < p.k; j += kTopkThreads) {
    if (j < kk) {
      io[j] = static_cast<int32_t>(~static_cast<uint32_t>(sh.key[j] & 0xffffffffull));
      if (vo) vo[j] = row[sh.col[j]];
    } else {
      io[j] = -1;
      if (vo) vo[j] = neg_inf();
    }
  }
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(TopkShared)));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  if (p.R == 0) return cudaSuccess;
  topk_kernel<<<p.R, kTopkThreads, sizeof(TopkShared), st>>>(p);
  return cudaGetLastError();
}

}  // namespace lsi

// Exact row-wise top-k by (score desc, position asc).
//
// Selection order follows the packed-key radix select of "Latent Sparse
// Attention", section "What the kernels do about the top-p": the score's bits
// sit above the inverted id in one 64-bit key, so the largest keys are the
// highest scores with ties going to the lower id.  Scores are first mapped to
// an order-preserving 32-bit code (-0.0 and +0.0 share a code; NaN gets code
// 0, below -inf), so the 64-bit keys of a row are distinct and the k-th
// largest key is a unique threshold.
//
// One CTA of 1024 threads per row:
//   1. A 2048-bin histogram of the top 11 code bits, either handed over by the
//      scoring kernel (which counts its scores as it writes them) or built
//      here in one pass over the row.
//   2. The bin holding the k-th largest key splits the row: one pass copies
//      every key above that bin to the selection and every key inside it to a
//      shared-memory candidate buffer.
//   3. An MSB-first 8-bit radix select over the candidates' remaining bits
//      picks the rest; it stops as soon as every key sharing the current
//      prefix is wanted.
//   4. A bitonic sort of the k selected keys in shared memory gives the
//      canonical order.
// A row whose threshold bin holds more candidates than the buffer takes the
// plain path instead: the same radix select run over the whole row in global
// memory (one pass per 8-bit digit), then one collecting pass.
// Values are written as bit copies of the input.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

constexpr int kTopkThreads = 1024;
constexpr int kCandCap = 4096;  // threshold-bin candidates kept in shared memory

struct TopkShared {
  unsigned long long sel_key[kMaxTopK];
  uint32_t sel_col[kMaxTopK];
  unsigned long long cand_key[kCandCap];
  uint32_t cand_col[kCandCap];
  uint32_t hist[kHistBins];
  uint32_t digit, need, done, total, cnt, ccnt, bstar, above, eq;
};

// Warp 0: find the digit d of a descending histogram such that the keys in
// bins above d number fewer than `want` and those in bins >= d at least
// `want`.  Writes digit / need (= want - above) / done (bin d is taken whole).
template <int BINS>
__device__ __forceinline__ void find_digit(TopkShared& sh, const uint32_t* hist, uint32_t want) {
  const int lane = threadIdx.x;
  constexpr int PER = BINS / 32;
  uint32_t lsum = 0;
#pragma unroll 8
  for (int j = 0; j < PER; ++j) lsum += hist[BINS - 1 - PER * lane - j];
  uint32_t incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  uint32_t cum = incl - lsum;
  if (cum < want && cum + lsum >= want) {
    for (int j = 0; j < PER; ++j) {
      const uint32_t c = hist[BINS - 1 - PER * lane - j];
      if (cum + c >= want) {
        sh.digit = BINS - 1 - PER * lane - j;
        sh.need = want - cum;
        sh.above = cum;
        sh.eq = c;
        sh.done = (c == want - cum) ? 1u : 0u;
        break;
      }
      cum += c;
    }
  }
}

// MSB-first radix select over `count` 64-bit keys produced by get(i).  Bits
// at and above `hi` are equal across all keys; digits of 8 bits (the last one
// narrower) are resolved from bit hi-1 down.  Returns the largest threshold T
// such that exactly `want` keys are >= T (keys are distinct).
template <class Get>
__device__ unsigned long long radix_select(TopkShared& sh, Get get, int count, uint32_t want, int hi) {
  unsigned long long prefix = 0ull;
  while (hi > 0) {
    const int width = hi < 8 ? hi : 8;
    const int shift = hi - width;
    for (int i = threadIdx.x; i < 256; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += kTopkThreads) {
      unsigned long long key;
      if (!get(i, key)) continue;
      if (hi >= 64 || (key >> hi) == (prefix >> hi))
        atomicAdd(&sh.hist[(key >> shift) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_digit<256>(sh, sh.hist, want);
    __syncthreads();
    prefix |= static_cast<unsigned long long>(sh.digit) << shift;
    want = sh.need;
    const uint32_t done = sh.done;
    __syncthreads();
    hi = shift;
    if (done) break;
  }
  return prefix;
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = p.scores + static_cast<int64_t>(r) * p.ld;
  const int32_t* lab = p.labels ? p.labels + static_cast<int64_t>(r) * p.ld_labels : nullptr;
  int n = p.N;
  if (p.n_valid) n = max(0, min(n, p.n_valid[r]));

  // key of element i (false when absent)
  auto key_of = [&](int i, unsigned long long& key) -> bool {
    uint32_t label = static_cast<uint32_t>(i);
    if (lab) {
      const int32_t l = lab[i];
      if (l < 0) return false;
      label = static_cast<uint32_t>(l);
    }
    key = (static_cast<unsigned long long>(order_code(row[i])) << 32) | static_cast<uint32_t>(~label);
    return true;
  };

  // ---- 1. histogram of the top code bits ---------------------------------
  if (p.hist) {
    const uint32_t* gh = p.hist + static_cast<int64_t>(r) * kHistBins;
    for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = gh[i];
  } else {
    for (int i = tid; i < kHistBins; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      if (lab && lab[i] < 0) continue;
      atomicAdd(&sh.hist[hist_bin(order_code(row[i]))], 1u);
    }
  }
  __syncthreads();
  if (tid < 32) {
    uint32_t tot = 0;
    for (int j = tid; j < kHistBins; j += 32) tot += sh.hist[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    const uint32_t want = min(static_cast<uint32_t>(p.k), tot);
    if (tid == 0) {
      sh.total = tot;
      sh.cnt = 0;
      sh.ccnt = 0;
    }
    if (want > 0) find_digit<kHistBins>(sh, sh.hist, want);
  }
  __syncthreads();
  const int kk = static_cast<int>(min(static_cast<uint32_t>(p.k), sh.total));

  if (kk > 0) {
    const uint32_t bstar = sh.digit;
    const uint32_t need = sh.need;
    const uint32_t eq = sh.eq;
    __syncthreads();
    if (eq <= static_cast<uint32_t>(kCandCap)) {
      // ---- 2. split the row at the threshold bin --------------------------
      for (int i = tid; i < n; i += kTopkThreads) {
        unsigned long long key;
        if (!key_of(i, key)) continue;
        const uint32_t bin = static_cast<uint32_t>(key >> (64 - kHistBits));
        if (bin > bstar) {
          const uint32_t s = atomicAdd(&sh.cnt, 1u);
          if (s < static_cast<uint32_t>(kMaxTopK)) {
            sh.sel_key[s] = key;
            sh.sel_col[s] = static_cast<uint32_t>(i);
          }
        } else if (bin == bstar) {
          const uint32_t c = atomicAdd(&sh.ccnt, 1u);
          if (c < static_cast<uint32_t>(kCandCap)) {
            sh.cand_key[c] = key;
            sh.cand_col[c] = static_cast<uint32_t>(i);
          }
        }
      }
      __syncthreads();
      // ---- 3. radix select inside the threshold bin -----------------------
      const int nc = static_cast<int>(min(sh.ccnt, static_cast<uint32_t>(kCandCap)));
      unsigned long long thr = 0ull;
      if (need < static_cast<uint32_t>(nc)) {
        thr = radix_select(
            sh, [&](int i, unsigned long long& key) -> bool { key = sh.cand_key[i]; return true; }, nc, need,
            64 - kHistBits);
      }
      for (int i = tid; i < nc; i += kTopkThreads) {
        if (sh.cand_key[i] >= thr) {
          const uint32_t s = atomicAdd(&sh.cnt, 1u);
          if (s < static_cast<uint32_t>(kMaxTopK)) {
            sh.sel_key[s] = sh.cand_key[i];
            sh.sel_col[s] = sh.cand_col[i];
          }
        }
      }
    } else {
      // ---- plain path: radix select over the whole row --------------------
      const unsigned long long thr = radix_select(sh, key_of, n, static_cast<uint32_t>(kk), 64);
      for (int i = tid; i < n; i += kTopkThreads) {
        unsigned long long key;
        if (!key_of(i, key)) continue;
        if (key >= thr) {
          const uint32_t s = atomicAdd(&sh.cnt, 1u);
          if (s < static_cast<uint32_t>(kMaxTopK)) {
            sh.sel_key[s] = key;
            sh.sel_col[s] = static_cast<uint32_t>(i);
          }
        }
      }
    }
    __syncthreads();
    // ---- 4. canonical order ------------------------------------------------
    int P2 = 1;
    while (P2 < kk) P2 <<= 1;
    for (int i = kk + tid; i < P2; i += kTopkThreads) {
      sh.sel_key[i] = 0ull;
      sh.sel_col[i] = 0u;
    }
    __syncthreads();
    for (int size = 2; size <= P2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (P2 >> 1); i += kTopkThreads) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool desc = (lo & size) == 0;
          const unsigned long long a = sh.sel_key[lo], b = sh.sel_key[hi];
          if (desc ? (a < b) : (a > b)) {
            sh.sel_key[lo] = b;
            sh.sel_key[hi] = a;
            const uint32_t t = sh.sel_col[lo];
            sh.sel_col[lo] = sh.sel_col[hi];
            sh.sel_col[hi] = t;
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
      io[j] = static_cast<int32_t>(~static_cast<uint32_t>(sh.sel_key[j] & 0xffffffffull));
      if (vo) vo[j] = row[sh.sel_col[j]];
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

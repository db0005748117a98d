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
// The same article's threshold idea (a sampled threshold decides how many
// candidates are listed, never which are picked; a row whose estimate misses
// falls back to exact work) shapes the kernel.  One CTA of 1024 threads per
// row:
//   1. A 2048-bin histogram of the top 11 code bits: handed over by the
//      scoring kernel, counted exactly for rows of up to 8192 entries, or
//      counted on a sample of about 4096-8192 entries (groups of 8
//      consecutive entries, evenly spaced).
//   2. A low bin is chosen so that the entries at or above it hold the top k
//      (exactly, or with margin from the sample); one pass over the row lists
//      them in a shared-memory candidate buffer.
//   3. If the list is short of k or overflows the buffer, the row takes the
//      exact plain path: an MSB-first radix select over the whole row in
//      global memory, then one collecting pass.
//   4. Otherwise an MSB-first radix select inside the buffer finds the k-th
//      largest key and the k keys at or above it are compacted.
//   5. Canonical order: the k keys are bucketed by their position in the
//      [min, max] key range (2048 fine bins), and each key's output slot is
//      its bucket's offset plus the number of larger keys in its bucket.
//
// Row passes keep many loads in flight (4 float4 per thread per chunk); writes
// into shared buffers take one atomic per warp (a warp scan hands out slots).
// Values are written as bit copies of the input.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

constexpr int kCandCap = 8192;     // listed candidates kept in shared memory (the wide forms)
constexpr int kExactHistMax = 2048; // rows up to this length get an exact histogram; longer rows
                                    // sample about this many entries
constexpr int kVec = 4;            // float4 loads per thread per chunk
constexpr int kChunk = kVec * 4;   // entries per thread per chunk

// NT threads per CTA (one row each), KMAX the largest k the CTA holds.
template <int NT, int KMAX, int CAP>
struct TopkShared {
  float cand_val[CAP];                 // listed entries: value and label
  int32_t cand_lab[CAP];
  unsigned long long sel_key[KMAX];    // the k selected: packed key and value
  unsigned long long tmp_key[KMAX];    // bucketed copy for the final order
  float sel_val[KMAX];                 // (sel_key + tmp_key and sel_val + tmp_val are also
  float tmp_val[KMAX];                 //  used as one 2*KMAX array by the bucket select)
  uint32_t hist[kHistBins];
  uint32_t fill[kHistBins];
  uint32_t wsum[NT / 32];
  unsigned long long wmin[NT / 32], wmax[NT / 32];
  uint32_t digit, need, done, total, cnt, ccnt, eq;
};

__device__ __forceinline__ unsigned long long pack_key(float v, int32_t label) {
  return (static_cast<unsigned long long>(order_code(v)) << 32) |
         static_cast<uint32_t>(~static_cast<uint32_t>(label));
}

// Smallest float whose order code is `code` (codes >= 4 << 21 are finite).
__device__ __forceinline__ float code_floor_value(uint32_t code) {
  return __uint_as_float((code & 0x80000000u) ? (code & 0x7fffffffu) : ~code);
}

// One row of scores with optional labels.  `vec`: both row pointers are
// 16-byte aligned, so chunks use float4 / int4 loads.
struct RowRef {
  const float* v;
  const int32_t* lab;
  int n;
  bool vec;
};

struct Chunk {
  float v[kChunk];
  int32_t lab[kChunk];  // label (the column when the row has none); < 0 = absent
};

template <int NT>
__device__ __forceinline__ int chunk_count(const RowRef& rr) {
  if (rr.vec) {
    const int n4 = rr.n >> 2;
    return (n4 + kVec * NT - 1) / (kVec * NT) + ((rr.n & 3) ? 1 : 0);
  }
  return (rr.n + kChunk * NT - 1) / (kChunk * NT);
}

// Column of entry e of chunk `it` for this thread.
template <int NT>
__device__ __forceinline__ int chunk_col(const RowRef& rr, int it, int e) {
  if (rr.vec) {
    const int n4 = rr.n >> 2;
    const int body = (n4 + kVec * NT - 1) / (kVec * NT);
    if (it < body) return 4 * ((it * kVec + (e >> 2)) * NT + static_cast<int>(threadIdx.x)) + (e & 3);
    return 4 * n4 + static_cast<int>(threadIdx.x);  // tail chunk: entry 0 only
  }
  return (it * kChunk + e) * NT + static_cast<int>(threadIdx.x);
}

// Loads chunk `it`; returns a bit per present entry.
template <int NT>
__device__ __forceinline__ uint32_t load_chunk(const RowRef& rr, int it, Chunk& c) {
  uint32_t present = 0;
  if (rr.vec) {
    const int n4 = rr.n >> 2;
    const int body = (n4 + kVec * NT - 1) / (kVec * NT);
    if (it < body) {
      float4 a[kVec];
      int4 b[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int j = (it * kVec + u) * NT + static_cast<int>(threadIdx.x);
        a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        b[u] = make_int4(-1, -1, -1, -1);
        if (j < n4) {
          a[u] = __ldg(reinterpret_cast<const float4*>(rr.v) + j);
          b[u] = rr.lab ? __ldg(reinterpret_cast<const int4*>(rr.lab) + j) : make_int4(4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3);
        }
      }
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        c.v[4 * u] = a[u].x;
        c.v[4 * u + 1] = a[u].y;
        c.v[4 * u + 2] = a[u].z;
        c.v[4 * u + 3] = a[u].w;
        c.lab[4 * u] = b[u].x;
        c.lab[4 * u + 1] = b[u].y;
        c.lab[4 * u + 2] = b[u].z;
        c.lab[4 * u + 3] = b[u].w;
      }
    } else {
      const int i = 4 * n4 + static_cast<int>(threadIdx.x);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        c.v[e] = 0.f;
        c.lab[e] = -1;
      }
      if (i < rr.n) {
        c.v[0] = __ldg(rr.v + i);
        c.lab[0] = rr.lab ? __ldg(rr.lab + i) : i;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const int i = (it * kChunk + e) * NT + static_cast<int>(threadIdx.x);
      c.v[e] = 0.f;
      c.lab[e] = -1;
      if (i < rr.n) {
        c.v[e] = __ldg(rr.v + i);
        c.lab[e] = rr.lab ? __ldg(rr.lab + i) : i;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kChunk; ++e)
    if (c.lab[e] >= 0) present |= 1u << e;
  return present;
}

// Warp 0: in a 256-bin histogram scanned from the top, find the digit d with
// fewer than `want` keys above it and at least `want` at or above it.
template <class SH>
__device__ __forceinline__ void find_digit_256(SH& sh, uint32_t want) {
  const int lane = threadIdx.x;
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
  uint32_t cum = incl - lsum;
  if (cum < want && cum + lsum >= want) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (cum < want && cum + c[j] >= want) {
        sh.digit = 255 - 8 * lane - j;
        sh.need = want - cum;
        sh.eq = c[j];
        sh.done = (c[j] == want - cum) ? 1u : 0u;
      }
      cum += c[j];
    }
  }
}

// All threads: exclusive prefix of a 2048-bin histogram taken from the top
// (bin 2047 first) into `excl_out` (may alias nothing), the total into
// sh.total, and for want = min(want_cap, total) > 0 the bin holding the
// want-th entry (sh.digit / sh.need / sh.eq).  Thread t takes the 2048 / NT
// consecutive bins just below bin 2047 - t * (2048 / NT) + 1.
template <int NT, class SH>
__device__ __forceinline__ void scan_bins_2048(SH& sh, const uint32_t* hist, uint32_t* excl_out,
                                               uint32_t want_cap) {
  constexpr int BPT = kHistBins / NT;
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  uint32_t c[BPT];
  uint32_t csum = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    c[j] = hist[kHistBins - 1 - BPT * t - j];  // higher bin first
    csum += c[j];
  }
  uint32_t incl = csum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sh.wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = lane < NT / 32 ? sh.wsum[lane] : 0u;
    uint32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < NT / 32) sh.wsum[lane] = wi - wv;
    if (lane == 31) sh.total = wi;
  }
  __syncthreads();
  uint32_t excl = incl - csum + sh.wsum[warp];
  const uint32_t want = min(want_cap, sh.total);
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int bin = kHistBins - 1 - BPT * t - j;
    if (excl_out) excl_out[bin] = excl;
    if (want > 0 && excl < want && excl + c[j] >= want) {
      sh.digit = bin;
      sh.need = want - excl;
      sh.eq = c[j];
    }
    excl += c[j];
  }
  __syncthreads();
}

__device__ __forceinline__ float f4at(const float4& a, int q) {
  return q == 0 ? a.x : q == 1 ? a.y : q == 2 ? a.z : a.w;
}
__device__ __forceinline__ int32_t i4at(const int4& a, int q) {
  return q == 0 ? a.x : q == 1 ? a.y : q == 2 ? a.z : a.w;
}

// Warp-collective append of up to 16 flagged entries per thread: one atomic
// per warp hands out the slots; slots >= cap are counted, not stored.
__device__ __forceinline__ uint32_t warp_slots(uint32_t flags, uint32_t* counter) {
  const int lane = threadIdx.x & 31;
  const uint32_t mine = __popc(flags);
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
  uint32_t base = 0;
  if (lane == 31) base = atomicAdd(counter, tot);
  base = __shfl_sync(0xffffffffu, base, 31);
  return base + incl - mine;
}

// Listing pass: every present entry whose key passes `keep(value, label)` is
// appended to (vals, labs): its value and its label (the column when the row
// has no labels).  Threads read 4 float4 (and int4
// labels when the row has them) per step; all threads run the same number of
// steps.  Rows without labels skip every label computation until an entry is
// flagged.
template <int NT, bool HAS_LAB, class Keep>
__device__ __forceinline__ void list_row_t(const RowRef& rr, Keep keep, float* vals, int32_t* labs,
                                           uint32_t* counter, uint32_t cap) {
  const int tid = threadIdx.x;
  if (rr.vec) {
    const int n4 = rr.n >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(rr.v);
    const int4* l4 = reinterpret_cast<const int4*>(rr.lab);
    for (int base = 0; base < n4; base += kVec * NT) {
      float4 a[kVec];
      int4 l[kVec];
      uint32_t inb = 0;  // bit u: vector u exists
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int j = base + u * NT + tid;
        a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (HAS_LAB) l[u] = make_int4(-1, -1, -1, -1);
        if (j < n4) {
          a[u] = __ldg(v4 + j);
          if (HAS_LAB) l[u] = __ldg(l4 + j);
          inb |= 1u << u;
        }
      }
      uint32_t flags = 0;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        // label: the column when the row has none (dead code unless keep reads it)
        const int32_t lb = HAS_LAB ? i4at(l[e >> 2], e & 3) : 4 * (base + (e >> 2) * NT + tid) + (e & 3);
        const bool ok = HAS_LAB ? (lb >= 0) : ((inb >> (e >> 2)) & 1u);
        if (ok && keep(f4at(a[e >> 2], e & 3), lb)) flags |= 1u << e;
      }
      if (!__any_sync(0xffffffffu, flags != 0u)) continue;
      uint32_t slot = warp_slots(flags, counter);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        if (flags & (1u << e)) {
          if (slot < cap) {
            vals[slot] = f4at(a[e >> 2], e & 3);
            labs[slot] = HAS_LAB ? i4at(l[e >> 2], e & 3) : 4 * (base + (e >> 2) * NT + tid) + (e & 3);
          }
          ++slot;
        }
      }
    }
    // the n % 4 entries after the float4 body, one per thread
    const int i = 4 * n4 + tid;
    uint32_t flag = 0;
    float v = 0.f;
    int32_t lb = -1;
    if (i < rr.n) {
      v = __ldg(rr.v + i);
      lb = HAS_LAB ? __ldg(rr.lab + i) : i;
      if (lb >= 0 && keep(v, lb)) flag = 1u;
    }
    if (__any_sync(0xffffffffu, flag != 0u)) {
      const uint32_t slot = warp_slots(flag, counter);
      if (flag && slot < cap) {
        vals[slot] = v;
        labs[slot] = lb;
      }
    }
  } else {
    for (int base = 0; base < rr.n; base += kChunk * NT) {
      float a[kChunk];
      int32_t l[kChunk];
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const int i = base + e * NT + tid;
        a[e] = 0.f;
        l[e] = -1;
        if (i < rr.n) {
          a[e] = __ldg(rr.v + i);
          l[e] = HAS_LAB ? __ldg(rr.lab + i) : i;
        }
      }
      uint32_t flags = 0;
#pragma unroll
      for (int e = 0; e < kChunk; ++e)
        if (l[e] >= 0 && keep(a[e], l[e])) flags |= 1u << e;
      if (!__any_sync(0xffffffffu, flags != 0u)) continue;
      uint32_t slot = warp_slots(flags, counter);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        if (flags & (1u << e)) {
          if (slot < cap) {
            vals[slot] = a[e];
            labs[slot] = l[e];
          }
          ++slot;
        }
      }
    }
  }
}

template <int NT, class Keep>
__device__ __forceinline__ void list_row(const RowRef& rr, Keep keep, float* vals, int32_t* labs, uint32_t* counter,
                                         uint32_t cap) {
  if (rr.lab) list_row_t<NT, true>(rr, keep, vals, labs, counter, cap);
  else list_row_t<NT, false>(rr, keep, vals, labs, counter, cap);
}

// Plain path: MSB-first radix select over the whole row in global memory.
// Returns the threshold T with exactly `want` present keys >= T.
template <int NT, class SH>
__device__ unsigned long long radix_select_row(SH& sh, const RowRef& rr, uint32_t want) {
  unsigned long long prefix = 0ull;
  const int chunks = chunk_count<NT>(rr);
  for (int hi = 64; hi > 0; hi -= 8) {
    const int shift = hi - 8;
    for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0;
    __syncthreads();
    for (int it = 0; it < chunks; ++it) {
      Chunk c;
      const uint32_t present = load_chunk<NT>(rr, it, c);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        if (present & (1u << e)) {
          const unsigned long long key = pack_key(c.v[e], c.lab[e]);
          if (hi >= 64 || (key >> hi) == (prefix >> hi)) atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) find_digit_256(sh, want);
    __syncthreads();
    prefix |= static_cast<unsigned long long>(sh.digit) << shift;
    want = sh.need;
    const uint32_t done = sh.done;
    __syncthreads();
    if (done) break;
  }
  return prefix;
}

// MSB-first radix select over the `nc` keys of the candidate buffer.  It
// starts at the highest bit where the candidates differ (their common high
// bits are read off the smallest and largest key), so no pass is spent on
// bits every candidate shares.
template <int NT, class SH>
__device__ unsigned long long radix_select_cand(SH& sh, int nc, uint32_t want) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long kmin = ~0ull, kmax = 0ull;
  for (int i = threadIdx.x; i < nc; i += NT) {
    const unsigned long long key = pack_key(sh.cand_val[i], sh.cand_lab[i]);
    kmin = key < kmin ? key : kmin;
    kmax = key > kmax ? key : kmax;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (lane == 0) {
    sh.wmin[warp] = kmin;
    sh.wmax[warp] = kmax;
  }
  for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0;
  __syncthreads();
  if (warp == 0) {
    kmin = lane < NT / 32 ? sh.wmin[lane] : ~0ull;
    kmax = lane < NT / 32 ? sh.wmax[lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
      const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = a < kmin ? a : kmin;
      kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
      sh.wmin[0] = kmin;
      sh.wmax[0] = kmax;
    }
  }
  __syncthreads();
  kmin = sh.wmin[0];
  kmax = sh.wmax[0];
  const unsigned long long diff = kmin ^ kmax;
  int hi = diff ? 64 - __clzll(static_cast<long long>(diff)) : 0;
  unsigned long long prefix = hi >= 64 ? 0ull : (kmin >> hi) << hi;  // bits every candidate shares
  bool first = true;
  while (hi > 0) {
    const int width = hi < 8 ? hi : 8;
    const int shift = hi - width;
    if (!first) {
      for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0;
      __syncthreads();
    }
    first = false;
    for (int i = threadIdx.x; i < nc; i += NT) {
      const unsigned long long key = pack_key(sh.cand_val[i], sh.cand_lab[i]);
      if (hi >= 64 || (key >> hi) == (prefix >> hi))
        atomicAdd(&sh.hist[static_cast<uint32_t>(key >> shift) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_digit_256(sh, want);
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

// NT threads, largest k KMAX, CAP listed candidates: <1024, 4096, 8192> one
// CTA per SM; <512, 1024, 8192> two; <256, 512, 2048> four (rows of many
// queries with k <= 512: more rows in flight hide the per-row latency).
// LOOP: the CTAs walk the rows (launches with row flags, where most rows are
// left untouched); otherwise one CTA per row.
template <int NT, int KMAX, int CAP, bool LOOP>
__global__ void __launch_bounds__(NT, (NT == 256) ? 4 : 1024 / NT) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared<NT, KMAX, CAP>& sh = *reinterpret_cast<TopkShared<NT, KMAX, CAP>*>(topk_smem);
  if (p.run_if != nullptr && *p.run_if == 0) return;      // conditional launch with nothing to do
  // rows blockIdx.x, blockIdx.x + gridDim.x, ... (LOOP), else row blockIdx.x
  for (int r = blockIdx.x; r < p.R; r += (LOOP ? gridDim.x : p.R)) {
  if (p.row_flag != nullptr && p.row_flag[r] == 0) continue;  // row left untouched
  const int orow = p.out_row ? p.out_row[r] : r;               // where the row's output goes
  if (orow < 0) continue;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  RowRef rr;
  rr.v = p.scores + static_cast<int64_t>(r) * p.ld;
  rr.lab = p.labels ? p.labels + static_cast<int64_t>(r) * p.ld_labels : nullptr;
  rr.n = p.N;
  if (p.n_valid) rr.n = max(0, min(rr.n, p.n_valid[r] - p.nv_offset));
  rr.vec = ((reinterpret_cast<uintptr_t>(rr.v) & 15u) == 0) &&
           (rr.lab == nullptr || (reinterpret_cast<uintptr_t>(rr.lab) & 15u) == 0);
  const int chunks = chunk_count<NT>(rr);
  const uint32_t kcap = static_cast<uint32_t>(min(p.k, rr.n));  // k, or fewer entries

  // ---- 1. histogram of the top code bits ---------------------------------
  if (tid == 0) {
    sh.cnt = 0;
    sh.ccnt = 0;
  }
  bool exact_hist = true;
  int S = 1;  // sampling period in groups of 8 entries
  if (p.hist) {
    const uint32_t* gh = p.hist + static_cast<int64_t>(r) * kHistBins;
    for (int i = tid; i < kHistBins; i += NT) sh.hist[i] = gh[i];
  } else {
    for (int i = tid; i < kHistBins; i += NT) sh.hist[i] = 0;
    __syncthreads();
    if (rr.n <= kExactHistMax) {
      for (int i = tid; i < rr.n; i += NT) {
        const int32_t l = rr.lab ? __ldg(rr.lab + i) : i;
        if (l >= 0) atomicAdd(&sh.hist[hist_bin(order_code(__ldg(rr.v + i)))], 1u);
      }
    } else {
      exact_hist = false;
      while ((rr.n / S) > kExactHistMax) S <<= 1;
      // the list's margin (16 sampled entries, 16 * S row entries) must stay
      // well inside the candidate capacity: long rows are sampled more densely
      if (S > CAP / 64) S = CAP / 64 > 1 ? CAP / 64 : 1;
      const int groups = (rr.n + 7) >> 3;
      for (int g = tid * S; g < groups; g += NT * S) {
        const int i0 = g << 3;
        float v[8];
        int32_t l[8];
        if (rr.vec && i0 + 8 <= rr.n) {
          const float4 a0 = __ldg(reinterpret_cast<const float4*>(rr.v + i0));
          const float4 a1 = __ldg(reinterpret_cast<const float4*>(rr.v + i0) + 1);
          v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
          v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
#pragma unroll
          for (int e = 0; e < 8; ++e) l[e] = rr.lab ? __ldg(rr.lab + i0 + e) : i0 + e;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const bool in = i0 + e < rr.n;
            v[e] = in ? __ldg(rr.v + i0 + e) : 0.f;
            l[e] = in ? (rr.lab ? __ldg(rr.lab + i0 + e) : i0 + e) : -1;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (l[e] >= 0) atomicAdd(&sh.hist[hist_bin(order_code(v[e]))], 1u);
      }
    }
  }
  __syncthreads();

  // ---- 2. the low bin of the candidate list ---------------------------------
  // exact histogram: the bin holding the k-th entry.  Sample: the bin where the
  // sample holds k/S entries with a 25% + 16 margin.
  uint32_t want_bins = kcap;
  if (!exact_hist) want_bins = (kcap + kcap / 4) / static_cast<uint32_t>(S) + 16u;
  scan_bins_2048<NT>(sh, sh.hist, nullptr, max(want_bins, 1u));
  uint32_t blo = sh.digit;
  const uint32_t hist_total = sh.total;
  if (hist_total == 0) blo = 0;                          // nothing present (or nothing sampled)
  if (!exact_hist && hist_total <= want_bins) blo = 0;   // the sample cannot place the bin: list everything
  // Sampled rows whose boundary bin is coarse (the entries estimated at or
  // above it would crowd the candidate list): refine the boundary by the next
  // 11 code bits of the sampled entries inside that bin.  The list's lower
  // bound becomes a 22-bit code prefix.
  uint32_t lo_code = blo << (32 - kHistBits);
  if (!exact_hist && blo >= 4 && hist_total > want_bins) {
    const uint32_t above = max(want_bins, 1u) - sh.need;  // sampled entries in bins above blo
    if ((static_cast<uint64_t>(above) + sh.eq) * static_cast<uint64_t>(S) > static_cast<uint64_t>(CAP / 2)) {
      const uint32_t need_in = sh.need;                  // sampled entries wanted from bin blo
      __syncthreads();                                   // every thread has read sh.need / sh.eq
      for (int i = tid; i < kHistBins; i += NT) sh.fill[i] = 0;
      __syncthreads();
      const int groups = (rr.n + 7) >> 3;
      for (int g = tid * S; g < groups; g += NT * S) {
        const int i0 = g << 3;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (i0 + e < rr.n) {
            const int32_t l = rr.lab ? __ldg(rr.lab + i0 + e) : i0 + e;
            const uint32_t c = order_code(__ldg(rr.v + i0 + e));
            if (l >= 0 && hist_bin(c) == blo) atomicAdd(&sh.fill[(c >> (32 - 2 * kHistBits)) & (kHistBins - 1)], 1u);
          }
        }
      }
      __syncthreads();
      scan_bins_2048<NT>(sh, sh.fill, nullptr, max(need_in, 1u));
      if (sh.total >= need_in)                           // the bin's sampled entries place the sub-bin
        lo_code = (blo << (32 - kHistBits)) | (sh.digit << (32 - 2 * kHistBits));
    }
  }
  __syncthreads();

  int kk = 0;
  bool plain = false;
  if (kcap > 0 && !(exact_hist && hist_total == 0)) {
    {
      // ---- listing pass: every present entry in a bin >= blo -------------
      if (blo >= 4) {  // bins from 4 up start at finite values: compare the score itself
        const float tlo = code_floor_value(lo_code);
        list_row<NT>(rr, [&](float v, int32_t) { return v >= tlo; }, sh.cand_val, sh.cand_lab, &sh.ccnt, CAP);
      } else {
        list_row<NT>(rr, [&](float v, int32_t) { return hist_bin(order_code(v)) >= blo; }, sh.cand_val, sh.cand_lab,
                 &sh.ccnt, CAP);
      }
      __syncthreads();
      const uint32_t listed = sh.ccnt;
      // entries to select: exact when the histogram counted every present entry
      kk = static_cast<int>(exact_hist ? min(kcap, hist_total) : kcap);
      if (listed > static_cast<uint32_t>(CAP) || listed < static_cast<uint32_t>(kk)) plain = true;
    }
  }

  if (kk > 0 && plain) {
    // ---- 3. exact plain path ---------------------------------------------
    // count the present entries first when the histogram was only sampled
    if (!exact_hist) {
      if (tid == 0) sh.cnt = 0;
      __syncthreads();
      for (int it = 0; it < chunks; ++it) {
        Chunk c;
        const uint32_t present = load_chunk<NT>(rr, it, c);
        uint32_t cnt = __popc(present);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0 && cnt) atomicAdd(&sh.cnt, cnt);
      }
      __syncthreads();
      kk = static_cast<int>(min(kcap, sh.cnt));
      __syncthreads();
    }
    if (tid == 0) sh.ccnt = 0;
    __syncthreads();
    unsigned long long thr = 0ull;
    if (kk > 0) {
      thr = radix_select_row<NT>(sh, rr, static_cast<uint32_t>(kk));
      // exactly kk entries pass: they become the candidate list
      list_row<NT>(rr, [&](float v, int32_t lb) { return pack_key(v, lb) >= thr; }, sh.cand_val, sh.cand_lab, &sh.ccnt,
               CAP);
    }
    __syncthreads();
  }
  int32_t* io = p.idx_out + static_cast<int64_t>(orow) * p.ld_out;
  float* vo = p.val_out ? p.val_out + static_cast<int64_t>(orow) * p.ld_out : nullptr;
  const int lab_add = rr.lab ? 0 : p.label_base;
  const int nc_all = static_cast<int>(min(sh.ccnt, static_cast<uint32_t>(CAP)));
  // ---- 4'. bucket select: selection and canonical order in one pass -------
  // The candidates are bucketed by their position in the [min, max] key range
  // (2048 bins); the bins from the top hold the k largest keys up to the
  // boundary bin.  Keys of the bins down to the boundary are scattered (in
  // bin order) into a 2*KMAX buffer and ranked inside their bin; a key's rank
  // is its output slot, kept if below k.  When the boundary bin reaches past
  // the buffer, the radix path below runs instead.
  if (kk > 0) {
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int i = tid; i < nc_all; i += NT) {
      const unsigned long long key = pack_key(sh.cand_val[i], sh.cand_lab[i]);
      kmin = key < kmin ? key : kmin;
      kmax = key > kmax ? key : kmax;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
      const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = a < kmin ? a : kmin;
      kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
      sh.wmin[warp] = kmin;
      sh.wmax[warp] = kmax;
    }
    for (int i = tid; i < kHistBins; i += NT) {
      sh.hist[i] = 0;
      sh.fill[i] = 0;
    }
    __syncthreads();
    if (warp == 0) {
      kmin = lane < NT / 32 ? sh.wmin[lane] : ~0ull;
      kmax = lane < NT / 32 ? sh.wmax[lane] : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
        const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
        kmin = a < kmin ? a : kmin;
        kmax = b > kmax ? b : kmax;
      }
      if (lane == 0) {
        sh.wmin[0] = kmin;
        sh.wmax[0] = kmax;
      }
    }
    __syncthreads();
    kmin = sh.wmin[0];
    kmax = sh.wmax[0];
    const unsigned long long span = kmax - kmin;
    const int shift = span ? max(0, 64 - __clzll(static_cast<long long>(span)) - kHistBits) : 0;
    for (int i = tid; i < nc_all; i += NT) {
      const unsigned long long key = pack_key(sh.cand_val[i], sh.cand_lab[i]);
      atomicAdd(&sh.hist[static_cast<uint32_t>((key - kmin) >> shift)], 1u);
    }
    __syncthreads();
    scan_bins_2048<NT>(sh, sh.hist, sh.fill, static_cast<uint32_t>(kk));  // fill: offsets from the top
    const uint32_t b_end = sh.fill[sh.digit] + sh.hist[sh.digit];         // end of the boundary bin
    // Every thread holds b_end before any thread's scatter moves fill[]: a
    // thread that read fill[digit] after another warp's atomics would see a
    // larger end, rank slots the scatter never wrote (a bin index taken from
    // uninitialised shared memory) and take the other branch around the
    // barriers below.
    __syncthreads();
    if (b_end <= 2u * KMAX) {
      unsigned long long* bkey = sh.sel_key;  // 2*KMAX keys
      float* bval = sh.sel_val;               // 2*KMAX values
      for (int i = tid; i < nc_all; i += NT) {
        const float v = sh.cand_val[i];
        const unsigned long long key = pack_key(v, sh.cand_lab[i]);
        const uint32_t bin = static_cast<uint32_t>((key - kmin) >> shift);
        if (sh.fill[bin] < b_end) {  // a bin at or above the boundary (its offset only grows past b_end if not)
          const uint32_t pos = atomicAdd(&sh.fill[bin], 1u);
          bkey[pos] = key;
          bval[pos] = v;
        }
      }
      __syncthreads();
      // after the scatter fill[bin] is the bin's end
      for (int i = tid; i < static_cast<int>(b_end); i += NT) {
        const unsigned long long key = bkey[i];
        const uint32_t bin = static_cast<uint32_t>((key - kmin) >> shift);
        const uint32_t end = sh.fill[bin];
        const uint32_t beg = end - sh.hist[bin];
        uint32_t rank = beg;
        for (uint32_t j = beg; j < end; ++j) rank += (bkey[j] > key) ? 1u : 0u;
        if (rank < static_cast<uint32_t>(kk)) {
          io[rank] = static_cast<int32_t>(~static_cast<uint32_t>(key & 0xffffffffull)) + lab_add;
          if (vo) vo[rank] = bval[i];
        }
      }
      kk = -kk;  // done: only the padding is left
    }
    __syncthreads();
  }
  if (kk > 0) {
    // ---- 4. select inside the candidate list ------------------------------
    const int nc = nc_all;
    unsigned long long thr = 0ull;
    if (nc > kk) thr = radix_select_cand<NT>(sh, nc, static_cast<uint32_t>(kk));
    if (tid == 0) sh.cnt = 0;
    __syncthreads();
    const int rounds = (nc + NT - 1) / NT;
    for (int rd = 0; rd < rounds; ++rd) {
      const int i = rd * NT + tid;
      unsigned long long key = 0ull;
      float val = 0.f;
      if (i < nc) {
        val = sh.cand_val[i];
        key = pack_key(val, sh.cand_lab[i]);
      }
      const bool take = i < nc && key >= thr;
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      uint32_t base = 0;
      if (lane == 0 && bal) base = atomicAdd(&sh.cnt, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (take) {
        const uint32_t s = base + __popc(bal & ((1u << lane) - 1u));
        if (s < static_cast<uint32_t>(KMAX)) {
          sh.sel_key[s] = key;
          sh.sel_val[s] = val;
        }
      }
    }
    __syncthreads();
  }

  // ---- 5. canonical order: bucket by key range, rank inside the bucket ----
  if (kk > 0) {
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int i = tid; i < kk; i += NT) {
      const unsigned long long key = sh.sel_key[i];
      kmin = key < kmin ? key : kmin;
      kmax = key > kmax ? key : kmax;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
      const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = a < kmin ? a : kmin;
      kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
      sh.wmin[warp] = kmin;
      sh.wmax[warp] = kmax;
    }
    for (int i = tid; i < kHistBins; i += NT) {
      sh.hist[i] = 0;
      sh.fill[i] = 0;
    }
    __syncthreads();
    if (warp == 0) {
      kmin = lane < NT / 32 ? sh.wmin[lane] : ~0ull;
      kmax = lane < NT / 32 ? sh.wmax[lane] : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
        const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
        kmin = a < kmin ? a : kmin;
        kmax = b > kmax ? b : kmax;
      }
      if (lane == 0) {
        sh.wmin[0] = kmin;
        sh.wmax[0] = kmax;
      }
    }
    __syncthreads();
    kmin = sh.wmin[0];
    kmax = sh.wmax[0];
    const unsigned long long span = kmax - kmin;
    const int shift = span ? max(0, 64 - __clzll(static_cast<long long>(span)) - kHistBits) : 0;
    for (int i = tid; i < kk; i += NT)
      atomicAdd(&sh.hist[static_cast<uint32_t>((sh.sel_key[i] - kmin) >> shift)], 1u);
    __syncthreads();
    // bucket offsets from the top (largest keys first); fill holds the offsets
    scan_bins_2048<NT>(sh, sh.hist, sh.fill, 0u);
    // scatter into buckets
    for (int i = tid; i < kk; i += NT) {
      const unsigned long long key = sh.sel_key[i];
      const uint32_t bin = static_cast<uint32_t>((key - kmin) >> shift);
      const uint32_t pos = atomicAdd(&sh.fill[bin], 1u);
      sh.tmp_key[pos] = key;
      sh.tmp_val[pos] = sh.sel_val[i];
    }
    __syncthreads();
    // rank inside the bucket: after the scatter fill[bin] is the bucket's end
    for (int i = tid; i < kk; i += NT) {
      const unsigned long long key = sh.tmp_key[i];
      const uint32_t bin = static_cast<uint32_t>((key - kmin) >> shift);
      const uint32_t end = sh.fill[bin];
      const uint32_t beg = end - sh.hist[bin];
      uint32_t rank = beg;
      for (uint32_t j = beg; j < end; ++j) rank += (sh.tmp_key[j] > key) ? 1u : 0u;
      io[rank] = static_cast<int32_t>(~static_cast<uint32_t>(key & 0xffffffffull)) + lab_add;
      if (vo) vo[rank] = sh.tmp_val[i];
    }
  }
  if (kk < 0) kk = -kk;
  for (int j = kk + tid; j < p.k; j += NT) {
    io[j] = -1;
    if (vo) vo[j] = neg_inf();
  }
  if (LOOP) __syncthreads();  // the next row reuses the shared block
  }
}

template <int NT, int KMAX, int CAP>
static cudaError_t launch_topk_t(const TopkParams& p, cudaStream_t st, int num_sms) {
  using SH = TopkShared<NT, KMAX, CAP>;
  // flagged launches walk the rows with at most as many CTAs as fit the SMs
  // at once, so a launch with few (or no) flagged rows costs one wave
  constexpr int kCtasPerSm = (NT == 256) ? 4 : 1024 / NT;
  const bool loop = p.row_flag != nullptr && p.R > num_sms * kCtasPerSm;
  static std::atomic<uint64_t> attr_done[2] = {{0}, {0}};
  const void* fn = loop ? reinterpret_cast<const void*>(&topk_kernel<NT, KMAX, CAP, true>)
                        : reinterpret_cast<const void*>(&topk_kernel<NT, KMAX, CAP, false>);
  {
    const cudaError_t e = smem_limit_once(attr_done[loop ? 1 : 0], fn, sizeof(SH));
    if (e != cudaSuccess) return e;
  }
  if (loop) topk_kernel<NT, KMAX, CAP, true><<<num_sms * kCtasPerSm, NT, sizeof(SH), st>>>(p);
  else topk_kernel<NT, KMAX, CAP, false><<<p.R, NT, sizeof(SH), st>>>(p);
  return cudaGetLastError();
}

// More rows than SMs and k <= 1024: 512-thread CTAs, two per SM, so one
// row's latency-bound phases overlap another's streaming pass.  Otherwise one
// 1024-thread CTA per row.
cudaError_t launch_topk(const TopkParams& p, cudaStream_t st, int num_sms) {
  if (p.R == 0) return cudaSuccess;
  if (p.k <= 512 && p.R >= 2 * num_sms) return launch_topk_t<256, 512, 2048>(p, st, num_sms);
  if (p.k <= 1024 && p.R > num_sms) return launch_topk_t<512, 1024, kCandCap>(p, st, num_sms);
  return launch_topk_t<1024, kMaxTopK, kCandCap>(p, st, num_sms);
}

}  // namespace lsi

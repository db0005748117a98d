// Small kernels of the selection path and the library fault word.
//
//  * causal_counts: per query, the number of stride-m compressed entries whose
//    block is complete at the query's token position, floor((t + 1) / m)
//    (LeanSparse podcast transcript, 02:36-02:56: CSA keeps one entry per 4
//    tokens; an entry is eligible once all of its tokens precede the query).
//  * expand: best-first bucket expansion ("Latent Sparse Attention", "The
//    method, term by term", step 6): read the picked buckets in score order,
//    append their members until the budget is held, cut the last bucket short.
//  * fold_scales: w[t, h] * q_scale[t, h] for the fp8 scorer, which takes the
//    non-negative per-(query, head) scale out of the ReLU.
//  * pack_segments: the running prefill selection's per-row lists (the first
//    tile's top-k and each later tile's candidate segment) moved to one
//    contiguous prefix per row for the final top-k.
//  * wait_probe: a kernel whose mbarrier is never signalled, used by the tests
//    to show that a bounded wait returns with an error status.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

__global__ void causal_counts_kernel(const int64_t* q_pos, int T, int stride, int n_total, int32_t* out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int64_t qp = q_pos[t];
  int64_t e = qp < 0 ? 0 : (qp + 1) / stride;
  if (e > n_total) e = n_total;
  out[t] = static_cast<int32_t>(e);
}

cudaError_t launch_causal_counts(const int64_t* q_pos, int T, int stride, int n_total, int32_t* out,
                                 cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  causal_counts_kernel<<<(T + 255) / 256, 256, 0, st>>>(q_pos, T, stride, n_total, out);
  return cudaGetLastError();
}

__global__ void fold_scales_kernel(const float* __restrict__ w, const float* __restrict__ qs, int64_t n,
                                   float* __restrict__ out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = w[i] * qs[i];
}

cudaError_t launch_fold_scales(const float* w, const float* qs, int64_t n, float* out, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256;
  fold_scales_kernel<<<static_cast<int>(want < 2048 ? want : 2048), 256, 0, st>>>(w, qs, n, out);
  return cudaGetLastError();
}

// One CTA per row.  The first tile's top-k stays in place; each later
// segment is moved down to the end of what precedes it, 256 entries at a
// time: every thread reads its entry, a barrier, then every thread writes.
// The source of a segment never starts before its destination, so a chunk's
// writes land below every entry a later chunk still has to read.
constexpr int kPackThreads = 256;

__global__ void __launch_bounds__(kPackThreads)
    pack_segments_kernel(float* __restrict__ val, int32_t* __restrict__ lab, int64_t ld, int T, int k, int S,
                         int cap, const uint32_t* __restrict__ cnt, const int32_t* __restrict__ row_over,
                         int32_t* __restrict__ nv) {
  const int t = blockIdx.x;
  const int64_t row = static_cast<int64_t>(t) * ld;
  int total = k;                                   // the same in every thread
  for (int j = 1; j <= S; ++j) {
    const int64_t c = static_cast<int64_t>(j - 1) * T + t;
    const int64_t src = row + k + static_cast<int64_t>(j - 1) * cap;
    const int n = row_over[c] ? k : static_cast<int>(min(cnt[c], static_cast<uint32_t>(cap)));
    const int64_t dst = row + total;
    if (src != dst) {
      for (int c0 = 0; c0 < n; c0 += kPackThreads) {
        const int e = c0 + static_cast<int>(threadIdx.x);
        float v = 0.f;
        int32_t l = -1;
        if (e < n) {
          v = val[src + e];
          l = lab[src + e];
        }
        __syncthreads();
        if (e < n) {
          val[dst + e] = v;
          lab[dst + e] = l;
        }
      }
    }
    total += n;
  }
  if (threadIdx.x == 0) nv[t] = total;
}

cudaError_t launch_pack_segments(float* val, int32_t* lab, int64_t ld, int T, int k, int S, int cap,
                                 const uint32_t* cnt, const int32_t* row_over, int32_t* nv, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  pack_segments_kernel<<<T, kPackThreads, 0, st>>>(val, lab, ld, T, k, S, cap, cnt, row_over, nv);
  return cudaGetLastError();
}

// One warp per query.
__global__ void expand_kernel(const int32_t* picked, int T, int top_p, const int32_t* off, const int32_t* mem,
                              int P, int budget, int32_t* cand) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int32_t* pk = picked + static_cast<int64_t>(t) * top_p;
  int32_t* out = cand + static_cast<int64_t>(t) * budget;
  int base = 0;
  for (int c0 = 0; c0 < top_p && base < budget; c0 += 32) {
    const int j = c0 + lane;
    const int32_t pb = (j < top_p) ? pk[j] : -1;
    int sz = 0;
    int32_t o = 0;
    if (pb >= 0 && pb < P) {
      o = off[pb];
      sz = max(0, off[pb + 1] - o);
    }
    int incl = sz;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    const int start = base + incl - sz;
    for (int m = 0; m < sz && start + m < budget; ++m) out[start + m] = mem[o + m];
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int j = base + lane; j < budget; j += 32) out[j] = -1;
}

cudaError_t launch_expand(const int32_t* picked, int T, int top_p, const int32_t* off, const int32_t* mem, int P,
                          int budget, int32_t* cand, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (T * 32 + threads - 1) / threads;
  expand_kernel<<<blocks, threads, 0, st>>>(picked, T, top_p, off, mem, P, budget, cand);
  return cudaGetLastError();
}

// A wait on an mbarrier that no thread or copy ever completes.  It must give
// up after `limit_ns`, record FAULT_WAIT_TIMEOUT and return normally.
__global__ void wait_probe_kernel(uint64_t limit_ns, int* waited) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    int gave_up = 0;
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        gave_up = 1;
        atomicOr(&g_fault, FAULT_WAIT_TIMEOUT);
        break;
      }
    }
    *waited = gave_up;
  }
}

cudaError_t launch_wait_probe(uint64_t limit_ns, int* waited, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns, waited);
  return cudaGetLastError();
}

int read_and_clear_fault(cudaStream_t st, int* flags) {
  int h = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_fault, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return static_cast<int>(e);
  const int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_fault, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (flags) *flags = h;
  return static_cast<int>(e);
}

}  // namespace lsi

// Merge of partial top-k lists, the combine step of a prefill whose history
// is split into S contiguous shards (each shard's exact top-k of the same
// queries; the top-k of the union of the shards' top-k lists is the top-k of
// the whole history).  List s of query t holds positions local to shard s,
// sorted canonically, padded with -1 at the end.
//
//  * merge_pack: one CTA per query packs the valid prefixes of its S lists
//    into one row, positions made global by the shard's offset, and the
//    row's length; the exact top-k of the packed rows follows.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

__global__ void __launch_bounds__(256)
    merge_pack_kernel(const float* __restrict__ vals, const int32_t* __restrict__ idx,
                      const int32_t* __restrict__ offsets, int S, int T, int k_in, float* __restrict__ pv,
                      int32_t* __restrict__ pl, int32_t* __restrict__ nv) {
  __shared__ int first_pad;
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t row = static_cast<int64_t>(t) * S * k_in;
  int base = 0;                                   // the same in every thread
  for (int s = 0; s < S; ++s) {
    const int64_t src = (static_cast<int64_t>(s) * T + t) * k_in;
    // the list's valid prefix: the entries before its first -1
    if (tid == 0) first_pad = k_in;
    __syncthreads();
    for (int j = tid; j < k_in; j += 256)
      if (idx[src + j] < 0) atomicMin(&first_pad, j);
    __syncthreads();
    const int n = first_pad;
    const int32_t off = offsets[s];
    for (int j = tid; j < n; j += 256) {
      pv[row + base + j] = vals[src + j];
      pl[row + base + j] = idx[src + j] + off;
    }
    base += n;
    __syncthreads();                              // first_pad is set again for the next list
  }
  if (tid == 0) nv[t] = base;
}

cudaError_t launch_merge_pack(const float* vals, const int32_t* idx, const int32_t* offsets, int S, int T, int k_in,
                              float* pv, int32_t* pl, int32_t* nv, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  merge_pack_kernel<<<T, 256, 0, st>>>(vals, idx, offsets, S, T, k_in, pv, pl, nv);
  return cudaGetLastError();
}

}  // namespace lsi

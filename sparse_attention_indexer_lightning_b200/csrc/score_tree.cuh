// The LSA tree search's descent from node buckets to buckets ("Latent Sparse
// Attention", section "The tree, step by step"): every node_block buckets
// form a node cluster block whose buckets are grouped fanout to a node
// bucket (node n of a complete block covers buckets fanout*n ..
// fanout*n + fanout - 1); the beam keeps the best node buckets, steps down
// to their children plus the buckets no node covers yet, and picks the
// top-p there.  The node scores are a dense contraction (the single-dot
// tensor-core scorer); the children differ per query, so their scores are
// gathered dot products on the CUDA cores here.
//
//  * lsa_tree_visible: per query, visible buckets (complete key blocks
//    before its own) and visible node buckets (complete node blocks among
//    those).
//  * lsa_tree_levels_visible: the same per level of a tree of several node
//    levels (level l groups the complete node blocks of level l - 1).
//  * lsa_tree_candidates: one CTA per query lists and scores its candidate
//    entries of one level: the children of its beam (nodes of the level
//    above), then the visible entries past the last complete node block.

#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lsi {

__global__ void lsa_tree_visible_kernel(const int64_t* __restrict__ q_pos, int T, int block_keys, int bpb, int P,
                                        int node_block, int fanout, int P1, int32_t* __restrict__ vis,
                                        int32_t* __restrict__ vis_nodes) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int64_t qp = q_pos[t] < 0 ? 0 : q_pos[t];
  const int64_t v = (qp / block_keys) * bpb;
  const int vv = static_cast<int>(v < P ? v : P);
  vis[t] = vv;
  const int64_t vn = static_cast<int64_t>(vv / node_block) * (node_block / fanout);
  vis_nodes[t] = static_cast<int32_t>(vn < P1 ? vn : P1);
}

// Visible entries of every level of a tree of several node levels:
// vis[0][t] = visible buckets, vis[l][t] = the level-l nodes of the complete
// node blocks among the query's visible level-(l-1) entries, capped at the
// level's size (size[l]; size[0] = P).  vis is [n + 1][T].
struct TreeLevels {
  int n = 0;
  int size[kMaxTreeLevels + 1] = {};
};

__global__ void lsa_tree_levels_visible_kernel(const int64_t* __restrict__ q_pos, int T, int block_keys, int bpb,
                                               int node_block, int fanout, const TreeLevels lv,
                                               int32_t* __restrict__ vis) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int64_t qp = q_pos[t] < 0 ? 0 : q_pos[t];
  int64_t v = (qp / block_keys) * bpb;
  v = v < lv.size[0] ? v : lv.size[0];
  vis[t] = static_cast<int32_t>(v);
  for (int l = 1; l <= lv.n; ++l) {
    v = (v / node_block) * (node_block / fanout);
    v = v < lv.size[l] ? v : lv.size[l];
    vis[static_cast<int64_t>(l) * T + t] = static_cast<int32_t>(v);
  }
}

// q . c over 64 bf16 dimensions with the query held as 32 packed fp32 pairs:
// each 32-bit word of the row is two bf16 values (low = even dimension),
// widened exactly by a shift and a mask, then one packed FMA per pair.
__device__ __forceinline__ float dot64_bf16(const uint4* __restrict__ row, const uint64_t (&q2)[32]) {
  uint4 x[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) x[v] = __ldg(row + v);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint32_t w4[4] = {x[v].x, x[v].y, x[v].z, x[v].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint64_t cw = pack_f32x2(__uint_as_float(w4[e] << 16), __uint_as_float(w4[e] & 0xffff0000u));
      asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc[e]) : "l"(cw), "l"(q2[4 * v + e]));
    }
  }
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float lo, hi;
    unpack_f32x2(acc[e], lo, hi);
    s += lo + hi;
  }
  return s;
}

// Row t: candidates j < nb * fanout are the children of beam[t][j / fanout]
// (nb = the beam's valid entries), then the uncovered visible buckets
// [vis_nodes[t] * fanout, vis[t]).  Each candidate's score is its centroid's
// dot product with the index query (fp32).
__global__ void __launch_bounds__(256)
    lsa_tree_candidates_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ c,
                               const int32_t* __restrict__ beam, int beam_w, const int32_t* __restrict__ vis,
                               const int32_t* __restrict__ vis_nodes, int fanout, int cap,
                               float* __restrict__ cval, int32_t* __restrict__ clab, int32_t* __restrict__ nv) {
  __shared__ float qs[kLsaDim];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < kLsaDim) qs[tid] = __uint_as_float(static_cast<uint32_t>(q[static_cast<int64_t>(t) * kLsaDim + tid]) << 16);
  __syncthreads();
  uint64_t q2[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) q2[i] = pack_f32x2(qs[2 * i], qs[2 * i + 1]);
  const int nb = min(beam_w, vis_nodes[t]);                // the beam pads with -1 past the visible nodes
  const int covered = vis_nodes[t] * fanout;
  const int n_child = nb * fanout;
  const int total = min(cap, n_child + max(0, vis[t] - covered));
  const int32_t* bm = beam + static_cast<int64_t>(t) * beam_w;
  for (int j = tid; j < total; j += 256) {
    int p;
    if (j < n_child) {
      const int32_t node = bm[j / fanout];
      p = (node < 0) ? -1 : node * fanout + j % fanout;
    } else {
      p = covered + (j - n_child);
    }
    const float acc = (p >= 0) ? dot64_bf16(reinterpret_cast<const uint4*>(c + static_cast<int64_t>(p) * kLsaDim), q2)
                               : -__int_as_float(0x7f800000);   // a missing node leaves -inf
    cval[static_cast<int64_t>(t) * cap + j] = acc;
    clab[static_cast<int64_t>(t) * cap + j] = p;
  }
  if (tid == 0) nv[t] = total;
}

cudaError_t launch_lsa_tree_visible(const int64_t* q_pos, int T, int block_keys, int bpb, int P, int node_block,
                                    int fanout, int P1, int32_t* vis, int32_t* vis_nodes, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_tree_visible_kernel<<<(T + 255) / 256, 256, 0, st>>>(q_pos, T, block_keys, bpb, P, node_block, fanout, P1, vis,
                                                           vis_nodes);
  return cudaGetLastError();
}

cudaError_t launch_lsa_tree_levels_visible(const int64_t* q_pos, int T, int block_keys, int bpb, int node_block,
                                           int fanout, const int* sizes, int n_levels, int32_t* vis,
                                           cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (n_levels < 1 || n_levels > kMaxTreeLevels) return cudaErrorInvalidValue;
  TreeLevels lv;
  lv.n = n_levels;
  for (int l = 0; l <= n_levels; ++l) lv.size[l] = sizes[l];
  lsa_tree_levels_visible_kernel<<<(T + 255) / 256, 256, 0, st>>>(q_pos, T, block_keys, bpb, node_block, fanout, lv,
                                                                  vis);
  return cudaGetLastError();
}

cudaError_t launch_lsa_tree_candidates(const uint16_t* q, const uint16_t* c, const int32_t* beam, int beam_w,
                                       const int32_t* vis, const int32_t* vis_nodes, int T, int fanout, int cap,
                                       float* cval, int32_t* clab, int32_t* nv, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  lsa_tree_candidates_kernel<<<T, 256, 0, st>>>(q, c, beam, beam_w, vis, vis_nodes, fanout, cap, cval, clab, nv);
  return cudaGetLastError();
}

}  // namespace lsi

// Internal launchers shared between the kernel files and the C-ABI layer.
// Nothing here is exported from the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsi {

constexpr int kHeads = 32;   // indexer heads built
constexpr int kDim = 128;    // indexer key / query width
constexpr int kTileKeys = 128;
constexpr int kMaxTopK = 4096;
constexpr int kLsaDim = 64;    // native LSA index space width
constexpr int kMaxTreeLevels = 16;   // node levels of the LSA tree search

// ---------------------------------------------------------------- scoring
// Tensor-core scoring of bf16 keys read by TMA.  One launch covers B
// sequences, T queries per sequence and N keys per sequence (keys of sequence
// b are rows b*N .. b*N+N-1 of the key tensor map).
//   out[(b*T + t)*ld_out + key_base + n] = sum_h w[b,t,h] * relu(q[b,t,h] . k[b,n])
// or -inf where the key is masked: n >= n_valid[b] (when given) or, with
// q_pos, key_base + n >= (q_pos[b,t] + 1) / stride (block-complete causal rule),
// capped at n_total.
//
// Filter form (out == nullptr): nothing is stored per key; instead every
// eligible key whose score beats the row's threshold entry (kth_val /
// kth_lab[row * ld_kth]: the k-th entry of the row's list so far; a label < 0
// means the list is not full and every eligible key is taken) is appended as
// (score, key_base + n) to the row's candidate columns 0 .. cand_cap-1 of
// cand_val / cand_lab at the slot its counter cand_cnt[row] hands out; a row
// that runs out of slots sets row_over[row] and *any_over.  "Beats" compares
// order codes strictly: a later key that ties the threshold entry ranks
// below it.
struct ScoreParams {
  const float* w = nullptr;           // [B][T][H]
  const int32_t* n_valid = nullptr;   // [B] or nullptr
  const int64_t* q_pos = nullptr;     // [B][T] or nullptr
  float* out = nullptr;
  int64_t ld_out = 0;
  int out_col0 = 0;                   // column of key n in out: out_col0 + n
  int stride = 1;
  int B = 0, T = 0, N = 0;
  int key_base = 0;                   // position of key 0 of this launch in the history
  int n_total = 0;                    // causal cap: number of keys of the whole history
  uint32_t* hist = nullptr;           // [B*T][2048] selection histogram (counts added) or nullptr; qg == 1 only
  const int32_t* lim_rows = nullptr;  // [B*T] eligible keys of the whole history per query (replaces q_pos)
  // filter form
  float* cand_val = nullptr;          // row r's slots at cand_val + r * ld_cand
  int32_t* cand_lab = nullptr;
  int64_t ld_cand = 0;
  int cand_cap = 0;
  const float* kth_val = nullptr;     // row r's threshold entry at kth_val[r * ld_kth]
  const int32_t* kth_lab = nullptr;
  int64_t ld_kth = 0;
  uint32_t* cand_cnt = nullptr;       // [B*T]
  int32_t* row_over = nullptr;        // [B*T]
  int* any_over = nullptr;
  const int* run_if = nullptr;        // the launch does nothing unless *run_if != 0 (nullptr: always)
  const float* key_scale = nullptr;   // fp8 scorer: per-key scale [B][N] (scores are multiplied by it)
};

// qg = queries sharing one MMA B tile: 1 (one query per sequence) or 8.
cudaError_t launch_score_tc(int qg, const CUtensorMap* kmap, const CUtensorMap* qmap,
                            const ScoreParams& p, int num_sms, cudaStream_t st);

// fp8 queries and keys (e4m3 codes) on the tensor cores, eight queries per
// group: kmap over the keys [B*N][128 B], qmap over the query heads
// [B*T*H][128 B]; p.w holds w * q_scale (launch_fold_scales), p.key_scale the
// per-key scales [B][N].
cudaError_t launch_score_tc_f8(const CUtensorMap* kmap, const CUtensorMap* qmap, const ScoreParams& p, int num_sms,
                               cudaStream_t st);
// out[i] = w[i] * qs[i], i < n.
cudaError_t launch_fold_scales(const float* w, const float* qs, int64_t n, float* out, cudaStream_t st);

// Native LSA flat search: scores q[t] . c[p] over 64-d bf16 vectors (cmap over
// the centroids [P][128 B], qmap over the index queries [T][128 B]); stored
// to out[t][p] (out != nullptr), or, the filter form (out == nullptr),
// appended as (score, p) to row t's candidate list when p < vis[t] and the
// score's order code reaches that of tau[t * ld_tau].
struct DotParams {
  int T = 0, P = 0;
  float* out = nullptr;
  int64_t ld_out = 0;
  const int32_t* vis = nullptr;       // [T] visible buckets per row
  const float* tau = nullptr;         // thresholds, tau[t * ld_tau]
  int64_t ld_tau = 0;
  // row t's list (ld_cand (score bits, bucket) pairs at t * ld_cand) is
  // split into the segments lsa_segment() gives, one per CTA that scores the
  // row, each in four quarters (one per TMEM lane quadrant: the epilogue
  // warps that read it); counts [T][nseg][4] (nseg: the most CTAs one query
  // group meets), zeroed before the launch
  uint2* cand_list = nullptr;
  int64_t ld_cand = 0;
  int nseg = 0, cap2 = 0, slack = 0;
  uint32_t* cand_cnt = nullptr;
  int32_t* row_over = nullptr;        // [T]
  int* any_over = nullptr;
  const int* run_if = nullptr;        // the launch does nothing unless *run_if != 0 (nullptr: always)
  // storing form: only rows t < *live_rows - live_base are scored (nullptr: all T)
  const int* live_rows = nullptr;
  int live_base = 0;
};
cudaError_t launch_dot_tc(const CUtensorMap* cmap, const CUtensorMap* qmap, const DotParams& p, int num_sms,
                          cudaStream_t st);

// The filter form's list segments.  The scan's `grid` CTAs take contiguous
// runs of its units = G * NT (query group major, NT centroid tiles per
// group), so a query group is scored by a few consecutive CTAs, or by all of
// them when there is one group.  CTA c's segment of a row of group g holds
// cap2 * (the group's tiles it scores) / NT entries plus `slack`, the
// segments of one row laid out in order of c (index j = c - the group's
// first CTA); len = 0 when c scores none of the group.
struct LsaSeg {
  int64_t off;
  int len, j;
};
__host__ __device__ inline int lsa_first_cta(long long units, int grid, int NT, int g) {
  // the last CTA whose run starts at or before the group's first unit
  const long long x = static_cast<long long>(g) * NT;
  const long long c = ((x + 1) * grid + units - 1) / units - 1;
  return static_cast<int>(c < 0 ? 0 : (c >= grid ? grid - 1 : c));
}
__host__ __device__ inline LsaSeg lsa_segment(long long units, int grid, int NT, int g, int c, int cap2, int slack) {
  const long long gl = static_cast<long long>(g) * NT;
  const long long ub = units * c / grid, ue = units * (c + 1) / grid;
  const long long lo = (ub > gl ? ub : gl) - gl;
  const long long hi = (ue < gl + NT ? ue : gl + NT) - gl;
  LsaSeg s{0, 0, c - lsa_first_cta(units, grid, NT, g)};
  if (hi <= lo) return s;
  const long long a = static_cast<long long>(cap2) * lo / NT, b = static_cast<long long>(cap2) * hi / NT;
  s.off = a + static_cast<long long>(slack) * s.j;
  s.len = static_cast<int>(b - a) + slack;
  return s;
}
// The most CTAs one query group can meet (each CTA takes at least
// floor(units / grid) units).
inline int lsa_max_segments(long long units, int grid, int NT) {
  const long long per = units / grid > 0 ? units / grid : 1;
  const long long k = NT / per + 2;
  return static_cast<int>(k < grid ? k : grid);
}
// vis[t] = min(P, bpb * floor(q_pos[t] / block_keys)); n_samp[t] = ceil(vis[t] / stride) (if n_samp).
cudaError_t launch_lsa_visible(const int64_t* q_pos, int T, int block_keys, int bpb, int P, int stride, int32_t* vis,
                               int32_t* n_samp, cudaStream_t st);
// The grid size the LSA scan launches with (the filter form's segment count).
int dot_tc_grid(int T, int P, int num_sms);
// Pack each row's segments into cval / clab [T][cap] (nv[t] entries);
// flag rows that ran over or hold fewer than min(top_p, vis[t]).
cudaError_t launch_lsa_compact(const uint2* slist, const uint32_t* cnt, const DotParams& fp, int grid,
                               const int32_t* vis, int T, int top_p, int cap, float* cval, int32_t* clab, int32_t* nv,
                               int32_t* row_over, int* any_over, cudaStream_t st);
// The threshold form's fallback: the missed rows listed (ascending; -1 past
// the count) with run[c] = 1 for the chunks of `rows` list entries that hold
// any, then their queries and visible counts gathered into qbuf / vbuf [T]
// (zeros past the count), each chunk then scored in full and its picks
// written to the listed rows (launches that return at once when run_if[0] == 0).
cudaError_t launch_lsa_flag_list(const int32_t* row_over, int T, int rows, int n_chunks, int32_t* list,
                                 int32_t* count, int32_t* run, cudaStream_t st);
cudaError_t launch_lsa_gather_rows(const int32_t* list, const int32_t* count, int T, const uint16_t* q,
                                   const int32_t* vis, const int* run_if, uint16_t* qbuf, int32_t* vbuf,
                                   cudaStream_t st);
// The read list of each query: sinks below its window, the window, then the
// picked buckets' members best first (sinks and window skipped) up to budget.
cudaError_t launch_lsa_expand(const int32_t* picked, const int64_t* q_pos, int T, int top_p, const int32_t* off,
                              const int32_t* mem, int P, int block_keys, int n_sink, int budget, int32_t* keys_out,
                              int row_len, int32_t* n_out, cudaStream_t st);

// Source rows for the converting scorer.
enum SrcFormat : int { SRC_INT8 = 0, SRC_E4M3 = 1, SRC_BF16 = 2, SRC_PQ = 3 };
// PQ compact keys: kPqSub one-byte codes per key, sub-vector m (dimensions
// 4m..4m+3) = row code[m] of codebook m; codebooks fp16 [kPqSub][256][4].
constexpr int kPqSub = 32;

// Scoring of keys that are either int8 / fp8 e4m3 codes with a per-key fp32
// scale, or gathered bf16 rows.  Row j of problem b is key
//   rows == nullptr : b*N + j                      (contiguous)
//   rows != nullptr : b*key_stride + rows[b*N + j] (gathered; < 0 = padding)
//   out[b*N + j] = sum_h w[b,h] * relu(scale * (q[b,h] . code))   (or -inf)
struct CvtParams {
  const uint16_t* q;       // bf16 query rows (problem b, head h: row b*q_row_stride + h)
  const void* keys;        // base of the key rows
  const float* scale;      // per-key scale, indexed like the key rows (nullptr for bf16 / PQ)
  const uint16_t* books;   // PQ codebooks (fp16 bits, [32][256][4], 16-byte aligned) or nullptr
  const int32_t* rows;     // [B][N] gathered row ids or nullptr
  const int32_t* n_valid;  // [B] or nullptr (contiguous form only)
  const float* w;          // [B][H]
  float* out;              // [B][N]
  int64_t key_rows;        // gathered form: valid row ids are [0, key_rows)
  int64_t key_stride;      // gathered form: row offset of problem b is b*key_stride
  int64_t q_row_stride;    // q rows per problem (H for one query per problem)
  int B, N;
  int fmt;
  uint32_t* hist;          // [B][2048] selection histogram (counts added) or nullptr
};
cudaError_t launch_score_cvt(const CUtensorMap* qmap, const CvtParams& p, int num_sms, cudaStream_t st);
// 8-bit keys (int8 / e4m3, fmt SRC_INT8 / SRC_E4M3); kmap covers the contiguous
// key rows ([rows][128] bytes) and is ignored when p.rows gathers them.
cudaError_t launch_score_q8(const CUtensorMap* qmap, const CUtensorMap* kmap, const CvtParams& p, int num_sms,
                            cudaStream_t st);

// ---------------------------------------------------------------- top-k
// Row-wise top-k by (value desc, label asc); labels default to the column.
struct TopkParams {
  const float* scores = nullptr;     // row r starts at scores + r*ld
  int64_t ld = 0;
  const int32_t* n_valid = nullptr;  // [R] or nullptr: columns >= n_valid[r] - nv_offset are absent
  int nv_offset = 0;
  const int32_t* labels = nullptr;   // [R][ld_labels] or nullptr; label < 0 = absent
  int64_t ld_labels = 0;
  int label_base = 0;                // without labels, entry j is labelled label_base + j
  const uint32_t* hist = nullptr;    // [R][2048] counts of the top 11 order-code bits of the
                                     // present entries (from the scoring epilogue) or nullptr
  const int32_t* row_flag = nullptr; // [R] or nullptr: rows whose flag is 0 are left untouched
  const int32_t* out_row = nullptr;  // [R] or nullptr: row r's output goes to row out_row[r] (< 0: none)
  const int* run_if = nullptr;       // the launch does nothing unless *run_if != 0 (nullptr: always)
  int R = 0, N = 0, k = 0;
  int32_t* idx_out = nullptr;        // [R][k] labels, -1 padding
  float* val_out = nullptr;          // [R][k] values (bit copies), -inf padding; may be nullptr
  int64_t ld_out = 0;
};
cudaError_t launch_topk(const TopkParams& p, cudaStream_t st, int num_sms);

// ---------------------------------------------------------------- misc
// n_valid[t] = clamp((q_pos[t] + 1) / stride, 0, n_total)
cudaError_t launch_causal_counts(const int64_t* q_pos, int T, int stride, int n_total, int32_t* out,
                                 cudaStream_t st);

// Best-first bucket expansion: members of picked[t][0..top_p) in order until
// budget positions are held; cand[t][budget] padded with -1.
cudaError_t launch_expand(const int32_t* picked, int T, int top_p, const int32_t* off, const int32_t* mem,
                          int P, int budget, int32_t* cand, cudaStream_t st);

// Packs each row of the running prefill selection in place: row t of
// (val, lab) [T][ld] holds the first tile's top-k in columns [0, k) and, for
// each later tile j = 1 .. S, a segment of cap candidate slots at column
// k + (j-1)*cap with cnt[(j-1)*T + t] entries (min(cnt, cap); k entries -- the
// tile's recomputed top-k -- when row_over[(j-1)*T + t] is set).  The row's
// present entries are moved to its first nv[t] columns, in that order.
cudaError_t launch_pack_segments(float* val, int32_t* lab, int64_t ld, int T, int k, int S, int cap,
                                 const uint32_t* cnt, const int32_t* row_over, int32_t* nv, cudaStream_t st);

int read_and_clear_fault(cudaStream_t st, int* flags);
cudaError_t launch_wait_probe(uint64_t limit_ns, int* waited, cudaStream_t st);

}  // namespace lsi

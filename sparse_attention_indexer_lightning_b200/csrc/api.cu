// C ABI of the lightning-indexer selection library: argument checks,
// workspace carving, TMA descriptor set-up and the launch sequence of each
// search.  Every step of the path runs in the kernels of this library.
//
// The library is built as this single translation unit; the kernel headers
// (score_tc.cuh, score_cvt.cuh, topk.cuh, misc.cuh) are included below.

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "ls_indexer.h"
#include "misc.cuh"
#include "score_cvt.cuh"
#include "score_dot.cuh"
#include "score_tree.cuh"
#include "merge.cuh"
#include "sparse_attn.cuh"
#include "sparse_attn_tc.cuh"
#include "score_q8.cuh"
#include "score_tc.cuh"
#include "topk.cuh"

namespace {

using namespace lsi;

thread_local char g_err[512] = "";

ls_status fail(ls_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

#define LS_CHECK_ARG(cond, ...) \
  do {                          \
    if (!(cond)) return fail(LS_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define LS_CUDA(expr)                                                                               \
  do {                                                                                              \
    cudaError_t e_ = (expr);                                                                        \
    if (e_ != cudaSuccess) return fail(LS_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_));      \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- profiling
// When recording is on, every kernel launch of the library is bracketed by
// two CUDA events on its own stream; ls_profile_end() sums the durations per
// kernel name.
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
struct ProfSum {
  std::string name;
  double ms;
  long long launches;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<ProfSum> g_prof_sums;

struct ProfScope {
  ProfRec rec{};
  bool on = false;
  cudaStream_t st;
  ProfScope(const char* name, cudaStream_t s) : st(s) {
    if (!g_prof_on) return;
    rec.name = name;
    if (cudaEventCreate(&rec.a) != cudaSuccess) return;
    if (cudaEventCreate(&rec.b) != cudaSuccess) {
      cudaEventDestroy(rec.a);
      return;
    }
    on = cudaEventRecord(rec.a, st) == cudaSuccess;
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(rec.b, st);
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_recs.push_back(rec);
  }
};

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

int num_sms_current() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over [rows][128], box = 64 columns x box_rows, 128-byte swizzle.
ls_status make_bf16_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDim * 2)};
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LS_OK;
}

// 2-D map over [rows][128 bytes] (one 8-bit key or query head per row), box =
// 128 bytes x box_rows rows, 128-byte swizzle.  The bytes are described as 64
// 16-bit elements per row: the copy and the swizzle act on bytes either way.
ls_status make_u8_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows = kTileKeys) {
  auto fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDim)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kDim / 2), box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LS_OK;
}

// 2-D map over [rows][32 bytes] (PQ codes, one key per row), box = 32 bytes x
// 128 rows, no swizzle; the bytes are described as 16 16-bit elements.
ls_status make_pq_map(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kPqSub / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kPqSub)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kPqSub / 2), static_cast<cuuint32_t>(kTileKeys)};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LS_OK;
}

ls_status check_shape(int H, int d) {
  if (H != kHeads || d != kDim)
    return fail(LS_ERR_UNSUPPORTED, "only H=%d, d=%d are built (got H=%d, d=%d)", kHeads, kDim, H, d);
  return LS_OK;
}

cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// Scores of bf16 keys on the tensor cores (the TMA path), p filled by the
// caller apart from the shape.
ls_status score_tc_launch(const uint16_t* q, const uint16_t* keys, int B, int T, int N, ScoreParams p, cudaStream_t st,
                          const char* prof_name = nullptr) {
  if (B == 0 || T == 0 || N == 0) return LS_OK;
  const int qg = (T == 1) ? 1 : 8;
  CUtensorMap kmap, qmap;
  ls_status s = make_bf16_map(&kmap, keys, static_cast<uint64_t>(B) * N, kTileKeys);
  if (s != LS_OK) return s;
  s = make_bf16_map(&qmap, q, static_cast<uint64_t>(B) * T * kHeads, qg * kHeads);
  if (s != LS_OK) return s;
  p.B = B;
  p.T = T;
  p.N = N;
  ProfScope prof(prof_name ? prof_name : qg == 1 ? "score_tc_kernel<1>" : "score_tc_kernel<8>", st);
  LS_CUDA(launch_score_tc(qg, &kmap, &qmap, p, num_sms_current(), st));
  return LS_OK;
}

// 2-D map over [rows][64] bf16 vectors (128 bytes each: one swizzle row),
// box = 64 x box_rows, 128-byte swizzle.
ls_status make_vec64_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows,
                         uint64_t row_step = 1) {
  auto fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kLsaDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kLsaDim * 2 * row_step)};   // row i at base + i * row_step * 128 B
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kLsaDim), box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LS_OK;
}

// 2-D bf16 map over the latent / query rows [rows][576], box = 64 elements x
// box_rows, 128-byte swizzle (one 128-byte panel of box_rows rows per copy).
ls_status make_latent_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kAttnLatent), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kAttnLatent * 2)};
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LS_OK;
}

// The fp8 scorer's head weights: w * q_scale per (query, head), n values.
ls_status fold_scales(const float* w, const float* q_scale, int64_t n, float* w_eff, cudaStream_t st) {
  ProfScope prof("fold_scales_kernel", st);
  LS_CUDA(launch_fold_scales(w, q_scale, n, w_eff, st));
  return LS_OK;
}

// Scores of fp8 queries and keys on the tensor cores; p.w must hold w *
// q_scale (fold_scales), p is filled by the caller apart from the shape.
ls_status score_f8_launch(const uint8_t* q8, const uint8_t* keys, const float* key_scale, int B, int T, int N,
                          ScoreParams p, cudaStream_t st, const char* prof_name = nullptr) {
  if (B == 0 || T == 0 || N == 0) return LS_OK;
  CUtensorMap kmap, qmap;
  ls_status s = make_u8_map(&kmap, keys, static_cast<uint64_t>(B) * N, kTileKeys);
  if (s != LS_OK) return s;
  s = make_u8_map(&qmap, q8, static_cast<uint64_t>(B) * T * kHeads, 8 * kHeads);
  if (s != LS_OK) return s;
  p.B = B;
  p.T = T;
  p.N = N;
  p.key_scale = key_scale;
  ProfScope prof(prof_name ? prof_name : "score_tc_kernel<8,fp8>", st);
  LS_CUDA(launch_score_tc_f8(&kmap, &qmap, p, num_sms_current(), st));
  return LS_OK;
}

ls_status score_bf16(const uint16_t* q, const float* w, const uint16_t* keys, const int32_t* n_valid,
                     const int64_t* q_pos, int stride, int B, int T, int N, int key_base, int n_total, float* out,
                     int64_t ld_out, cudaStream_t st, uint32_t* hist = nullptr,
                     const int32_t* lim_rows = nullptr) {
  ScoreParams p;
  p.w = w;
  p.n_valid = n_valid;
  p.q_pos = q_pos;
  p.out = out;
  p.ld_out = ld_out;
  p.stride = stride;
  p.B = B;
  p.T = T;
  p.N = N;
  p.out_col0 = key_base;
  p.key_base = key_base;
  p.n_total = n_total;
  p.hist = hist;
  p.lim_rows = lim_rows;
  return score_tc_launch(q, keys, B, T, N, p, st);
}

ls_status score_convert(const uint16_t* q, int64_t q_row_stride, int64_t q_rows_total, const float* w,
                        const void* keys, const float* scale, const int32_t* rows, const int32_t* n_valid,
                        int64_t key_rows, int64_t key_stride, int B, int N, int fmt, float* out, cudaStream_t st,
                        uint32_t* hist = nullptr, const uint16_t* books = nullptr) {
  if (B == 0 || N == 0) return LS_OK;
  CUtensorMap qmap;
  ls_status s = make_bf16_map(&qmap, q, static_cast<uint64_t>(q_rows_total), kHeads);
  if (s != LS_OK) return s;
  CvtParams p;
  p.q = q;
  p.keys = keys;
  p.scale = scale;
  p.books = books;
  p.rows = rows;
  p.n_valid = n_valid;
  p.w = w;
  p.out = out;
  p.key_rows = key_rows;
  p.key_stride = key_stride;
  p.q_row_stride = q_row_stride;
  p.B = B;
  p.N = N;
  p.fmt = fmt;
  p.hist = hist;
  if (fmt == SRC_BF16) {
    ProfScope prof("score_cvt_kernel<bf16>", st);
    LS_CUDA(launch_score_cvt(&qmap, p, num_sms_current(), st));
    return LS_OK;
  }
  // 8-bit keys: contiguous rows ([B][key_stride][128], key_stride == N) come in
  // by 2-D TMA; gathered rows by per-row bulk copies (kmap unused)
  CUtensorMap kmap = qmap;
  if (rows == nullptr) {
    const uint64_t nrows = static_cast<uint64_t>(B) * static_cast<uint64_t>(key_stride);
    s = fmt == SRC_PQ ? make_pq_map(&kmap, keys, nrows) : make_u8_map(&kmap, keys, nrows);
    if (s != LS_OK) return s;
  }
  ProfScope prof(fmt == SRC_INT8 ? "score_q8_kernel<int8>" : fmt == SRC_PQ ? "score_q8_kernel<pq>"
                                                                           : "score_q8_kernel<e4m3>",
                 st);
  LS_CUDA(launch_score_q8(&qmap, &kmap, p, num_sms_current(), st));
  return LS_OK;
}

ls_status topk_launch(const TopkParams& p, cudaStream_t st, const char* prof_name = "topk_kernel") {
  ProfScope prof(prof_name, st);
  LS_CUDA(launch_topk(p, st, num_sms_current()));
  return LS_OK;
}

ls_status topk(const float* scores, int64_t ld, const int32_t* n_valid, const int32_t* labels, int64_t ld_labels,
               int R, int N, int k, int32_t* idx, float* val, int64_t ld_out, cudaStream_t st,
               const uint32_t* hist = nullptr) {
  TopkParams p;
  p.hist = hist;
  p.scores = scores;
  p.ld = ld;
  p.n_valid = n_valid;
  p.labels = labels;
  p.ld_labels = ld_labels;
  p.R = R;
  p.N = N;
  p.k = k;
  p.idx_out = idx;
  p.val_out = val;
  p.ld_out = ld_out;
  return topk_launch(p, st);
}

struct Carver {
  uint8_t* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used += align_up(count * sizeof(T));
    return p;
  }
};

}  // namespace

extern "C" {

const char* ls_last_error(void) { return g_err; }

int ls_version(void) { return 100; }

ls_status ls_device_status(int* flags, void* stream) {
  int h = 0;
  const int e = read_and_clear_fault(S(stream), &h);
  if (e != 0) return fail(LS_ERR_CUDA, "reading the fault word: %s", cudaGetErrorString(static_cast<cudaError_t>(e)));
  if (flags) *flags = h;
  if (h & FAULT_WAIT_TIMEOUT) return fail(LS_ERR_TIMEOUT, "a device wait exceeded its time limit");
  if (h & FAULT_BAD_INDEX) return fail(LS_ERR_INVALID_ARG, "a gathered row id was outside the key array");
  return LS_OK;
}

ls_status ls_indexer_score(const uint16_t* q, const float* w, const void* keys, int key_dtype,
                           const float* key_scale, const int32_t* n_valid, const int64_t* q_pos, int stride,
                           int B, int T, int H, int d, int N, float* scores, uint32_t* hist_out, void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(B >= 0 && T >= 0 && N >= 0, "negative size (B=%d T=%d N=%d)", B, T, N);
  if (B == 0 || T == 0 || N == 0) return LS_OK;
  LS_CHECK_ARG(q && w && keys && scores, "null tensor pointer");
  LS_CHECK_ARG(aligned16(q) && aligned16(w) && aligned16(keys), "q, w and keys must be 16-byte aligned");
  LS_CHECK_ARG(q_pos == nullptr || stride >= 1, "stride must be >= 1 with q_pos");
  if (hist_out && T != 1)
    return fail(LS_ERR_UNSUPPORTED, "hist_out is built for one query per sequence (T == 1)");
  if (key_dtype == LS_KEY_BF16) {
    return score_bf16(q, w, static_cast<const uint16_t*>(keys), n_valid, q_pos, stride, B, T, N, 0, N, scores, N,
                      S(stream), hist_out);
  }
  LS_CHECK_ARG(key_dtype == LS_KEY_FP8_E4M3 || key_dtype == LS_KEY_INT8, "unknown key_dtype %d", key_dtype);
  LS_CHECK_ARG(key_scale != nullptr, "FP8/INT8 keys need key_scale");
  if (T != 1 || q_pos != nullptr)
    return fail(LS_ERR_UNSUPPORTED, "FP8/INT8 keys are built for one query per sequence without q_pos");
  return score_convert(q, kHeads, static_cast<int64_t>(B) * kHeads, w, keys, key_scale, nullptr, n_valid, N, N, B, N,
                       key_dtype == LS_KEY_INT8 ? SRC_INT8 : SRC_E4M3, scores, S(stream), hist_out);
}

ls_status ls_topk_select(const float* scores, int64_t ld, const int32_t* n_valid, const uint32_t* hist, int R,
                         int N, int k, int32_t* idx_out, float* val_out, void* stream) {
  LS_CHECK_ARG(R >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(ld >= N, "ld (%lld) < N (%d)", static_cast<long long>(ld), N);
  if (R == 0) return LS_OK;
  LS_CHECK_ARG(idx_out && (scores || N == 0), "null tensor pointer");
  return topk(scores, ld, n_valid, nullptr, 0, R, N, k, idx_out, val_out, k, S(stream), hist);
}

size_t ls_decode_select_workspace_size(int B, int N) {
  if (B <= 0 || N <= 0) return 0;
  return align_up(static_cast<size_t>(B) * N * sizeof(float));  // the score rows
}

ls_status ls_decode_select(const uint16_t* q, const float* w, const uint16_t* keys, const int32_t* n_valid, int B,
                           int H, int d, int N, int k, int32_t* idx_out, float* val_out, void* ws,
                           size_t ws_bytes, void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(B >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  if (B == 0) return LS_OK;
  LS_CHECK_ARG(idx_out != nullptr, "null idx_out");
  const size_t need = ls_decode_select_workspace_size(B, N);
  if (ws_bytes < need || (need && !ws))
    return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  Carver cv(ws);
  float* sc = cv.take<float>(static_cast<size_t>(B) * N);
  if (N > 0) {
    LS_CHECK_ARG(q && w && keys, "null tensor pointer");
    LS_CHECK_ARG(aligned16(q) && aligned16(w) && aligned16(keys), "q, w and keys must be 16-byte aligned");
    // The top-k samples its own threshold; counting a histogram in the scan
    // epilogue costs the scan more than it saves the selection.
    s = score_bf16(q, w, keys, n_valid, nullptr, 1, B, 1, N, 0, N, sc, N, S(stream));
    if (s != LS_OK) return s;
  }
  return topk(sc, N, n_valid, nullptr, 0, B, N, k, idx_out, val_out, k, S(stream));
}

// Candidate slots per row for each tile after the first in the running top-k
// of the prefill.
int prefill_cand_cap(int k) { return 2 * k; }

// Row width of the running form's lists: the first tile's top-k, then one
// candidate segment per later tile.
int64_t prefill_list_width(int N, int tile_keys, int k) {
  const int ntiles = (N + tile_keys - 1) / tile_keys;
  return ntiles > 1 ? k + static_cast<int64_t>(ntiles - 1) * prefill_cand_cap(k) : 0;
}

size_t ls_prefill_select_workspace_size(int T, int N, int tile_keys, int k, int full_scores) {
  if (T <= 0 || N <= 0 || tile_keys <= 0 || k <= 0) return 0;
  // full_scores: the whole T x N score matrix (one top-k at the end), no lists
  const int tk = full_scores ? N : (tile_keys < N ? tile_keys : N);
  const int ntiles = (N + tile_keys - 1) / tile_keys;
  const int64_t ldc = full_scores ? 0 : prefill_list_width(N, tile_keys, k);
  const int64_t S = full_scores ? 0 : ntiles - 1;  // later tiles, each with its counters
  return align_up(static_cast<size_t>(T) * tk * sizeof(float)) +    // one tile of scores
         align_up(static_cast<size_t>(T) * ldc * sizeof(float)) +   // first tile's top-k + candidate segments
         align_up(static_cast<size_t>(T) * ldc * sizeof(int32_t)) +
         align_up(static_cast<size_t>(T) * sizeof(int32_t)) +       // eligible counts
         align_up(static_cast<size_t>(T) * sizeof(int32_t)) +       // packed list lengths
         align_up(static_cast<size_t>(S) * (static_cast<size_t>(T) * 2 * sizeof(int32_t) + sizeof(int)));  // counters, overflow flags
}

}  // extern "C"

namespace {

// History sources of the streamed prefill: how a tile of the history reaches
// a device buffer and how the keys in a buffer are scored.
struct Bf16History {
  const uint16_t* q;
  const uint16_t* hist;
  uint16_t* bufs[2];
  const char* overflow_name = "score_tc_kernel<8>:overflow";
  cudaError_t copy(int slot, int k0, int len, cudaStream_t xs) const {
    return cudaMemcpyAsync(bufs[slot], hist + static_cast<size_t>(k0) * kDim,
                           static_cast<size_t>(len) * kDim * sizeof(uint16_t), cudaMemcpyDefault, xs);
  }
  ls_status score(int slot, int T, int len, const ScoreParams& sp, cudaStream_t cs, const char* name) const {
    return score_tc_launch(q, bufs[slot], 1, T, len, sp, cs, name);
  }
};

// fp8 history: e4m3 codes [N][128] and fp32 scales [N]; a device buffer holds
// a tile's codes followed by its scales (at tile_keys * 128 bytes).
struct F8History {
  const uint8_t* q8;
  const uint8_t* hist;
  const float* hist_scale;
  uint8_t* bufs[2];
  int tile_keys;
  const char* overflow_name = "score_tc_kernel<8,fp8>:overflow";
  cudaError_t copy(int slot, int k0, int len, cudaStream_t xs) const {
    cudaError_t e = cudaMemcpyAsync(bufs[slot], hist + static_cast<size_t>(k0) * kDim, static_cast<size_t>(len) * kDim,
                                    cudaMemcpyDefault, xs);
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(bufs[slot] + static_cast<size_t>(tile_keys) * kDim, hist_scale + k0,
                           static_cast<size_t>(len) * sizeof(float), cudaMemcpyDefault, xs);
  }
  ls_status score(int slot, int T, int len, const ScoreParams& sp, cudaStream_t cs, const char* name) const {
    const float* ks = reinterpret_cast<const float*>(bufs[slot] + static_cast<size_t>(tile_keys) * kDim);
    return score_f8_launch(q8, bufs[slot], ks, 1, T, len, sp, cs, name);
  }
};

// The streamed prefill over tiles of tile_keys history keys: copy tile j on
// the copy stream while tile j-1 is scored; either every tile into the full
// T x N matrix and one top-k at the end, or a running top-k (tile 0 in full,
// later tiles through the filter form, then a merge).
template <class Src>
ls_status prefill_stream(const Src& src, Carver& cv, const float* w, const int64_t* q_pos, int T, int N, int stride,
                         int tile_keys, int k, int full_scores, int32_t* idx_out, float* val_out, cudaStream_t cs,
                         cudaStream_t xs) {
  const int tk = full_scores ? N : (tile_keys < N ? tile_keys : N);
  const int ntiles = (N + tile_keys - 1) / tile_keys;
  const int cap = prefill_cand_cap(k);
  const int64_t ldc = full_scores ? 0 : prefill_list_width(N, tile_keys, k);
  const int S = full_scores ? 0 : ntiles - 1;
  float* tile_sc = cv.take<float>(static_cast<size_t>(T) * tk);  // full_scores: the T x N matrix
  float* run_val = cv.take<float>(static_cast<size_t>(T) * ldc);
  int32_t* run_lab = cv.take<int32_t>(static_cast<size_t>(T) * ldc);
  int32_t* counts = cv.take<int32_t>(T);
  int32_t* nv = cv.take<int32_t>(T);
  // per later tile j (1..S): candidate counters [T], overflow flags [T], and
  // one "some row overflowed" word, zeroed once per call
  const size_t ctr_bytes = static_cast<size_t>(S) * (static_cast<size_t>(T) * 2 * sizeof(int32_t) + sizeof(int));
  uint8_t* ctr = cv.take<uint8_t>(ctr_bytes);
  uint32_t* cnt_all = reinterpret_cast<uint32_t*>(ctr);
  int32_t* over_all = reinterpret_cast<int32_t*>(ctr) + static_cast<size_t>(S) * T;
  int* any_all = reinterpret_cast<int*>(ctr) + static_cast<size_t>(S) * 2 * T;

  cudaEvent_t start_ev, copied[2], freed[2];
  LS_CUDA(cudaEventCreateWithFlags(&start_ev, cudaEventDisableTiming));
  for (int i = 0; i < 2; ++i) {
    LS_CUDA(cudaEventCreateWithFlags(&copied[i], cudaEventDisableTiming));
    LS_CUDA(cudaEventCreateWithFlags(&freed[i], cudaEventDisableTiming));
  }
  ls_status st = LS_OK;
  {
    ProfScope prof("causal_counts_kernel", cs);
    LS_CUDA(launch_causal_counts(q_pos, T, stride, N, counts, cs));
  }
  cudaError_t e = cudaSuccess;
  if (S > 0) e = cudaMemsetAsync(ctr, 0, ctr_bytes, cs);
  // Earlier work on the compute stream may still read the buffers.
  if (e == cudaSuccess) e = cudaEventRecord(start_ev, cs);
  if (e == cudaSuccess && xs != cs) e = cudaStreamWaitEvent(xs, start_ev, 0);
  for (int j = 0; j < ntiles && e == cudaSuccess && st == LS_OK; ++j) {
    const int slot = j & 1;
    const int k0 = j * tile_keys;
    const int len = (N - k0 < tile_keys) ? (N - k0) : tile_keys;
    const bool last = j + 1 == ntiles;
    if (j >= 2 && xs != cs) e = cudaStreamWaitEvent(xs, freed[slot], 0);
    if (e != cudaSuccess) break;
    e = src.copy(slot, k0, len, xs);
    if (e != cudaSuccess) break;
    if (xs != cs) {
      e = cudaEventRecord(copied[slot], xs);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, copied[slot], 0);
      if (e != cudaSuccess) break;
    }
    ScoreParams sp;
    sp.w = w;
    sp.q_pos = q_pos;
    sp.stride = stride;
    sp.key_base = k0;
    sp.n_total = N;
    sp.lim_rows = counts;
    TopkParams tp;                     // top-k of one full tile of scores
    tp.scores = tile_sc;
    tp.ld = tk;
    tp.n_valid = counts;
    tp.nv_offset = k0;
    tp.label_base = k0;
    tp.R = T;
    tp.N = len;
    tp.k = k;
    if (full_scores) {
      // every tile into its columns of the T x N matrix; one top-k at the end
      sp.out = tile_sc;
      sp.ld_out = N;
      sp.out_col0 = k0;
      st = src.score(slot, T, len, sp, cs, nullptr);
      if (st != LS_OK) break;
      if (last) {
        TopkParams fp;
        fp.scores = tile_sc;
        fp.ld = N;
        fp.n_valid = counts;
        fp.R = T;
        fp.N = N;
        fp.k = k;
        fp.idx_out = idx_out;
        fp.val_out = val_out;
        fp.ld_out = k;
        st = topk_launch(fp, cs);
        if (st != LS_OK) break;
      }
    } else if (j == 0) {
      // the first tile is scored in full; its exact top-k starts every row's
      // list, and the row's k-th entry there is its threshold for the rest
      sp.out = tile_sc;
      sp.ld_out = tk;
      st = src.score(slot, T, len, sp, cs, nullptr);
      if (st != LS_OK) break;
      tp.idx_out = last ? idx_out : run_lab;
      tp.val_out = last ? val_out : run_val;
      tp.ld_out = last ? k : ldc;
      st = topk_launch(tp, cs);
      if (st != LS_OK) break;
    } else {
      // later tiles append the keys that beat the row's threshold to the
      // row's segment for this tile
      const size_t seg = static_cast<size_t>(k) + static_cast<size_t>(j - 1) * cap;
      uint32_t* cnt = cnt_all + static_cast<size_t>(j - 1) * T;
      int32_t* row_over = over_all + static_cast<size_t>(j - 1) * T;
      int* any_over = any_all + (j - 1);
      ScoreParams fp = sp;
      fp.cand_val = run_val + seg;
      fp.cand_lab = run_lab + seg;
      fp.ld_cand = ldc;
      fp.cand_cap = cap;
      fp.kth_val = run_val + (k - 1);
      fp.kth_lab = run_lab + (k - 1);
      fp.ld_kth = ldc;
      fp.cand_cnt = cnt;
      fp.row_over = row_over;
      fp.any_over = any_over;
      st = src.score(slot, T, len, fp, cs, nullptr);
      if (st != LS_OK) break;
      // rows that ran out of slots: this tile again in full (the launches
      // return at once when no row overflowed), its top-k into the row's
      // segment
      sp.out = tile_sc;
      sp.ld_out = tk;
      sp.run_if = any_over;
      st = src.score(slot, T, len, sp, cs, src.overflow_name);
      if (st != LS_OK) break;
      tp.run_if = any_over;
      tp.row_flag = row_over;
      tp.idx_out = run_lab + seg;
      tp.val_out = run_val + seg;
      tp.ld_out = ldc;
      st = topk_launch(tp, cs, "topk_kernel:overflow");
      if (st != LS_OK) break;
      if (last) {
        // every row's lists packed into one prefix, then one exact top-k
        {
          ProfScope prof("pack_segments_kernel", cs);
          LS_CUDA(launch_pack_segments(run_val, run_lab, ldc, T, k, S, cap, cnt_all, over_all, nv, cs));
        }
        TopkParams mp;
        mp.scores = run_val;
        mp.ld = ldc;
        mp.n_valid = nv;
        mp.labels = run_lab;
        mp.ld_labels = ldc;
        mp.R = T;
        mp.N = static_cast<int>(ldc);
        mp.k = k;
        mp.idx_out = idx_out;
        mp.val_out = val_out;
        mp.ld_out = k;
        st = topk_launch(mp, cs);
        if (st != LS_OK) break;
      }
    }
    if (xs != cs) e = cudaEventRecord(freed[slot], cs);
  }
  // The copy stream must not run ahead of this call's last kernels.
  if (e == cudaSuccess && st == LS_OK && xs != cs) {
    e = cudaEventRecord(start_ev, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(xs, start_ev, 0);
  }
  cudaEventDestroy(start_ev);
  for (int i = 0; i < 2; ++i) {
    cudaEventDestroy(copied[i]);
    cudaEventDestroy(freed[i]);
  }
  if (st != LS_OK) return st;
  if (e != cudaSuccess) return fail(LS_ERR_CUDA, "history streaming: %s", cudaGetErrorString(e));
  return LS_OK;
}


}  // namespace

extern "C" {

ls_status ls_prefill_select_stream(const uint16_t* q, const float* w, const int64_t* q_pos, int T, int H, int d,
                                   const uint16_t* hist_k, int N, int stride, int tile_keys, uint16_t* buf0,
                                   uint16_t* buf1, int k, int full_scores, int32_t* idx_out, float* val_out,
                                   void* ws, size_t ws_bytes, void* compute_stream, void* copy_stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(T >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(stride >= 1, "stride must be >= 1");
  LS_CHECK_ARG(tile_keys >= 1, "tile_keys must be >= 1");
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q && w && q_pos && idx_out, "null tensor pointer");
  LS_CHECK_ARG(aligned16(q) && aligned16(w), "q and w must be 16-byte aligned");
  cudaStream_t cs = S(compute_stream);
  cudaStream_t xs = copy_stream ? S(copy_stream) : cs;
  if (N == 0) {  // no history: every row is padding
    TopkParams p;
    p.R = T;
    p.k = k;
    p.idx_out = idx_out;
    p.val_out = val_out;
    p.ld_out = k;
    return topk_launch(p, cs);
  }
  const size_t need = ls_prefill_select_workspace_size(T, N, tile_keys, k, full_scores);
  if (ws_bytes < need || (need && !ws))
    return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  LS_CHECK_ARG(hist_k && buf0 && buf1, "null history or buffer pointer");
  LS_CHECK_ARG(aligned16(buf0) && aligned16(buf1) && aligned16(hist_k), "history and buffers must be 16-byte aligned");
  cudaPointerAttributes attr;
  LS_CUDA(cudaPointerGetAttributes(&attr, hist_k));
  LS_CHECK_ARG(attr.type == cudaMemoryTypeHost || attr.type == cudaMemoryTypeDevice ||
                   attr.type == cudaMemoryTypeManaged,
               "hist_k must be pinned host memory or device memory (pageable memory cannot be streamed)");
  Carver cv(ws);
  Bf16History src{q, hist_k, {buf0, buf1}};
  return prefill_stream(src, cv, w, q_pos, T, N, stride, tile_keys, k, full_scores, idx_out, val_out, cs, xs);
}

size_t ls_indexer_score_fp8_workspace_size(int B, int T) {
  if (B <= 0 || T <= 0) return 0;
  return align_up(static_cast<size_t>(B) * T * kHeads * sizeof(float));  // w * q_scale
}

ls_status ls_indexer_score_fp8(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                               const float* k_scale, const int32_t* n_valid, const int64_t* q_pos, int stride, int B,
                               int T, int H, int d, int N, float* scores, void* ws, size_t ws_bytes, void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(B >= 0 && T >= 0 && N >= 0, "negative size (B=%d T=%d N=%d)", B, T, N);
  if (B == 0 || T == 0 || N == 0) return LS_OK;
  LS_CHECK_ARG(q8 && q_scale && w && k8 && k_scale && scores, "null tensor pointer");
  LS_CHECK_ARG(aligned16(q8) && aligned16(k8), "q8 and k8 must be 16-byte aligned");
  LS_CHECK_ARG(q_pos == nullptr || stride >= 1, "stride must be >= 1 with q_pos");
  const size_t need = ls_indexer_score_fp8_workspace_size(B, T);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  LS_CHECK_ARG(aligned16(ws), "workspace must be 16-byte aligned");
  cudaStream_t st = S(stream);
  float* w_eff = static_cast<float*>(ws);
  s = fold_scales(w, q_scale, static_cast<int64_t>(B) * T * kHeads, w_eff, st);
  if (s != LS_OK) return s;
  ScoreParams p;
  p.w = w_eff;
  p.n_valid = n_valid;
  p.q_pos = q_pos;
  p.out = scores;
  p.ld_out = N;
  p.stride = stride;
  p.n_total = N;
  return score_f8_launch(q8, k8, k_scale, B, T, N, p, st);
}

size_t ls_prefill_select_fp8_workspace_size(int T, int N, int tile_keys, int k, int full_scores) {
  const size_t base = ls_prefill_select_workspace_size(T, N, tile_keys, k, full_scores);
  if (base == 0) return 0;
  return base + align_up(static_cast<size_t>(T) * kHeads * sizeof(float));  // + w * q_scale, after the generic part
}

ls_status ls_prefill_select_stream_fp8(const uint8_t* q8, const float* q_scale, const float* w, const int64_t* q_pos,
                                       int T, int H, int d, const uint8_t* hist_k8, const float* hist_kscale, int N,
                                       int stride, int tile_keys, void* buf0, void* buf1, int k, int full_scores,
                                       int32_t* idx_out, float* val_out, void* ws, size_t ws_bytes,
                                       void* compute_stream, void* copy_stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(T >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(stride >= 1, "stride must be >= 1");
  LS_CHECK_ARG(tile_keys >= 1, "tile_keys must be >= 1");
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q8 && q_scale && w && q_pos && idx_out, "null tensor pointer");
  LS_CHECK_ARG(aligned16(q8), "q8 must be 16-byte aligned");
  cudaStream_t cs = S(compute_stream);
  cudaStream_t xs = copy_stream ? S(copy_stream) : cs;
  if (N == 0) {  // no history: every row is padding
    TopkParams p;
    p.R = T;
    p.k = k;
    p.idx_out = idx_out;
    p.val_out = val_out;
    p.ld_out = k;
    return topk_launch(p, cs);
  }
  const size_t need = ls_prefill_select_fp8_workspace_size(T, N, tile_keys, k, full_scores);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  LS_CHECK_ARG(aligned16(ws), "workspace must be 16-byte aligned");
  LS_CHECK_ARG(hist_k8 && hist_kscale && buf0 && buf1, "null history or buffer pointer");
  LS_CHECK_ARG(aligned16(buf0) && aligned16(buf1) && aligned16(hist_k8),
               "history codes and buffers must be 16-byte aligned");
  for (const void* hp : {static_cast<const void*>(hist_k8), static_cast<const void*>(hist_kscale)}) {
    cudaPointerAttributes attr;
    LS_CUDA(cudaPointerGetAttributes(&attr, hp));
    LS_CHECK_ARG(attr.type == cudaMemoryTypeHost || attr.type == cudaMemoryTypeDevice ||
                     attr.type == cudaMemoryTypeManaged,
                 "the history must be pinned host memory or device memory (pageable memory cannot be streamed)");
  }
  // w * q_scale sits at the end of the workspace, after the generic part
  float* w_eff = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + need -
                                          align_up(static_cast<size_t>(T) * kHeads * sizeof(float)));
  s = fold_scales(w, q_scale, static_cast<int64_t>(T) * kHeads, w_eff, cs);
  if (s != LS_OK) return s;
  Carver cv(ws);
  F8History src{q8, hist_k8, hist_kscale, {static_cast<uint8_t*>(buf0), static_cast<uint8_t*>(buf1)}, tile_keys};
  return prefill_stream(src, cv, w_eff, q_pos, T, N, stride, tile_keys, k, full_scores, idx_out, val_out, cs, xs);
}

size_t ls_two_stage_workspace_size(int B, int N, int shortlist) {
  if (B <= 0 || N <= 0 || shortlist <= 0) return 0;
  return align_up(static_cast<size_t>(B) * N * sizeof(float)) +
         align_up(static_cast<size_t>(B) * shortlist * sizeof(int32_t)) +
         align_up(static_cast<size_t>(B) * shortlist * sizeof(float)) +
         align_up(static_cast<size_t>(B) * kHistBins * sizeof(uint32_t));
}

// The two-stage search over either compact key form: int8 codes + per-key
// scale (coarse_fmt SRC_INT8) or PQ codes + codebooks (SRC_PQ).
static ls_status two_stage_run(const uint16_t* q, const float* w, const void* ck, const float* ck_scale,
                               const uint16_t* books, int coarse_fmt, const uint8_t* fk, const float* fk_scale,
                               const int32_t* n_valid, int B, int H, int d, int N, int shortlist, int k,
                               int32_t* idx_out, float* val_out, int32_t* shortlist_out, void* ws, size_t ws_bytes,
                               void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(B >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(shortlist >= k && shortlist <= kMaxTopK, "shortlist must be in [k, %d] (got %d)", kMaxTopK,
               shortlist);
  if (B == 0) return LS_OK;
  LS_CHECK_ARG(idx_out != nullptr, "null idx_out");
  const size_t need = ls_two_stage_workspace_size(B, N, shortlist);
  if (ws_bytes < need || (need && !ws))
    return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  Carver cv(ws);
  float* s_hat = cv.take<float>(static_cast<size_t>(B) * N);
  int32_t* short_ws = cv.take<int32_t>(static_cast<size_t>(B) * shortlist);
  float* exact = cv.take<float>(static_cast<size_t>(B) * shortlist);
  int32_t* sl = shortlist_out ? shortlist_out : short_ws;
  cudaStream_t st = S(stream);
  if (N > 0) {
    const bool pq = coarse_fmt == SRC_PQ;
    LS_CHECK_ARG(q && w && ck && fk && fk_scale && (pq ? books != nullptr : ck_scale != nullptr),
                 "null tensor pointer");
    LS_CHECK_ARG(aligned16(q) && aligned16(w) && aligned16(ck) && aligned16(fk) && aligned16(fk_scale) &&
                     (pq ? aligned16(books) : aligned16(ck_scale)),
                 "tensors must be 16-byte aligned");
    // coarse pass over the compact keys
    s = score_convert(q, kHeads, static_cast<int64_t>(B) * kHeads, w, ck, ck_scale, nullptr, n_valid, N, N, B, N,
                      coarse_fmt, s_hat, st, nullptr, books);
    if (s != LS_OK) return s;
  }
  // shortlist: top-S positions by coarse score
  s = topk(s_hat, N, n_valid, nullptr, 0, B, N, shortlist, sl, nullptr, shortlist, st);
  if (s != LS_OK) return s;
  if (N > 0) {
    // exact re-rank: gather the shortlist's fp8 keys, score with the full query
    s = score_convert(q, kHeads, static_cast<int64_t>(B) * kHeads, w, fk, fk_scale, sl, nullptr, N, N, B, shortlist,
                      SRC_E4M3, exact, st);
    if (s != LS_OK) return s;
  }
  return topk(exact, shortlist, nullptr, sl, shortlist, B, shortlist, k, idx_out, val_out, k, st);
}

ls_status ls_decode_two_stage_select(const uint16_t* q, const float* w, const int8_t* ck, const float* ck_scale,
                                     const uint8_t* fk, const float* fk_scale, const int32_t* n_valid, int B,
                                     int H, int d, int N, int shortlist, int k, int32_t* idx_out, float* val_out,
                                     int32_t* shortlist_out, void* ws, size_t ws_bytes, void* stream) {
  return two_stage_run(q, w, ck, ck_scale, nullptr, SRC_INT8, fk, fk_scale, n_valid, B, H, d, N, shortlist, k,
                       idx_out, val_out, shortlist_out, ws, ws_bytes, stream);
}

ls_status ls_decode_two_stage_pq_select(const uint16_t* q, const float* w, const uint8_t* pq_codes,
                                        const uint16_t* pq_books, const uint8_t* fk, const float* fk_scale,
                                        const int32_t* n_valid, int B, int H, int d, int N, int shortlist, int k,
                                        int32_t* idx_out, float* val_out, int32_t* shortlist_out, void* ws,
                                        size_t ws_bytes, void* stream) {
  return two_stage_run(q, w, pq_codes, nullptr, pq_books, SRC_PQ, fk, fk_scale, n_valid, B, H, d, N, shortlist, k,
                       idx_out, val_out, shortlist_out, ws, ws_bytes, stream);
}

ls_status ls_indexer_score_pq(const uint16_t* q, const float* w, const uint8_t* pq_codes, const uint16_t* pq_books,
                              const int32_t* n_valid, int B, int H, int d, int N, float* scores, void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(B >= 0 && N >= 0, "negative size (B=%d N=%d)", B, N);
  if (B == 0 || N == 0) return LS_OK;
  LS_CHECK_ARG(q && w && pq_codes && pq_books && scores, "null tensor pointer");
  LS_CHECK_ARG(aligned16(q) && aligned16(w) && aligned16(pq_codes) && aligned16(pq_books),
               "q, w, codes and codebooks must be 16-byte aligned");
  return score_convert(q, kHeads, static_cast<int64_t>(B) * kHeads, w, pq_codes, nullptr, nullptr, n_valid, N, N, B,
                       N, SRC_PQ, scores, S(stream), nullptr, pq_books);
}

size_t ls_bucket_workspace_size(int T, int P, int top_p, int budget) {
  if (T <= 0 || P <= 0 || top_p <= 0 || budget <= 0) return 0;
  return align_up(static_cast<size_t>(T) * P * sizeof(float)) +
         align_up(static_cast<size_t>(T) * top_p * sizeof(int32_t)) +
         align_up(static_cast<size_t>(T) * budget * sizeof(int32_t)) +
         align_up(static_cast<size_t>(T) * budget * sizeof(float));
}

ls_status ls_bucket_select(const uint16_t* q, const float* w, const uint16_t* centroids, const int32_t* bucket_off,
                           const int32_t* bucket_mem, const uint16_t* keys, int T, int H, int d, int P, int N,
                           int top_p, int budget, int k, int32_t* idx_out, float* val_out, int32_t* picked_out,
                           void* ws, size_t ws_bytes, void* stream) {
  ls_status s = check_shape(H, d);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(T >= 0 && P >= 0 && N >= 0, "negative size");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(top_p >= 1 && top_p <= kMaxTopK, "top_p must be in [1, %d] (got %d)", kMaxTopK, top_p);
  LS_CHECK_ARG(budget >= k, "budget (%d) must be >= k (%d)", budget, k);
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(idx_out != nullptr, "null idx_out");
  const size_t need = ls_bucket_workspace_size(T, P, top_p, budget);
  if (ws_bytes < need || (need && !ws))
    return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  Carver cv(ws);
  float* cscore = cv.take<float>(static_cast<size_t>(T) * P);
  int32_t* picked_ws = cv.take<int32_t>(static_cast<size_t>(T) * top_p);
  int32_t* cand = cv.take<int32_t>(static_cast<size_t>(T) * budget);
  float* exact = cv.take<float>(static_cast<size_t>(T) * budget);
  int32_t* picked = picked_out ? picked_out : picked_ws;
  cudaStream_t st = S(stream);
  if (P > 0) {
    LS_CHECK_ARG(q && w && centroids && bucket_off && bucket_mem, "null tensor pointer");
    LS_CHECK_ARG(aligned16(q) && aligned16(w) && aligned16(centroids), "q, w and centroids must be 16-byte aligned");
    s = score_bf16(q, w, centroids, nullptr, nullptr, 1, 1, T, P, 0, P, cscore, P, st);
    if (s != LS_OK) return s;
  }
  s = topk(cscore, P, nullptr, nullptr, 0, T, P, top_p, picked, nullptr, top_p, st);
  if (s != LS_OK) return s;
  {
    ProfScope prof("expand_kernel", st);
    LS_CUDA(launch_expand(picked, T, top_p, bucket_off, bucket_mem, P, budget, cand, st));
  }
  if (N > 0) {
    LS_CHECK_ARG(keys && aligned16(keys), "keys must be a 16-byte aligned device pointer");
    s = score_convert(q, kHeads, static_cast<int64_t>(T) * kHeads, w, keys, nullptr, cand, nullptr, N, 0, T, budget,
                      SRC_BF16, exact, st);
    if (s != LS_OK) return s;
  }
  return topk(exact, budget, nullptr, cand, budget, T, budget, k, idx_out, val_out, k, st);
}

}  // extern "C"

namespace {

// Sampled-threshold parameters of the LSA search: every stride-th bucket is
// sampled (stride = top_p / 16) and the 32nd best sample sets the threshold,
// so about 2 * top_p buckets of a row clear it (the count's relative spread is
// about 1/sqrt(32): a row comes up short with a probability of a few in a
// thousand); a row lists up to 4 * top_p.
struct LsaThreshold {
  int stride, rank, cap;
  explicit LsaThreshold(int top_p)
      : stride(top_p / 16 > 1 ? top_p / 16 : 1), rank(32), cap(4 * top_p) {}
};

// List segments of the filtered scan: each row's list holds 2 * cap entries
// shared out among the scan's CTAs in proportion to the centroid tiles of
// the row each one scores (about 4x the expected count of its share of the
// 2 * top_p listed buckets), plus 64 slack entries per CTA.
struct LsaSegments {
  int grid, nseg, cap2, slack;
  long long per_row;
  LsaSegments(int T, int P, int cap) {
    grid = dot_tc_grid(T, P, num_sms_current());
    const int NT = (P + DotCfg::BM - 1) / DotCfg::BM;
    const long long units = static_cast<long long>((T + DotCfg::QB - 1) / DotCfg::QB) * NT;
    nseg = grid > 0 ? lsa_max_segments(units, grid, NT) : 1;
    cap2 = 2 * cap;
    slack = 64;
    per_row = cap2 + static_cast<long long>(slack) * nseg;
  }
};

// The threshold form's fallback scores the missed rows in full, `rows` of
// them at a time: at most kLsaFallbackBytes of scores (a multiple of the
// scorer's 256-query group when that many fit), unless the caller asks for
// fewer rows.
constexpr size_t kLsaFallbackBytes = size_t(4) << 30;
struct LsaFallback {
  int rows, chunks;
  LsaFallback(int T, int P, int fallback_rows) {
    long long r = static_cast<long long>(kLsaFallbackBytes / (sizeof(float) * static_cast<size_t>(P > 0 ? P : 1)));
    if (r >= DotCfg::QB) r -= r % DotCfg::QB;
    if (fallback_rows > 0 && fallback_rows < r) r = fallback_rows;
    if (r > T) r = T;
    if (r < 1) r = 1;
    rows = static_cast<int>(r);
    chunks = (T + rows - 1) / rows;
  }
};

struct LsaWorkspace {
  float* sc;        // the full-matrix form: [T][P] scores; the threshold form: [rows][P] of the fallback
  int32_t* vis;     // [T]
  int32_t* nsamp;   // [T]
  int32_t* picked;  // [T][top_p]
  float* ss;        // [T][n_samp] sample scores
  float* sv;        // [T][rank] best samples
  int32_t* si;      // [T][rank]
  uint2* slist;     // [T][per_row] the scan's list segments, (score bits, bucket) pairs
  uint32_t* scnt;   // [T][nseg][4]
  float* cval;      // [T][cap] packed lists
  int32_t* clab;
  int32_t* nv;      // [T]
  uint8_t* ctr;     // row_over [T], any_over
  int32_t* fb_list; // [T] missed rows (-1 after the count), then the count, then the chunk flags
  int32_t* fb_count;
  int32_t* fb_run;
  uint16_t* fb_q;   // [T][64] their index queries, in list order
  int32_t* fb_vis;  // [T] their visible counts
  size_t ctr_bytes;
  size_t scnt_bytes;
  size_t used;
};

LsaWorkspace carve_lsa(void* ws, int T, int P, int top_p, int threshold, int fallback_rows) {
  Carver cv(ws);
  LsaWorkspace w{};
  const LsaThreshold th(top_p);
  const int n_samp = (P + th.stride - 1) / th.stride;
  const LsaFallback fb(T, P, fallback_rows);
  w.sc = cv.take<float>(static_cast<size_t>(threshold ? fb.rows : T) * P);
  w.vis = cv.take<int32_t>(T);
  w.nsamp = cv.take<int32_t>(T);
  w.picked = cv.take<int32_t>(static_cast<size_t>(T) * top_p);
  if (threshold) {
    w.ss = cv.take<float>(static_cast<size_t>(T) * n_samp);
    w.sv = cv.take<float>(static_cast<size_t>(T) * th.rank);
    w.si = cv.take<int32_t>(static_cast<size_t>(T) * th.rank);
    const LsaSegments sg(T, P, th.cap);
    w.slist = cv.take<uint2>(static_cast<size_t>(T) * sg.per_row);
    w.scnt_bytes = static_cast<size_t>(T) * sg.nseg * 4 * sizeof(uint32_t);
    w.scnt = cv.take<uint32_t>(static_cast<size_t>(T) * sg.nseg * 4);
    w.cval = cv.take<float>(static_cast<size_t>(T) * th.cap);
    w.clab = cv.take<int32_t>(static_cast<size_t>(T) * th.cap);
    w.nv = cv.take<int32_t>(T);
    w.ctr_bytes = static_cast<size_t>(T) * sizeof(int32_t) + sizeof(int);   // row flags, then the any-row flag
    w.ctr = cv.take<uint8_t>(w.ctr_bytes);
    w.fb_list = cv.take<int32_t>(T);
    w.fb_count = cv.take<int32_t>(1);
    w.fb_run = cv.take<int32_t>(fb.chunks);
    w.fb_q = cv.take<uint16_t>(static_cast<size_t>(T) * kLsaDim);
    w.fb_vis = cv.take<int32_t>(T);
  }
  w.used = cv.used;
  return w;
}

}  // namespace

extern "C" {

size_t ls_lsa_flat_workspace_size(int T, int P, int top_p, int threshold, int fallback_rows) {
  if (T <= 0 || top_p <= 0 || P < 0) return 0;
  return carve_lsa(nullptr, T, P, top_p, threshold, fallback_rows).used;
}

ls_status ls_lsa_flat_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                             const int32_t* bucket_off, const int32_t* bucket_mem, int T, int d, int P,
                             int block_keys, int buckets_per_block, int n_sink, int top_p, int budget, int threshold,
                             int fallback_rows, int32_t* keys_out, int32_t* n_out, int32_t* picked_out, void* ws,
                             size_t ws_bytes, void* stream) {
  if (d != kLsaDim) return fail(LS_ERR_UNSUPPORTED, "only d=%d is built for the LSA index space (got %d)", kLsaDim, d);
  LS_CHECK_ARG(T >= 0 && P >= 0, "negative size");
  LS_CHECK_ARG(block_keys >= 1 && buckets_per_block >= 1, "block_keys and buckets_per_block must be >= 1");
  LS_CHECK_ARG(n_sink >= 0 && budget >= 1, "n_sink must be >= 0 and budget >= 1");
  LS_CHECK_ARG(top_p >= 1 && top_p <= kMaxTopK, "top_p must be in [1, %d] (got %d)", kMaxTopK, top_p);
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q_pos && keys_out && n_out, "null tensor pointer");
  const size_t need = ls_lsa_flat_workspace_size(T, P, top_p, threshold, fallback_rows);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  const LsaWorkspace w = carve_lsa(ws, T, P, top_p, threshold, fallback_rows);
  const LsaThreshold th(top_p);
  int32_t* picked = picked_out ? picked_out : w.picked;
  cudaStream_t st = S(stream);
  {
    ProfScope prof("lsa_visible_kernel", st);
    LS_CUDA(launch_lsa_visible(q_pos, T, block_keys, buckets_per_block, P, th.stride, w.vis,
                               threshold ? w.nsamp : nullptr, st));
  }
  if (P > 0) {
    LS_CHECK_ARG(q_idx && centroids && bucket_off && bucket_mem, "null tensor pointer");
    LS_CHECK_ARG(aligned16(q_idx) && aligned16(centroids), "q_idx and centroids must be 16-byte aligned");
    CUtensorMap cmap, qmap;
    ls_status s = make_vec64_map(&cmap, centroids, static_cast<uint64_t>(P), kTileKeys);
    if (s != LS_OK) return s;
    s = make_vec64_map(&qmap, q_idx, static_cast<uint64_t>(T), DotCfg::QB);
    if (s != LS_OK) return s;
    DotParams full;
    full.T = T;
    full.P = P;
    full.out = w.sc;
    full.ld_out = P;
    TopkParams tp;                        // top-p of each row's visible prefix (padding -1)
    tp.scores = w.sc;
    tp.ld = P;
    tp.n_valid = w.vis;
    tp.R = T;
    tp.N = P;
    tp.k = top_p;
    tp.idx_out = picked;
    tp.ld_out = top_p;
    if (!threshold) {
      {
        ProfScope prof("dot_tc_kernel", st);
        LS_CUDA(launch_dot_tc(&cmap, &qmap, full, num_sms_current(), st));
      }
      s = topk_launch(tp, st);
      if (s != LS_OK) return s;
    } else {
      // 1. thresholds from a sample of every stride-th bucket, scored by the
      //    same tensor-core scorer through a map that steps stride rows
      const int n_samp = (P + th.stride - 1) / th.stride;
      {
        CUtensorMap smap;
        s = make_vec64_map(&smap, centroids, static_cast<uint64_t>(n_samp), kTileKeys,
                           static_cast<uint64_t>(th.stride));
        if (s != LS_OK) return s;
        DotParams sd;
        sd.T = T;
        sd.P = n_samp;
        sd.out = w.ss;
        sd.ld_out = n_samp;
        ProfScope prof("dot_tc_kernel:sample", st);
        LS_CUDA(launch_dot_tc(&smap, &qmap, sd, num_sms_current(), st));
      }
      TopkParams sp;
      sp.scores = w.ss;
      sp.ld = n_samp;
      sp.n_valid = w.nsamp;
      sp.R = T;
      sp.N = n_samp;
      sp.k = th.rank;
      sp.idx_out = w.si;
      sp.val_out = w.sv;
      sp.ld_out = th.rank;
      s = topk_launch(sp, st, "topk_kernel:sample");
      if (s != LS_OK) return s;
      // 2. the scan lists the buckets that reach the threshold
      int32_t* row_over = reinterpret_cast<int32_t*>(w.ctr);
      int* any_over = reinterpret_cast<int*>(w.ctr) + static_cast<size_t>(T);
      LS_CUDA(cudaMemsetAsync(w.ctr, 0, w.ctr_bytes, st));
      LS_CUDA(cudaMemsetAsync(w.scnt, 0, w.scnt_bytes, st));
      const LsaSegments sg(T, P, th.cap);
      DotParams fp;
      fp.T = T;
      fp.P = P;
      fp.vis = w.vis;
      fp.tau = w.sv + (th.rank - 1);
      fp.ld_tau = th.rank;
      fp.cand_list = w.slist;
      fp.ld_cand = sg.per_row;
      fp.nseg = sg.nseg;
      fp.cap2 = sg.cap2;
      fp.slack = sg.slack;
      fp.cand_cnt = w.scnt;
      fp.row_over = row_over;
      fp.any_over = any_over;
      {
        ProfScope prof("dot_tc_kernel:filter", st);
        LS_CUDA(launch_dot_tc(&cmap, &qmap, fp, num_sms_current(), st));
      }
      {
        ProfScope prof("lsa_compact_kernel", st);
        LS_CUDA(launch_lsa_compact(w.slist, w.scnt, fp, sg.grid, w.vis, T, top_p, th.cap, w.cval, w.clab,
                                   w.nv, row_over, any_over, st));
      }
      // 3. top-p of each list
      TopkParams cp;
      cp.scores = w.cval;
      cp.ld = th.cap;
      cp.n_valid = w.nv;
      cp.labels = w.clab;
      cp.ld_labels = th.cap;
      cp.R = T;
      cp.N = th.cap;
      cp.k = top_p;
      cp.idx_out = picked;
      cp.ld_out = top_p;
      s = topk_launch(cp, st);
      if (s != LS_OK) return s;
      // 4. rows whose list ran over or came up short: listed, their queries
      //    gathered, then scored in full fb.rows at a time, each chunk's
      //    top-p written to its listed rows (the two launches of a chunk that
      //    holds none of them return at once)
      const LsaFallback fb(T, P, fallback_rows);
      {
        ProfScope prof("lsa_flag_list_kernel", st);
        LS_CUDA(launch_lsa_flag_list(row_over, T, fb.rows, fb.chunks, w.fb_list, w.fb_count, w.fb_run, st));
      }
      {
        ProfScope prof("lsa_gather_rows_kernel", st);
        LS_CUDA(launch_lsa_gather_rows(w.fb_list, w.fb_count, T, q_idx, w.vis, any_over, w.fb_q, w.fb_vis, st));
      }
      for (int c = 0; c < fb.chunks; ++c) {
        const int32_t* run = w.fb_run + c;
        const int c0 = c * fb.rows;
        const int rows = std::min(fb.rows, T - c0);
        CUtensorMap fqmap;
        s = make_vec64_map(&fqmap, w.fb_q + static_cast<size_t>(c0) * kLsaDim, static_cast<uint64_t>(rows),
                           DotCfg::QB);
        if (s != LS_OK) return s;
        DotParams fd;
        fd.T = rows;
        fd.P = P;
        fd.out = w.sc;
        fd.ld_out = P;
        fd.run_if = run;
        fd.live_rows = w.fb_count;            // only the chunk's listed rows are scored
        fd.live_base = c0;
        {
          ProfScope prof("dot_tc_kernel:fallback", st);
          LS_CUDA(launch_dot_tc(&cmap, &fqmap, fd, num_sms_current(), st));
        }
        TopkParams fk;
        fk.scores = w.sc;
        fk.ld = P;
        fk.n_valid = w.fb_vis + c0;
        fk.R = rows;
        fk.N = P;
        fk.k = top_p;
        fk.out_row = w.fb_list + c0;
        fk.idx_out = picked;
        fk.ld_out = top_p;
        fk.run_if = run;
        s = topk_launch(fk, st, "topk_kernel:fallback");
        if (s != LS_OK) return s;
      }
    }
  } else {
    TopkParams tp;                        // nothing visible anywhere: every row is padding
    tp.R = T;
    tp.k = top_p;
    tp.idx_out = picked;
    tp.ld_out = top_p;
    ls_status s = topk_launch(tp, st);
    if (s != LS_OK) return s;
  }
  ProfScope prof("lsa_expand_kernel", st);
  LS_CUDA(launch_lsa_expand(picked, q_pos, T, top_p, bucket_off, bucket_mem, P, block_keys, n_sink, budget, keys_out,
                            n_sink + block_keys + budget, n_out, st));
  return LS_OK;
}

size_t ls_lsa_tree_workspace_size(int T, int P1, int beam, int fanout, int node_block, int top_p) {
  if (T <= 0 || beam <= 0 || fanout <= 0 || node_block <= 0 || top_p <= 0 || P1 < 0) return 0;
  const size_t cap = static_cast<size_t>(beam) * fanout + node_block;
  return align_up(static_cast<size_t>(T) * P1 * sizeof(float)) +       // node scores
         align_up(static_cast<size_t>(T) * sizeof(int32_t)) * 3 +       // visible buckets, nodes, list lengths
         align_up(static_cast<size_t>(T) * beam * sizeof(int32_t)) +    // the beam
         align_up(static_cast<size_t>(T) * cap * sizeof(float)) +       // candidate scores
         align_up(static_cast<size_t>(T) * cap * sizeof(int32_t)) +     // candidate buckets
         align_up(static_cast<size_t>(T) * top_p * sizeof(int32_t));    // picked buckets
}

ls_status ls_lsa_tree_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                             const uint16_t* node_centroids, const int32_t* bucket_off, const int32_t* bucket_mem,
                             int T, int d, int P, int P1, int block_keys, int buckets_per_block, int node_block,
                             int fanout, int beam, int n_sink, int top_p, int budget, int32_t* keys_out,
                             int32_t* n_out, int32_t* picked_out, int32_t* beam_out, void* ws, size_t ws_bytes,
                             void* stream) {
  if (d != kLsaDim) return fail(LS_ERR_UNSUPPORTED, "only d=%d is built for the LSA index space (got %d)", kLsaDim, d);
  LS_CHECK_ARG(T >= 0 && P >= 0 && P1 >= 0, "negative size");
  LS_CHECK_ARG(block_keys >= 1 && buckets_per_block >= 1, "block_keys and buckets_per_block must be >= 1");
  LS_CHECK_ARG(fanout >= 1 && node_block >= fanout && node_block % fanout == 0,
               "node_block must be a positive multiple of fanout");
  LS_CHECK_ARG(static_cast<int64_t>(P1) * fanout <= P, "P1 * fanout (%lld) exceeds P (%d)",
               static_cast<long long>(P1) * fanout, P);
  LS_CHECK_ARG(n_sink >= 0 && budget >= 1, "n_sink must be >= 0 and budget >= 1");
  LS_CHECK_ARG(top_p >= 1 && top_p <= kMaxTopK, "top_p must be in [1, %d] (got %d)", kMaxTopK, top_p);
  LS_CHECK_ARG(beam >= 1 && beam <= kMaxTopK, "beam must be in [1, %d] (got %d)", kMaxTopK, beam);
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q_idx && q_pos && centroids && bucket_off && bucket_mem && keys_out && n_out, "null tensor pointer");
  LS_CHECK_ARG(P1 == 0 || node_centroids != nullptr, "null node_centroids");
  LS_CHECK_ARG(aligned16(q_idx) && aligned16(centroids) && (P1 == 0 || aligned16(node_centroids)),
               "q_idx and the centroids must be 16-byte aligned");
  const size_t need = ls_lsa_tree_workspace_size(T, P1, beam, fanout, node_block, top_p);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  const int cap = beam * fanout + node_block;
  Carver cv(ws);
  float* sc1 = cv.take<float>(static_cast<size_t>(T) * P1);
  int32_t* vis = cv.take<int32_t>(T);
  int32_t* vis_nodes = cv.take<int32_t>(T);
  int32_t* nv = cv.take<int32_t>(T);
  int32_t* beam_ws = cv.take<int32_t>(static_cast<size_t>(T) * beam);
  float* cval = cv.take<float>(static_cast<size_t>(T) * cap);
  int32_t* clab = cv.take<int32_t>(static_cast<size_t>(T) * cap);
  int32_t* picked_ws = cv.take<int32_t>(static_cast<size_t>(T) * top_p);
  int32_t* bm = beam_out ? beam_out : beam_ws;
  int32_t* picked = picked_out ? picked_out : picked_ws;
  cudaStream_t st = S(stream);
  {
    ProfScope prof("lsa_tree_visible_kernel", st);
    LS_CUDA(launch_lsa_tree_visible(q_pos, T, block_keys, buckets_per_block, P, node_block, fanout, P1, vis, vis_nodes,
                                    st));
  }
  // the beam: the best node buckets among each query's visible ones
  if (P1 > 0) {
    CUtensorMap cmap, qmap;
    ls_status s = make_vec64_map(&cmap, node_centroids, static_cast<uint64_t>(P1), kTileKeys);
    if (s != LS_OK) return s;
    s = make_vec64_map(&qmap, q_idx, static_cast<uint64_t>(T), DotCfg::QB);
    if (s != LS_OK) return s;
    DotParams dp;
    dp.T = T;
    dp.P = P1;
    dp.out = sc1;
    dp.ld_out = P1;
    ProfScope prof("dot_tc_kernel:nodes", st);
    LS_CUDA(launch_dot_tc(&cmap, &qmap, dp, num_sms_current(), st));
  }
  TopkParams bp;
  bp.scores = sc1;
  bp.ld = P1;
  bp.n_valid = vis_nodes;
  bp.R = T;
  bp.N = P1;
  bp.k = beam;
  bp.idx_out = bm;
  bp.ld_out = beam;
  ls_status s = topk_launch(bp, st, "topk_kernel:beam");
  if (s != LS_OK) return s;
  // the beam's children and the uncovered buckets, scored; their top-p
  {
    ProfScope prof("lsa_tree_candidates_kernel", st);
    LS_CUDA(launch_lsa_tree_candidates(q_idx, centroids, bm, beam, vis, vis_nodes, T, fanout, cap, cval, clab, nv, st));
  }
  TopkParams cp;
  cp.scores = cval;
  cp.ld = cap;
  cp.n_valid = nv;
  cp.labels = clab;
  cp.ld_labels = cap;
  cp.R = T;
  cp.N = cap;
  cp.k = top_p;
  cp.idx_out = picked;
  cp.ld_out = top_p;
  s = topk_launch(cp, st);
  if (s != LS_OK) return s;
  ProfScope prof("lsa_expand_kernel", st);
  LS_CUDA(launch_lsa_expand(picked, q_pos, T, top_p, bucket_off, bucket_mem, P, block_keys, n_sink, budget, keys_out,
                            n_sink + block_keys + budget, n_out, st));
  return LS_OK;
}

}  // extern "C"

namespace {

// The shape of a tree search over several node levels: level sizes
// (size[0] = P), the start level (the lowest with at most start_nodes node
// buckets, else the top one) and the candidate list width of the levels
// below it (the beam's children plus the most uncovered entries a level can
// hold: less than a node block, or what the level above leaves uncovered when
// it is cut short).
struct TreePlan {
  int L = 0, start = 0;
  int size[kMaxTreeLevels + 1] = {};
  long long cap = 0;
};

ls_status tree_plan(int P, const int* level_sizes, int L, int node_block, int fanout, int beam, int start_nodes,
                    TreePlan* tp) {
  LS_CHECK_ARG(L >= 1 && L <= kMaxTreeLevels, "L must be in [1, %d] (got %d)", kMaxTreeLevels, L);
  LS_CHECK_ARG(level_sizes != nullptr, "null level_sizes");
  LS_CHECK_ARG(P >= 0, "negative size");
  LS_CHECK_ARG(fanout >= 1 && node_block >= fanout && node_block % fanout == 0,
               "node_block must be a positive multiple of fanout");
  LS_CHECK_ARG(beam >= 1 && beam <= kMaxTopK, "beam must be in [1, %d] (got %d)", kMaxTopK, beam);
  LS_CHECK_ARG(start_nodes >= 1, "start_nodes must be >= 1");
  tp->L = L;
  tp->size[0] = P;
  for (int l = 1; l <= L; ++l) {
    tp->size[l] = level_sizes[l - 1];
    LS_CHECK_ARG(tp->size[l] >= 0 && static_cast<int64_t>(tp->size[l]) * fanout <= tp->size[l - 1],
                 "level %d: %d nodes of %d children each exceed the %d entries below", l, tp->size[l], fanout,
                 tp->size[l - 1]);
  }
  tp->start = L;
  for (int l = 1; l <= L; ++l)
    if (tp->size[l] <= start_nodes) {
      tp->start = l;
      break;
    }
  long long ucap = 0;
  for (int l = 0; l < tp->start; ++l)
    ucap = std::max(ucap, std::max<long long>(node_block - 1,
                                              tp->size[l] - static_cast<long long>(fanout) * tp->size[l + 1]));
  tp->cap = static_cast<long long>(beam) * fanout + ucap;
  LS_CHECK_ARG(tp->cap <= (1LL << 30), "candidate lists of %lld entries are too wide", tp->cap);
  return LS_OK;
}

struct TreeWorkspace {
  int32_t* vis;     // [L + 1][T] visible entries per level
  float* sc;        // [T][size[start]] start-level scores
  int32_t* beams;   // [2][T][beam] the beams of alternate levels
  float* cval;      // [T][cap] candidates of one level
  int32_t* clab;
  int32_t* nv;      // [T]
  int32_t* picked;  // [T][top_p]
  size_t used;
};

TreeWorkspace carve_tree(void* ws, int T, const TreePlan& tp, int beam, int top_p) {
  Carver cv(ws);
  TreeWorkspace w{};
  w.vis = cv.take<int32_t>(static_cast<size_t>(tp.L + 1) * T);
  w.sc = cv.take<float>(static_cast<size_t>(T) * tp.size[tp.start]);
  w.beams = cv.take<int32_t>(2 * static_cast<size_t>(T) * beam);
  w.cval = cv.take<float>(static_cast<size_t>(T) * tp.cap);
  w.clab = cv.take<int32_t>(static_cast<size_t>(T) * tp.cap);
  w.nv = cv.take<int32_t>(T);
  w.picked = cv.take<int32_t>(static_cast<size_t>(T) * top_p);
  w.used = cv.used;
  return w;
}

}  // namespace

extern "C" {

size_t ls_lsa_tree_levels_workspace_size(int T, int P, const int* level_sizes, int L, int node_block, int fanout,
                                         int beam, int start_nodes, int top_p) {
  if (T <= 0 || top_p <= 0) return 0;
  TreePlan tp;
  if (tree_plan(P, level_sizes, L, node_block, fanout, beam, start_nodes, &tp) != LS_OK) return 0;
  return carve_tree(nullptr, T, tp, beam, top_p).used;
}

ls_status ls_lsa_tree_levels_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                                    const uint16_t* const* node_centroids, const int* level_sizes, int L,
                                    const int32_t* bucket_off, const int32_t* bucket_mem, int T, int d, int P,
                                    int block_keys, int buckets_per_block, int node_block, int fanout, int beam,
                                    int start_nodes, int n_sink, int top_p, int budget, int32_t* keys_out,
                                    int32_t* n_out, int32_t* picked_out, int32_t* beams_out, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (d != kLsaDim) return fail(LS_ERR_UNSUPPORTED, "only d=%d is built for the LSA index space (got %d)", kLsaDim, d);
  LS_CHECK_ARG(T >= 0, "negative size");
  TreePlan tp;
  ls_status s = tree_plan(P, level_sizes, L, node_block, fanout, beam, start_nodes, &tp);
  if (s != LS_OK) return s;
  LS_CHECK_ARG(block_keys >= 1 && buckets_per_block >= 1, "block_keys and buckets_per_block must be >= 1");
  LS_CHECK_ARG(n_sink >= 0 && budget >= 1, "n_sink must be >= 0 and budget >= 1");
  LS_CHECK_ARG(top_p >= 1 && top_p <= kMaxTopK, "top_p must be in [1, %d] (got %d)", kMaxTopK, top_p);
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q_idx && q_pos && centroids && bucket_off && bucket_mem && keys_out && n_out && node_centroids,
               "null tensor pointer");
  LS_CHECK_ARG(aligned16(q_idx) && aligned16(centroids), "q_idx and the centroids must be 16-byte aligned");
  for (int l = 1; l <= L; ++l)
    LS_CHECK_ARG(tp.size[l] == 0 || (node_centroids[l - 1] != nullptr && aligned16(node_centroids[l - 1])),
                 "level %d node centroids must be non-null and 16-byte aligned", l);
  const size_t need = ls_lsa_tree_levels_workspace_size(T, P, level_sizes, L, node_block, fanout, beam, start_nodes,
                                                        top_p);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  const TreeWorkspace w = carve_tree(ws, T, tp, beam, top_p);
  const int cap = static_cast<int>(tp.cap);
  int32_t* picked = picked_out ? picked_out : w.picked;
  auto beam_of = [&](int l) {   // level l's beam (1 <= l <= start)
    return beams_out ? beams_out + static_cast<size_t>(l - 1) * T * beam
                     : w.beams + ((l & 1) ? static_cast<size_t>(T) * beam : 0);
  };
  auto vis_of = [&](int l) { return w.vis + static_cast<size_t>(l) * T; };
  cudaStream_t st = S(stream);
  {
    ProfScope prof("lsa_tree_levels_visible_kernel", st);
    LS_CUDA(launch_lsa_tree_levels_visible(q_pos, T, block_keys, buckets_per_block, node_block, fanout, tp.size, L,
                                           w.vis, st));
  }
  // the start level: every visible node scored, the best `beam` kept
  const int S0 = tp.start;
  const int PS = tp.size[S0];
  if (PS > 0) {
    CUtensorMap cmap, qmap;
    s = make_vec64_map(&cmap, node_centroids[S0 - 1], static_cast<uint64_t>(PS), kTileKeys);
    if (s != LS_OK) return s;
    s = make_vec64_map(&qmap, q_idx, static_cast<uint64_t>(T), DotCfg::QB);
    if (s != LS_OK) return s;
    DotParams dp;
    dp.T = T;
    dp.P = PS;
    dp.out = w.sc;
    dp.ld_out = PS;
    ProfScope prof("dot_tc_kernel:nodes", st);
    LS_CUDA(launch_dot_tc(&cmap, &qmap, dp, num_sms_current(), st));
  }
  TopkParams bp;
  bp.scores = w.sc;
  bp.ld = PS;
  bp.n_valid = vis_of(S0);
  bp.R = T;
  bp.N = PS;
  bp.k = beam;
  bp.idx_out = beam_of(S0);
  bp.ld_out = beam;
  s = topk_launch(bp, st, "topk_kernel:beam");
  if (s != LS_OK) return s;
  // each level below: the beam's children and the uncovered entries, scored;
  // the best `beam` of them (top_p at the bucket level)
  for (int l = S0 - 1; l >= 0; --l) {
    const uint16_t* c = (l == 0) ? centroids : node_centroids[l - 1];
    {
      ProfScope prof("lsa_tree_candidates_kernel", st);
      LS_CUDA(launch_lsa_tree_candidates(q_idx, c, beam_of(l + 1), beam, vis_of(l), vis_of(l + 1), T, fanout, cap,
                                         w.cval, w.clab, w.nv, st));
    }
    TopkParams cp;
    cp.scores = w.cval;
    cp.ld = cap;
    cp.n_valid = w.nv;
    cp.labels = w.clab;
    cp.ld_labels = cap;
    cp.R = T;
    cp.N = cap;
    cp.k = (l > 0) ? beam : top_p;
    cp.idx_out = (l > 0) ? beam_of(l) : picked;
    cp.ld_out = cp.k;
    s = topk_launch(cp, st, l > 0 ? "topk_kernel:beam" : "topk_kernel");
    if (s != LS_OK) return s;
  }
  ProfScope prof("lsa_expand_kernel", st);
  LS_CUDA(launch_lsa_expand(picked, q_pos, T, top_p, bucket_off, bucket_mem, P, block_keys, n_sink, budget, keys_out,
                            n_sink + block_keys + budget, n_out, st));
  return LS_OK;
}

size_t ls_merge_select_workspace_size(int S, int T, int k_in) {
  if (S <= 0 || T <= 0 || k_in <= 0) return 0;
  const size_t n = static_cast<size_t>(T) * S * k_in;
  return align_up(n * sizeof(float)) + align_up(n * sizeof(int32_t)) + align_up(static_cast<size_t>(T) * sizeof(int32_t));
}

ls_status ls_merge_select(const float* vals, const int32_t* idx, const int32_t* offsets, int S, int T, int k_in,
                          int k, int32_t* idx_out, float* val_out, void* ws, size_t ws_bytes, void* stream) {
  LS_CHECK_ARG(S >= 1 && T >= 0 && k_in >= 1, "S and k_in must be >= 1, T >= 0");
  LS_CHECK_ARG(k >= 1 && k <= kMaxTopK, "k must be in [1, %d] (got %d)", kMaxTopK, k);
  LS_CHECK_ARG(static_cast<int64_t>(S) * k_in <= (1LL << 30), "S * k_in too large");
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(vals && idx && offsets && idx_out, "null tensor pointer");
  const size_t need = ls_merge_select_workspace_size(S, T, k_in);
  if (ws_bytes < need || !ws) return fail(LS_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  Carver cv(ws);
  const size_t n = static_cast<size_t>(T) * S * k_in;
  float* pv = cv.take<float>(n);
  int32_t* pl = cv.take<int32_t>(n);
  int32_t* nv = cv.take<int32_t>(T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    ProfScope prof("merge_pack_kernel", st);
    LS_CUDA(launch_merge_pack(vals, idx, offsets, S, T, k_in, pv, pl, nv, st));
  }
  return topk(pv, static_cast<int64_t>(S) * k_in, nv, pl, static_cast<int64_t>(S) * k_in, T, S * k_in, k, idx_out,
              val_out, k, st);
}

ls_status ls_sparse_attention(const uint16_t* q, const uint16_t* latent, const int32_t* idx, const int64_t* row_off,
                              int T, int H, int d, int d_v, int64_t n_rows, int k, float scale, int flags, float* out,
                              float* lse, void* stream) {
  LS_CHECK_ARG((flags & ~(LS_ATTN_FOREIGN_ROWS | LS_ATTN_CUDA_CORES)) == 0, "unknown flags 0x%x", flags);
  LS_CHECK_ARG(T >= 0 && H >= 0 && k >= 0 && n_rows >= 0, "negative size (T=%d H=%d k=%d)", T, H, k);
  if (d != kAttnLatent || d_v != kAttnValue)
    return fail(LS_ERR_UNSUPPORTED, "latent rows of %d elements with %d value elements are built (got d=%d d_v=%d)",
                kAttnLatent, kAttnValue, d, d_v);
  LS_CHECK_ARG(H >= kAttnHeads && H % kAttnHeads == 0 && H <= 1024, "H must be a multiple of %d in [%d, 1024] (got %d)",
               kAttnHeads, kAttnHeads, H);
  LS_CHECK_ARG(k >= 1 && k <= kAttnMaxK, "k must be in [1, %d] (got %d)", kAttnMaxK, k);
  LS_CHECK_ARG(n_rows <= 0x7fffffffLL, "at most 2^31 - 1 latent rows");
  LS_CHECK_ARG(static_cast<int64_t>(T) * (H / kAttnHeads) <= 0x7fffffffLL, "T * H / 8 too large");
  LS_CHECK_ARG(scale == scale && scale > -3.4e38f && scale < 3.4e38f, "scale must be finite");
  if (T == 0) return LS_OK;
  LS_CHECK_ARG(q && idx && out, "null tensor pointer");
  LS_CHECK_ARG(latent || n_rows == 0, "null latent with n_rows > 0");
  LS_CHECK_ARG(aligned16(q) && aligned16(out) && (!latent || aligned16(latent)),
               "q, latent and out must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int foreign_ok = (flags & LS_ATTN_FOREIGN_ROWS) ? 1 : 0;
  if (H % kTcHeads == 0 && k <= kTcMaxK && n_rows > 0 && !(flags & LS_ATTN_CUDA_CORES)) {
    // groups of 128 heads over at most 512 slots: the tensor-core kernel
    CUtensorMap qmap;
    ls_status s = make_latent_map(&qmap, q, static_cast<uint64_t>(T) * H, kTcHeads);
    if (s != LS_OK) return s;
    ProfScope prof("sparse_attn_tc_kernel", st);
    LS_CUDA(launch_sparse_attn_tc(&qmap, latent, idx, row_off, T, H, k, n_rows, scale, foreign_ok, out, lse, st));
    return LS_OK;
  }
  ProfScope prof("sparse_attn_kernel", st);
  LS_CUDA(launch_sparse_attn(q, latent, idx, row_off, T, H, k, n_rows, scale, foreign_ok, out, lse, st));
  return LS_OK;
}

ls_status ls_attention_merge(const float* o_parts, const float* lse_parts, int S, int64_t rows, int d_v, float* o,
                             float* lse, void* stream) {
  LS_CHECK_ARG(S >= 1 && rows >= 0, "S must be >= 1 and rows >= 0 (S=%d)", S);
  LS_CHECK_ARG(d_v >= 2 && d_v % 2 == 0, "d_v must be even (got %d)", d_v);
  if (rows == 0) return LS_OK;
  LS_CHECK_ARG(o_parts && lse_parts && o, "null tensor pointer");
  LS_CHECK_ARG((reinterpret_cast<uintptr_t>(o_parts) & 7u) == 0 && (reinterpret_cast<uintptr_t>(o) & 7u) == 0,
               "o_parts and o must be 8-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope prof("attn_merge_kernel", st);
  LS_CUDA(launch_attn_merge(o_parts, lse_parts, S, rows, d_v, o, lse, num_sms_current(), st));
  return LS_OK;
}

ls_status ls_profile_begin(void) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  for (auto& r : g_prof_recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof_recs.clear();
  g_prof_sums.clear();
  g_prof_on = true;
  return LS_OK;
}

ls_status ls_profile_end(int* n_kernels) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = false;
  g_prof_sums.clear();
  cudaError_t err = cudaSuccess;
  for (auto& r : g_prof_recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    ProfSum* hit = nullptr;
    for (auto& sum : g_prof_sums)
      if (sum.name == r.name) hit = &sum;
    if (!hit) {
      g_prof_sums.push_back({r.name, 0.0, 0});
      hit = &g_prof_sums.back();
    }
    hit->ms += ms;
    hit->launches += 1;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof_recs.clear();
  if (n_kernels) *n_kernels = static_cast<int>(g_prof_sums.size());
  if (err != cudaSuccess) return fail(LS_ERR_CUDA, "profiling events: %s", cudaGetErrorString(err));
  return LS_OK;
}

ls_status ls_profile_kernel(int i, const char** name, double* total_ms, long long* launches) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  LS_CHECK_ARG(i >= 0 && i < static_cast<int>(g_prof_sums.size()), "kernel index %d out of range", i);
  if (name) *name = g_prof_sums[i].name.c_str();
  if (total_ms) *total_ms = g_prof_sums[i].ms;
  if (launches) *launches = g_prof_sums[i].launches;
  return LS_OK;
}

ls_status ls_selftest_wait_probe(uint64_t limit_ns, int* gave_up_dev, void* stream) {
  LS_CHECK_ARG(gave_up_dev != nullptr, "null output");
  LS_CUDA(launch_wait_probe(limit_ns, gave_up_dev, S(stream)));
  return LS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode selection for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: an engine that
// reserves the whole device pool at start-up and gives its plugins no
// allocator, or a latency-critical loop where the implicit device-wide
// synchronisation of cudaMalloc / cudaFree is not acceptable.  For them,
// ls_decode_select_noalloc runs the same decode selection as
// ls_decode_select with its scratch (the score rows) in the fixed device
// array below, which the library holds on every device that loads it until
// the process exits.
//
// The array's host-side name is not a device address, so the first call on
// each device (with that device current) asks the runtime for the address
// with cudaGetSymbolAddress and caches it.  That first call should therefore
// be made before any stream capture is started on that device.  A
// cudaDeviceReset ends the context the cached address belongs to: a process
// that resets a device must not call this entry point on it again.  Nothing
// else is allocated: no cudaMalloc, cudaFree or allocating library call.
//
// All calls share the one array and it keeps the contents of the last call.
// Nothing in it has to start at zero: every call overwrites the score rows it
// reads (the decode selection keeps no counters there).  Calls whose work overlaps
// on the GPU (on different streams, or from different host threads) race on
// the array: order them on one stream or serialise them.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(10) << 20;  // 10 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

}  // namespace

extern "C" ls_status ls_decode_select_noalloc(const uint16_t* q, const float* w, const uint16_t* keys,
                                              const int32_t* n_valid, int B, int H, int d, int N, int k,
                                              int32_t* idx_out, float* val_out, void* stream) {
  LS_CHECK_ARG(B >= 0 && N >= 0, "negative size");
  const size_t need = ls_decode_select_workspace_size(B, N);
  if (need > kNoAllocScratchBytes)
    return fail(LS_ERR_WORKSPACE,
                "B=%d x N=%d needs %zu B of scratch; the fixed scratch of ls_decode_select_noalloc holds %zu B "
                "(2,621,440 score entries in all); use ls_decode_select with a workspace",
                B, N, need, kNoAllocScratchBytes);
  int dev = 0;
  LS_CUDA(cudaGetDevice(&dev));
  LS_CHECK_ARG(dev >= 0 && dev < 64, "device ordinal %d beyond the 64 this call tracks", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess)
        return fail(LS_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch on device %d: %s", dev,
                    cudaGetErrorString(e));
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return ls_decode_select(q, w, keys, n_valid, B, H, d, N, k, idx_out, val_out, scratch, kNoAllocScratchBytes,
                          stream);
}

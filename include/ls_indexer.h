/*
 * ls_indexer.h -- C ABI of the B200 (sm_100a) lightning-indexer selection
 * library, libls_indexer.so.
 *
 * The library computes the lightning-indexer pass of a compressed-sparse-
 * attention layer: every eligible compressed history position s of a query t
 * is scored as
 *
 *     score(t, s) = sum_h w[t, h] * max(0, q[t, h] . k[s])
 *
 * (the weighted-ReLU dot product of the DSA lightning indexer, "03 long
 * context" lecture, section "The Architectural Answer: Read Less of the Past",
 * stage 1; the 32-head x 128-d GLM-shaped form with ReLU and head weights,
 * "Latent Sparse Attention", section "Where the time goes"), and the top-k
 * positions are selected (k = 512 in DeepSeek-V4-Flash, LeanSparse podcast
 * transcript 01:33-02:06).
 *
 * Conventions for every call
 * --------------------------
 * - Tensor arguments are DEVICE pointers owned by the caller, row-major and
 *   contiguous, unless a call says otherwise.  bf16 tensors are passed as
 *   16-bit patterns (uint16_t), fp8 e4m3 as uint8_t codes.
 * - q, key and centroid tensors must be 16-byte aligned (they are read by TMA
 *   or bulk copies); w, scales and outputs must be 16-byte aligned too.
 * - Only H = 32 heads and d = 128 are built; other shapes return
 *   LS_ERR_UNSUPPORTED.  k <= 4096 (no 2048 cap).
 * - All work is enqueued asynchronously on the caller's stream(s); a stream
 *   argument is a cudaStream_t passed as void* (NULL = legacy default stream).
 * - Scratch memory comes from the caller: calls that need it take (ws,
 *   ws_bytes) and have a *_workspace_size() query.  The library allocates no
 *   device memory.  A short workspace returns LS_ERR_WORKSPACE.
 * - Ordering of selections: score descending, then position ascending; -0.0
 *   equals +0.0; NaN ranks below -inf.  Selected lists are written in that
 *   order.  Rows with fewer than k eligible positions are padded with
 *   idx = -1, val = -inf.  Values are bit copies of the scores.
 * - Masked (ineligible) positions in score outputs hold -inf.
 * - Errors: every call returns an ls_status; ls_last_error() gives a
 *   thread-local message for the last failing call of the thread.  No C++
 *   exception crosses the ABI.  Kernels never trap: a wait inside a kernel
 *   that exceeds its time limit sets a device fault word that
 *   ls_device_status() reads (LS_FAULT_* bits).
 */
#ifndef LS_INDEXER_H
#define LS_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int ls_status;
#define LS_OK 0
#define LS_ERR_INVALID_ARG 1  /* null / misaligned pointer, bad size, bad enum */
#define LS_ERR_WORKSPACE 2    /* ws_bytes smaller than the *_workspace_size() answer */
#define LS_ERR_UNSUPPORTED 3  /* shape or dtype not built (H != 32, d != 128, ...) */
#define LS_ERR_CUDA 4         /* a CUDA runtime call failed; see ls_last_error() */
#define LS_ERR_TIMEOUT 5      /* a bounded device wait ran out (ls_device_status) */

/* device fault bits reported by ls_device_status() */
#define LS_FAULT_WAIT_TIMEOUT 1 /* an in-kernel wait exceeded its limit */
#define LS_FAULT_BAD_INDEX 2    /* a gathered row id was outside the key array */

/*
 * Selection histogram: LS_HIST_BINS counts per row of the top 11 bits of each
 * score's order code, where the order code of an fp32 score with bit pattern
 * b is: 0 for NaN; else with b = 0 for -0.0, (b & 0x80000000 ? ~b : b | 0x80000000).
 * The scan produces it for free; the top-k uses it to skip its own counting
 * pass.  A histogram that does not match the scores gives wrong selections.
 */
#define LS_HIST_BINS 2048

/* key storage formats */
#define LS_KEY_BF16 0     /* [.][d] bf16 */
#define LS_KEY_FP8_E4M3 1 /* [.][d] e4m3 codes + per-key fp32 scale (128 B + 4 B) */
#define LS_KEY_INT8 2     /* [.][d] int8 codes + per-key fp32 scale */

/* Message describing the last failing call on this thread ("" if none). */
const char* ls_last_error(void);

/* ABI version of this header (major*100 + minor). */
int ls_version(void);

/*
 * Read and clear the device fault word (LS_FAULT_* bits) after synchronising
 * `stream`.  Returns LS_ERR_TIMEOUT if LS_FAULT_WAIT_TIMEOUT was set,
 * LS_ERR_INVALID_ARG if only LS_FAULT_BAD_INDEX was set, LS_OK otherwise;
 * *flags (may be NULL) receives the bits.  Blocks the host.
 */
ls_status ls_device_status(int* flags, void* stream);

/*
 * ls_indexer_score -- indexer scores of every key for every query.
 * ("03 long context", "The Architectural Answer: Read Less of the Past".)
 *
 *   q        [B][T][H][d] bf16        queries (T per sequence)
 *   w        [B][T][H]    fp32        head weights
 *   keys     [B][N][d]    key_dtype   keys of each sequence
 *   key_scale[B][N]       fp32        per-key scale (FP8/INT8 keys; NULL for BF16);
 *                                     FP8/INT8 scores use max(0, scale*(q.code))
 *   n_valid  [B] int32 or NULL        keys n >= n_valid[b] are masked
 *   q_pos    [B][T] int64 or NULL     token position of each query; when given,
 *                                     key n is masked unless stride*n+stride-1 <= q_pos
 *                                     (a compressed entry is visible once its whole
 *                                     block of `stride` tokens precedes the query;
 *                                     LeanSparse transcript 02:36-02:56)
 *   scores   [B][T][N]    fp32        output; masked entries are -inf
 *   hist_out [B*T][2048] uint32 or NULL selection histogram of the unmasked scores
 *                                     (see LS_HIST_BINS); counts are ADDED, so the
 *                                     caller zeroes it first.  T == 1 only.
 * BF16 keys take any T >= 1 (tensor-core tiles of 8 queries x 32 heads when
 * T > 1, one query per tile when T == 1).  FP8/INT8 keys take T == 1 and no
 * q_pos.  No workspace.
 */
ls_status ls_indexer_score(const uint16_t* q, const float* w, const void* keys, int key_dtype,
                           const float* key_scale, const int32_t* n_valid, const int64_t* q_pos, int stride,
                           int B, int T, int H, int d, int N, float* scores, uint32_t* hist_out, void* stream);

/*
 * ls_topk_select -- exact row-wise top-k of given fp32 scores, bit-exact.
 * (Packed score-above-inverted-id radix select, "Latent Sparse Attention",
 * "What the kernels do about the top-p".)
 *
 *   scores  row r starts at scores + r*ld (ld >= N)
 *   n_valid [R] int32 or NULL: columns >= n_valid[r] are not candidates
 *   hist    [R][LS_HIST_BINS] uint32 or NULL: the rows' selection histograms
 *           (e.g. from ls_indexer_score); NULL = counted here in one extra pass
 *   idx_out [R][k] int32 column ids (-1 padding);  val_out [R][k] fp32 or NULL
 * 1 <= k <= 4096.  No workspace.
 */
ls_status ls_topk_select(const float* scores, int64_t ld, const int32_t* n_valid, const uint32_t* hist, int R,
                         int N, int k, int32_t* idx_out, float* val_out, void* stream);

/*
 * ls_decode_select -- decode selection: one query per sequence over bf16 keys,
 * full scan then exact top-k (ls_indexer_score + ls_topk_select fused in one
 * call).  Shapes as ls_indexer_score with T = 1; outputs [B][k].  ("03 long
 * context", "The Architectural Answer: Read Less of the Past": the new token's
 * query scores every cached position with the weighted-ReLU indexer, and the k
 * best positions go on to the sparse attention.)
 * Workspace: ls_decode_select_workspace_size(B, N) bytes.
 */
size_t ls_decode_select_workspace_size(int B, int N);
ls_status ls_decode_select(const uint16_t* q, const float* w, const uint16_t* keys, const int32_t* n_valid, int B,
                           int H, int d, int N, int k, int32_t* idx_out, float* val_out, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * ls_decode_select_noalloc -- ls_decode_select for callers that cannot
 * allocate device memory (an engine that owns the whole device pool and gives
 * its plugins no allocator; a latency-critical loop that cannot take the
 * device-wide synchronisation of cudaMalloc).  The pages describe no such
 * call; it is a deployment convenience of this library.
 *
 * Same arguments and results as ls_decode_select, without (ws, ws_bytes):
 * the scratch is a fixed 10 MiB device array inside the library, held on
 * every device that loads it until the process exits.  Sizes whose
 * ls_decode_select_workspace_size(B, N) exceeds 10 MiB (B*N above 2,621,440
 * scores) return LS_ERR_WORKSPACE.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current and
 * keeps it; make that call before any stream capture, and do not call again
 * on a device after cudaDeviceReset (the kept address belonged to the ended
 * context).  The call allocates nothing.  All calls share the array: calls
 * that overlap on the GPU race and must be serialised by the caller; nothing
 * in it needs clearing (each call overwrites the score rows it reads).
 */
ls_status ls_decode_select_noalloc(const uint16_t* q, const float* w, const uint16_t* keys, const int32_t* n_valid,
                                   int B, int H, int d, int N, int k, int32_t* idx_out, float* val_out,
                                   void* stream);

/*
 * ls_prefill_select_stream -- causal top-k for a chunk of prefill queries
 * against a history that lives in host memory and is streamed through two
 * alternating device buffers (LeanSparse podcast transcript, 05:36-06:44:
 * one buffer is scored while the other receives the next part of history).
 *
 *   q       [T][H][d] bf16, w [T][H] fp32, q_pos [T] int64 (device)
 *   hist_k  [N][d] bf16 history keys in PINNED host memory (device memory is
 *           accepted too); tile j holds keys [j*tile_keys, min(N, (j+1)*tile_keys))
 *   buf0, buf1 [tile_keys][d] bf16 device buffers, caller-owned, 16-B aligned
 *   stride  compression stride (4 for CSA); query t sees keys n < (q_pos[t]+1)/stride
 *   idx_out [T][k] int32, val_out [T][k] fp32 (or NULL)
 * Copies run on copy_stream and are ordered against the scoring kernels on
 * compute_stream with events; the outputs are complete when compute_stream
 * reaches the end of the call.  The call never blocks the host.  The first
 * copy waits for work already queued on compute_stream (buffers may be in use).
 *
 * full_scores = 0: selection runs across the tiles (running top-k).  The
 * first tile is scored in full; its exact top-k starts each query's list and
 * the list's k-th entry is the query's threshold for the rest of the call.
 * Every later tile emits only the keys whose score beats that threshold
 * (strictly: a later key that ties it ranks lower) into the query's 2k
 * candidate slots for that tile; a query that fills them gets that tile's
 * exact top-k instead, from the tile scored again in full (a launch that does
 * nothing when no query overflowed).  After the last tile each query's lists
 * are packed and one exact top-k selects from them: every key of the true
 * top k scores at least the threshold, so it is in a list.  No T x N score
 * matrix is held: the workspace is one T x tile_keys tile plus
 * T x (k + 2k * (tiles - 1)) list entries, so N is bounded by the history's
 * host memory, not by the device.
 * full_scores = 1: every tile's scores go into a T x N matrix in the
 * workspace and one top-k runs at the end (fewer launches; needs T*N*4 B).
 * Both forms return the same selection.
 * Workspace: ls_prefill_select_workspace_size(T, N, tile_keys, k, full_scores) bytes.
 */
size_t ls_prefill_select_workspace_size(int T, int N, int tile_keys, int k, int full_scores);
ls_status ls_prefill_select_stream(const uint16_t* q, const float* w, const int64_t* q_pos, int T, int H, int d,
                                   const uint16_t* hist_k, int N, int stride, int tile_keys, uint16_t* buf0,
                                   uint16_t* buf1, int k, int full_scores, int32_t* idx_out, float* val_out,
                                   void* ws, size_t ws_bytes, void* compute_stream, void* copy_stream);

/*
 * ls_indexer_score_fp8 -- the indexer's scores with fp8 e4m3 queries and keys
 * (the FP8 GEMM of the indexer, "03 long context" lecture, section "Sparsity
 * Is a Systems Feature: The Blast Radius", kernel layer; 128-dim FP8 keys
 * with a 4 B scale, section "The Architectural Answer: Read Less of the
 * Past", stage 1):
 *
 *   scores[b][t][n] = sum_h w[b,t,h] * max(0, (qs[b,t,h] * q8[b,t,h]) . (ks[b,n] * k8[b,n]))
 *                   (or -inf where n is not eligible)
 *
 *   q8 [B][T][H][d] e4m3 codes, q_scale [B][T][H] fp32 (one scale per query head)
 *   w  [B][T][H] fp32
 *   k8 [B][N][d] e4m3 codes, k_scale [B][N] fp32 (one scale per key)
 *   n_valid [B] or NULL, q_pos [B][T] int64 or NULL (causal eligibility
 *   floor((q_pos + 1) / stride), as in ls_indexer_score)
 *   scores [B][T][N] fp32
 * Scales must be non-negative and finite (magnitudes, amax / 448): the
 * kernel takes them out of the ReLU, scaling the head weights by q_scale and
 * the head sum by k_scale.  The q8 . k8 products of e4m3 codes are exact and
 * summed in fp32 on the tensor cores (kind::f8f6f4); the head-weighted ReLU
 * sum runs in fp32, so the scores match the exact value of the formula to
 * fp32 rounding.
 * q8 and k8 must be 16-byte aligned; w, q_scale and k_scale 4-byte aligned.
 * Workspace: ls_indexer_score_fp8_workspace_size(B, T) bytes, 16-byte aligned
 * (w * q_scale, B*T*H floats).
 */
size_t ls_indexer_score_fp8_workspace_size(int B, int T);
ls_status ls_indexer_score_fp8(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                               const float* k_scale, const int32_t* n_valid, const int64_t* q_pos, int stride, int B,
                               int T, int H, int d, int N, float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * ls_prefill_select_stream_fp8 -- ls_prefill_select_stream with fp8 queries
 * and an fp8 history (the scores of ls_indexer_score_fp8; "03 long context",
 * "Sparsity Is a Systems Feature: The Blast Radius": the indexer key stored
 * as 128 fp8 bytes plus a 4-byte scale):
 *
 *   q8 [T][H][d] e4m3, q_scale [T][H] fp32, w [T][H] fp32, q_pos [T] int64
 *   hist_k8 [N][d] e4m3 codes and hist_kscale [N] fp32, both in PINNED host
 *           memory (device memory is accepted too)
 *   buf0, buf1  device buffers of tile_keys * (d + 4) bytes each, 16-B
 *           aligned: a tile's codes, then its scales at byte tile_keys * d
 * Streaming, the two forms (full_scores 0 / 1), outputs and ordering are as
 * in ls_prefill_select_stream; both forms return the same selection.
 * Workspace: ls_prefill_select_fp8_workspace_size(T, N, tile_keys, k,
 * full_scores) bytes, 16-byte aligned.
 */
size_t ls_prefill_select_fp8_workspace_size(int T, int N, int tile_keys, int k, int full_scores);
ls_status ls_prefill_select_stream_fp8(const uint8_t* q8, const float* q_scale, const float* w, const int64_t* q_pos,
                                       int T, int H, int d, const uint8_t* hist_k8, const float* hist_kscale, int N,
                                       int stride, int tile_keys, void* buf0, void* buf1, int k, int full_scores,
                                       int32_t* idx_out, float* val_out, void* ws, size_t ws_bytes,
                                       void* compute_stream, void* copy_stream);

/*
 * ls_lsa_flat_select -- the native LSA flat search ("Latent Sparse
 * Attention", sections "How LSA finds the keys" and "The method, term by
 * term", steps 5-6): a query scores the unit centroid of every bucket of
 * the blocks before its own with one 64-d dot product, keeps the best top_p
 * buckets and reads them best first until it holds `budget` long-range keys,
 * plus the sink keys and the window (its own, not yet clustered block).
 *
 *   q_idx      [T][64] bf16 index queries (unit vectors; the projection that
 *              makes them is the caller's)
 *   q_pos      [T] int64 token positions
 *   centroids  [P][64] bf16 unit centroids, block-major: the buckets of key
 *              block j (positions [j*block_keys, (j+1)*block_keys)) are
 *              [j*buckets_per_block, (j+1)*buckets_per_block)
 *   bucket_off [P+1] int32, bucket_mem [bucket_off[P]] int32: bucket p's
 *              member positions, ascending, in bucket_mem[off[p] .. off[p+1])
 *   n_sink     sink keys (positions 0 .. n_sink-1), block_keys the window
 *   keys_out   [T][n_sink + block_keys + budget] int32: per query, the sinks
 *              below its window, the window [block_start, t], then the
 *              long-range keys in read order (members that fall in the sinks
 *              or the window skipped, the last bucket cut short); -1 after
 *              n_out[t] entries
 *   n_out      [T] int32 entries per row
 *   picked_out [T][top_p] int32 picked buckets, best first (or NULL); -1
 *              where fewer than top_p buckets are visible
 * Visible buckets of a query at position t: the first
 * min(P, buckets_per_block * floor(t / block_keys)).  Bucket order: score
 * descending, then bucket id ascending.  Only d = 64 is built.
 * threshold = 0: every (query, bucket) score is written to a T x P matrix in
 * the workspace and the top_p of each row's visible prefix selected.
 * threshold = 1: the LSA article's sampled threshold (section "What the
 * kernels do about the top-p"): each query scores every (top_p / 16)-th
 * bucket, its 32nd best sample becomes its threshold (about 2 * top_p
 * buckets clear it; the article measures lists of about 1.7 * top_p), the
 * scan appends only the visible buckets that reach the threshold to a list
 * of up to 4 * top_p, and the top_p of the list is
 * kept; a query whose list overflows or holds fewer than min(top_p, visible)
 * buckets is scored in full instead.  Both forms pick the same buckets.
 * The threshold form never holds the T x P matrix: the missed queries are
 * listed on the device and scored in full fallback_rows at a time (a few
 * launches per chunk of rows, which return at once when the chunk holds
 * none); fallback_rows <= 0 takes the default, the most rows whose scores
 * fit 4 GiB (a multiple of 256 when that many fit), at most T.  The launches
 * for every chunk are queued whether or not a row misses: ceil(T /
 * fallback_rows) chunks.
 * Workspace: ls_lsa_flat_workspace_size(T, P, top_p, threshold,
 * fallback_rows) bytes: threshold = 0 holds the T x P matrix; threshold = 1
 * holds the samples (T x P / (top_p / 16)), the lists (about T x 8 top_p
 * entries of 8 bytes) and fallback_rows x P scores.
 */
size_t ls_lsa_flat_workspace_size(int T, int P, int top_p, int threshold, int fallback_rows);
ls_status ls_lsa_flat_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                             const int32_t* bucket_off, const int32_t* bucket_mem, int T, int d, int P,
                             int block_keys, int buckets_per_block, int n_sink, int top_p, int budget, int threshold,
                             int fallback_rows, int32_t* keys_out, int32_t* n_out, int32_t* picked_out, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * ls_lsa_tree_select -- the LSA tree search's beam over one level of node
 * buckets ("Latent Sparse Attention", section "The tree, step by step"):
 * every node_block buckets form a node cluster block, grouped fanout to a
 * node bucket (node n covers buckets fanout*n .. fanout*n + fanout - 1; nodes
 * exist for complete node blocks only).  A query scores the node buckets of
 * the complete node blocks among its visible buckets, keeps the best `beam`,
 * steps down to their children plus the visible buckets no node covers yet,
 * picks the best top_p of those and reads them as ls_lsa_flat_select does.
 *
 *   node_centroids [P1][64] bf16 unit centroids of the node buckets
 *   beam_out [T][beam] int32 picked node buckets, best first (or NULL)
 *   other arguments and outputs as in ls_lsa_flat_select
 * With beam >= every visible node bucket the picks are those of the flat
 * search.  Only d = 64 is built; ls_lsa_tree_levels_select is the search
 * over several node levels.
 * Workspace: ls_lsa_tree_workspace_size(T, P1, beam, fanout, node_block, top_p) bytes.
 */
size_t ls_lsa_tree_workspace_size(int T, int P1, int beam, int fanout, int node_block, int top_p);
ls_status ls_lsa_tree_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                             const uint16_t* node_centroids, const int32_t* bucket_off, const int32_t* bucket_mem,
                             int T, int d, int P, int P1, int block_keys, int buckets_per_block, int node_block,
                             int fanout, int beam, int n_sink, int top_p, int budget, int32_t* keys_out,
                             int32_t* n_out, int32_t* picked_out, int32_t* beam_out, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * ls_lsa_tree_levels_select -- the LSA tree search over L >= 1 levels of node
 * buckets ("Latent Sparse Attention", section "The tree, step by step").
 * Level 0 is the buckets; every node_block entries of level l - 1 (complete
 * blocks only) are grouped fanout to a node of level l, node n covering
 * entries fanout*n .. fanout*n + fanout - 1.  A query sees, at each level,
 * the nodes of the complete node blocks among its visible entries below.  The
 * beam starts at the lowest level with at most start_nodes node buckets (the
 * top level if none has so few), scores every visible node there and keeps
 * the best `beam`; at each level below it scores the kept nodes' children
 * plus the visible entries no node of the level above covers and keeps the
 * best `beam` again; at the bucket level it keeps the best top_p and reads
 * them as ls_lsa_flat_select does.
 *
 *   node_centroids  HOST array of L device pointers: level l's node
 *                   centroids [level_sizes[l-1]][64] bf16 at node_centroids[l-1]
 *   level_sizes     HOST array of L ints, P1 .. PL; fanout * P_l <= P_{l-1}
 *   L               1 .. 16
 *   beam            1 .. 4096; start_nodes >= 1 (the pages: 32768)
 *   picked_out      [T][top_p] int32 picked buckets, best first (or NULL)
 *   beams_out       [L][T][beam] int32: level l's beam at [l-1], best first,
 *                   -1 past its end (or NULL); levels above the start level
 *                   are not written
 *   other arguments and outputs as in ls_lsa_flat_select
 * Ties go to the lower entry at every level.  With beam >= every level's
 * visible entries the picks are those of the flat search.  The host arrays
 * are read before the call returns; the device buffers must stay valid until
 * the stream's work ends.
 * Errors: LS_ERR_INVALID_ARG for sizes out of range, a level larger than its
 * children allow, null or misaligned pointers; LS_ERR_UNSUPPORTED for d != 64;
 * LS_ERR_WORKSPACE below the size returned by
 * ls_lsa_tree_levels_workspace_size(T, P, level_sizes, L, node_block, fanout,
 * beam, start_nodes, top_p) (0 for invalid arguments).
 */
size_t ls_lsa_tree_levels_workspace_size(int T, int P, const int* level_sizes, int L, int node_block, int fanout,
                                         int beam, int start_nodes, int top_p);
ls_status ls_lsa_tree_levels_select(const uint16_t* q_idx, const int64_t* q_pos, const uint16_t* centroids,
                                    const uint16_t* const* node_centroids, const int* level_sizes, int L,
                                    const int32_t* bucket_off, const int32_t* bucket_mem, int T, int d, int P,
                                    int block_keys, int buckets_per_block, int node_block, int fanout, int beam,
                                    int start_nodes, int n_sink, int top_p, int budget, int32_t* keys_out,
                                    int32_t* n_out, int32_t* picked_out, int32_t* beams_out, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * ls_merge_select -- the combine step of a prefill whose history is split into
 * S contiguous shards (one per GPU, say): each shard's exact top-k lists of
 * the same T queries are merged into the top-k of the whole history (the
 * top-k of the union of the shards' top-k lists is the global top-k, since
 * every shard contributes its own best).  ("03 long context", "Teamwork
 * First: Ring Attention for the Giant Prefill": the sequence is sharded over
 * GPUs and partial results are combined; this is that combine for the
 * selection.)
 *
 *   vals [S][T][k_in] fp32, idx [S][T][k_in] int32: list s of query t, in
 *        canonical order, positions local to shard s, padded with -1 / -inf
 *        at the end (the output form of ls_prefill_select_stream)
 *   offsets [S] int32 (device): shard s's first position in the history
 *   idx_out [T][k] int32 global positions, val_out [T][k] fp32 (or NULL)
 * Ordering and padding as everywhere (score descending, position ascending;
 * -1 / -inf past the end); values are bit copies of the inputs.
 * Workspace: ls_merge_select_workspace_size(S, T, k_in) bytes.
 */
size_t ls_merge_select_workspace_size(int S, int T, int k_in);
ls_status ls_merge_select(const float* vals, const int32_t* idx, const int32_t* offsets, int S, int T, int k_in,
                          int k, int32_t* idx_out, float* val_out, void* ws, size_t ws_bytes, void* stream);

#define LS_ATTN_FOREIGN_ROWS 1   /* ls_sparse_attention: rows outside [0, n_rows) are another shard's */
#define LS_ATTN_CUDA_CORES 2     /* ls_sparse_attention: take the CUDA-core kernel even where the tensor-core one applies */

/*
 * ls_sparse_attention -- sparse main attention over the selected rows, stage
 * 2 of DSA ("03 long context", section "The Architectural Answer: Read Less
 * of the Past"): exact attention of every query head over only the k rows the
 * indexer selected, in the absorbed MLA form where one cached latent row of
 * d = 576 bf16 elements (512 latent + 64 rotary; "Derivation 6" of the same
 * lecture) is the key of every head and its first d_v = 512 elements the
 * value.  For query t, head h and the selected rows S_t:
 *   logit(s) = scale * q[t,h,:] . latent[s,:]
 *   lse[t,h] = log sum_{s in S_t} exp(logit(s))
 *   out[t,h,:] = sum_{s in S_t} exp(logit(s) - lse[t,h]) * latent[s,:512]
 *
 *   q [T][H][576] bf16, latent [n_rows][576] bf16 (16-byte aligned)
 *   idx [T][k] int32: selected positions, -1 = unused slot (anywhere in the row)
 *   row_off [T] int64 or NULL: row of latent = idx + row_off[t] (one buffer
 *        holding several sequences' caches); a row outside [0, n_rows) is
 *        skipped and sets LS_FAULT_BAD_INDEX (see ls_device_status)
 *   H a multiple of 8; k <= 65536 (the selection streams through in chunks
 *        of 64 slots: an LSA read list of 4612 slots fits)
 *   scale: the softmax scale (1/sqrt(576) is the plain choice; the pages do
 *        not fix it)
 *   flags: 0, or LS_ATTN_FOREIGN_ROWS when latent holds one shard of the
 *        rows (row_off = -first row of the shard, n_rows = its length): rows
 *        outside it belong to other shards and are skipped without the fault;
 *        LS_ATTN_CUDA_CORES forces the CUDA-core kernel (below)
 * Kernels: H a multiple of 128 and k <= 512 run on the tensor cores (tcgen05:
 *        logits and the value contraction as MMAs, the weights rounded to
 *        bf16 for the value contraction, so an output is within 2^-8 of the
 *        largest selected value magnitude; lse in fp32); other shapes, or
 *        LS_ATTN_CUDA_CORES, take the fp32 CUDA-core kernel (within 1e-4).
 *   out [T][H][512] fp32; lse [T][H] fp32 natural-log sum or NULL.  An empty
 *        selection gives out = 0 and lse = -inf; partial results over
 *        disjoint selections combine exactly by their lse (online softmax).
 * Errors: LS_ERR_UNSUPPORTED for d != 576 or d_v != 512, LS_ERR_INVALID_ARG
 * for the other limits.  No workspace; asynchronous on `stream`.
 */
ls_status ls_sparse_attention(const uint16_t* q, const uint16_t* latent, const int32_t* idx, const int64_t* row_off,
                              int T, int H, int d, int d_v, int64_t n_rows, int k, float scale, int flags, float* out,
                              float* lse, void* stream);

/*
 * ls_attention_merge -- combine S partial attentions of the same T x H
 * (query, head) rows over disjoint selected-row sets into the attention over
 * their union, by the online-softmax rule (the merge of the ring-attention
 * section of "03 long context", "Teamwork First: Ring Attention for the Giant
 * Prefill"): with m = max_s lse_s and w_s = exp(lse_s - m),
 *   o = sum_s w_s o_s / sum_s w_s,   lse = m + log sum_s w_s.
 * The combine step of a history-sharded attention: each rank attends over the
 * selected rows it holds (LS_ATTN_FOREIGN_ROWS), the (o, lse) parts are
 * gathered, and this call merges them.
 *
 *   o_parts [S][rows][d_v] fp32 (8-byte aligned), lse_parts [S][rows] fp32
 *   o [rows][d_v] fp32, lse [rows] fp32 or NULL; rows = T * H, d_v even
 * A part with lse = -inf (an empty selection) weighs 0; when every part is
 * empty, o = 0 and lse = -inf.  No workspace; asynchronous on `stream`.
 */
ls_status ls_attention_merge(const float* o_parts, const float* lse_parts, int S, int64_t rows, int d_v, float* o,
                             float* lse, void* stream);

/*
 * ls_decode_two_stage_select -- LeanSparse two-stage decode search
 * (podcast transcript, 07:12-08:00): scan compact keys, keep a shortlist,
 * fetch the shortlist's original keys and re-rank exactly, keep the top k.
 *
 *   q [B][H][d] bf16, w [B][H] fp32
 *   ck [B][N][d] int8, ck_scale [B][N] fp32      compact keys (coarse pass)
 *   fk [B][N][d] fp8 e4m3, fk_scale [B][N] fp32  original keys (132 B per key)
 *   n_valid [B] int32 or NULL
 *   shortlist  shortlist length S (k <= S <= 4096)
 *   idx_out [B][k] positions, val_out [B][k] exact scores (or NULL)
 *   shortlist_out [B][S] int32 or NULL: the shortlist (positions in coarse-score
 *   order, -1 padding)
 * Workspace: ls_two_stage_workspace_size(B, N, S) bytes.
 */
size_t ls_two_stage_workspace_size(int B, int N, int shortlist);
ls_status ls_decode_two_stage_select(const uint16_t* q, const float* w, const int8_t* ck, const float* ck_scale,
                                     const uint8_t* fk, const float* fk_scale, const int32_t* n_valid, int B,
                                     int H, int d, int N, int shortlist, int k, int32_t* idx_out, float* val_out,
                                     int32_t* shortlist_out, void* ws, size_t ws_bytes, void* stream);

/*
 * ls_decode_two_stage_pq_select -- the same search with 32-byte product-
 * quantised compact keys, the LeanSparse compact-key form (podcast
 * transcript, 07:12-07:34): a key is 32 one-byte codes, code m choosing row
 * code[m] of codebook m, whose 4 values are dimensions 4m..4m+3 of the
 * decoded key.  The coarse score is the indexer score of the decoded key;
 * the shortlist is re-ranked exactly with the fp8 originals as above.
 *
 *   pq_codes [B][N][32] uint8
 *   pq_books [32][256][4] fp16 (IEEE binary16 bit patterns), 16-byte aligned
 * Other arguments, outputs, errors and workspace as ls_decode_two_stage_select.
 */
ls_status ls_decode_two_stage_pq_select(const uint16_t* q, const float* w, const uint8_t* pq_codes,
                                        const uint16_t* pq_books, const uint8_t* fk, const float* fk_scale,
                                        const int32_t* n_valid, int B, int H, int d, int N, int shortlist, int k,
                                        int32_t* idx_out, float* val_out, int32_t* shortlist_out, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * ls_indexer_score_pq -- coarse scores of PQ compact keys (one query per
 * sequence): scores[b][n] = sum_h w[b,h] * max(0, q[b,h] . key(b,n)), key
 * decoded from pq_codes[b][n] with pq_books as in
 * ls_decode_two_stage_pq_select; -inf for n >= n_valid[b].  (LeanSparse
 * podcast transcript, 07:12-07:34: the coarse pass over 32-byte compact keys.)
 *   q [B][H][d] bf16, w [B][H] fp32, pq_codes [B][N][32], pq_books [32][256][4]
 *   fp16, scores [B][N] fp32; all device pointers, 16-byte aligned.
 */
ls_status ls_indexer_score_pq(const uint16_t* q, const float* w, const uint8_t* pq_codes, const uint16_t* pq_books,
                              const int32_t* n_valid, int B, int H, int d, int N, float* scores, void* stream);

/*
 * ls_bucket_select -- LSA-style flat bucket search with indexer-form scoring
 * ("Latent Sparse Attention", "How LSA finds the keys" and "The method, term
 * by term", steps 5-6): score every bucket centroid, keep the top_p buckets,
 * expand them best first into `budget` key positions (members in stored
 * order, the last bucket cut short), score those keys exactly, keep the top k.
 *
 *   q [T][H][d] bf16, w [T][H] fp32
 *   centroids [P][d] bf16
 *   bucket_off [P+1] int32, bucket_mem [M] int32   CSR member lists (positions < N)
 *   keys [N][d] bf16
 *   top_p <= 4096, k <= budget, k <= 4096
 *   idx_out [T][k], val_out [T][k] (or NULL), picked_out [T][top_p] or NULL
 * Workspace: ls_bucket_workspace_size(T, P, top_p, budget) bytes.
 */
size_t ls_bucket_workspace_size(int T, int P, int top_p, int budget);
ls_status ls_bucket_select(const uint16_t* q, const float* w, const uint16_t* centroids, const int32_t* bucket_off,
                           const int32_t* bucket_mem, const uint16_t* keys, int T, int H, int d, int P, int N,
                           int top_p, int budget, int k, int32_t* idx_out, float* val_out, int32_t* picked_out,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Profiling: between ls_profile_begin() and ls_profile_end(), every kernel the
 * library launches is bracketed by two CUDA events on its launch stream.
 * ls_profile_end() waits for those events and sums the durations per kernel
 * name; ls_profile_kernel(i, ...) reads kernel i (0 <= i < *n_kernels).  The
 * name pointer stays valid until the next ls_profile_begin().  Host thread
 * safe; recording adds two event records per launch.
 */
ls_status ls_profile_begin(void);
ls_status ls_profile_end(int* n_kernels);
ls_status ls_profile_kernel(int i, const char** name, double* total_ms, long long* launches);

/*
 * ls_selftest_wait_probe -- failure-detection check: launches a kernel whose
 * mbarrier is never completed; its bounded wait gives up after limit_ns
 * nanoseconds, sets LS_FAULT_WAIT_TIMEOUT and returns.  *gave_up_dev (device
 * int) receives 1 when the wait gave up.  The context stays usable.
 */
ls_status ls_selftest_wait_probe(uint64_t limit_ns, int* gave_up_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LS_INDEXER_H */

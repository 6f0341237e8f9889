/*
 * zha.h -- C ABI of libzha: tree-indexed sparse decode attention on B200 (sm_100a).
 *
 * The method ("Subquadratic Attention with a Hierarchical Tree-Structured
 * Indexer", abstract): a tree of recursively compressed key summaries is kept
 * over the KV cache; at decode time each query walks the tree from the top
 * down and keeps a sparse subset of keys; exact attention then runs over that
 * subset.  The tree grows in depth as the cache grows.  The tree is static over
 * token order ("ALHR" news item, technical features: static trees route keys
 * hierarchically).  This library fixes the open points as follows:
 *
 *   leaf i            = mean of keys t in [i*leaf_block, min((i+1)*leaf_block, N))
 *   node i, level l   = unweighted mean of its existing children
 *                       j in [b*i, min(b*i+b, n_{l-1}))
 *   levels            L = smallest L >= 1 with b^L >= n0 = ceil(N / leaf_block);
 *                       level L holds the single root, level 0 the leaves
 *   routing           survivors = {root}; for l = L-1 .. 0: score every child c
 *                       of a survivor by q . S_l[c] (unscaled, fp32), keep the
 *                       top-min(beam, #candidates) by score, lower index first
 *                       on equal scores
 *   attention         softmax(scale * q . K[t]) weighted V over the tokens
 *                       t < N of the selected leaves (exact, split-KV online
 *                       softmax with an fp32 combine)
 *
 * Conventions for every call:
 *   - Every pointer named d_* is device memory owned by the caller.  The
 *     library never allocates device memory (no cudaMalloc anywhere).
 *   - Layouts are dense row-major:
 *       K, V  [batch, kv_heads, capacity_tokens, head_dim]  (tree's kv_dtype)
 *       Q, O  [batch, q_heads, nq, head_dim]
 *       leaf_idx / leaf_score  [batch, q_heads, nq, beam]
 *     Query head h reads KV head h / (q_heads / kv_heads).
 *   - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and return a status.  Argument errors are found on the
 *     host before any launch (ZHA_ERR_INVALID_ARG, ZHA_ERR_CAPACITY,
 *     ZHA_ERR_UNSUPPORTED) and leave the tree unchanged.  A failed launch
 *     returns ZHA_ERR_CUDA.  Problems only the device can see (a leaf index
 *     out of range, a bounded wait that ran out) are recorded in a device
 *     error word that zha_tree_check reads.
 *   - A zha_tree handle is not thread-safe; calls that share a tree must be
 *     ordered by the caller (same stream, or events).
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ZHA_OK = 0,
  ZHA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad order of calls  */
  ZHA_ERR_CAPACITY = 2,    /* seq_len beyond the tree's capacity_tokens              */
  ZHA_ERR_UNSUPPORTED = 3, /* shape outside what the kernels are built for            */
  ZHA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed             */
  ZHA_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (reported by check)       */
  ZHA_ERR_DEVICE = 6       /* a kernel met invalid data, e.g. a leaf index >= n0      */
} zha_status;

typedef enum { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;

/* Geometry of one tree set: one tree per (batch, kv head) "unit". */
typedef struct {
  int batch;                 /* >= 1                                               */
  int kv_heads;              /* >= 1; batch * kv_heads <= 65535                    */
  int head_dim;              /* 64 or 128                                          */
  int branching;             /* b >= 2                                             */
  int leaf_block;            /* tokens per leaf >= 1                               */
  long long capacity_tokens; /* rows allocated per unit in K and V, >= 1          */
  zha_dtype kv_dtype;        /* storage type of K, V                               */
  /* Storage type of the summaries.  ZHA_F32 (0, the default of a zeroed desc): each node
   * holds its fp64 mean rounded to fp32.  ZHA_BF16: each node holds that fp32 value rounded
   * to the nearest bf16 (ties to even), and a parent averages its children's stored bf16
   * values; a route then reads half the bytes.  Scores are formed in fp32 either way. */
  zha_dtype summary_dtype;
} zha_tree_desc;

typedef struct zha_tree zha_tree; /* opaque host handle */

/* Device bytes the caller must provide to zha_tree_init: a 256-byte header
 * (device error word) followed by the summaries of every unit (fp32 or bf16, the desc's
 * summary_dtype), laid out unit-major, level-contiguous with capacity-sized levels.
 * 0 on a bad desc. */
size_t zha_tree_workspace_bytes(const zha_tree_desc* desc);

/* Creates a host handle over caller-owned workspace (>= zha_tree_workspace_bytes,
 * 256-byte aligned).  The tree starts empty (seq_len 0).  Clears the device error
 * word with a synchronous cudaMemset on the current device.  *out receives the
 * handle; free it with zha_tree_destroy. */
zha_status zha_tree_init(const zha_tree_desc* desc, void* d_workspace, size_t workspace_bytes,
                         zha_tree** out);

/* Frees the host handle only; the workspace stays the caller's. */
zha_status zha_tree_destroy(zha_tree* tree);

/* Builds every summary from tokens [0, seq_len) of d_K (replacing any previous
 * state): the tree of recursively compressed key summaries kept over the KV cache
 * ("Subquadratic Attention with a Hierarchical Tree-Structured Indexer", abstract).  seq_len == 0 leaves an empty tree.  ZHA_ERR_CAPACITY if seq_len >
 * capacity_tokens. */
zha_status zha_tree_build(zha_tree* tree, const void* d_K, long long seq_len, void* stream);

/* Extends the tree to tokens [0, new_seq_len) as the cache grows, deepening it when needed
 * (same abstract: the tree's depth grows with the context): the caller has already written
 * rows [seq_len, new_seq_len) of K.  Recomputes the leaves that received tokens
 * and all of their ancestors; adds levels when the leaves outgrow b^L.
 * new_seq_len must be >= the current seq_len (equal: no-op). */
zha_status zha_tree_append(zha_tree* tree, const void* d_K, long long new_seq_len, void* stream);

/* Top-down beam routing of nq queries per query head: each query traverses the tree from
 * the top down to retrieve a sparse subset of keys (same abstract).
 *   d_Q          [batch, q_heads, nq, head_dim] in q_dtype; q_heads % kv_heads == 0
 *   beam         1 .. 1024, and beam * branching <= 4096
 *   d_leaf_idx   out [batch, q_heads, nq, beam] int32: selected leaves, ascending,
 *                -1 after the last one (only when the tree has fewer than beam leaves)
 *   d_leaf_score out, nullable: q . S_0[leaf] (fp32) beside each index, NaN on padding
 *   d_trace      out, nullable: [batch, q_heads, nq, L, beam] int32, the nodes kept at
 *                levels L-1 .. 0 in that order, ascending, -1 padded (L = zha_tree_levels)
 * The tree must be non-empty.  nq == 0 is a no-op. */
zha_status zha_route(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                     int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* stream);

/* Device scratch bytes zha_sparse_attn_decode needs for this shape (0 when the
 * call needs none).  The value depends on the tree geometry, q_heads, nq, beam
 * and the device's SM count, not on seq_len. */
size_t zha_attn_scratch_bytes(const zha_tree* tree, int q_heads, int nq, int beam);

/* Exact softmax attention of each query over the tokens t < seq_len of its leaves: the
 * final attention over the retrieved subset (same abstract).
 *   d_Q, d_leaf_idx  as produced for / by zha_route (indices < 0 are skipped)
 *   d_K, d_V         the cache the tree was built over
 *   scale            multiplies q . k before the softmax (e.g. 1/sqrt(head_dim))
 *   d_O              out [batch, q_heads, nq, head_dim] in o_dtype (bf16: RNE)
 *   d_scratch        >= zha_attn_scratch_bytes(tree, q_heads, nq, beam) bytes
 *                    (may be NULL when that is 0); contents need no initialisation
 * An index >= n0 sets ZHA_ERR_DEVICE in the error word and is skipped. */
zha_status zha_sparse_attn_decode(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype,
                                  int q_heads, int nq, const void* d_K, const void* d_V,
                                  const int* d_leaf_idx, int beam, float scale, void* d_O,
                                  zha_dtype o_dtype, void* d_scratch, size_t scratch_bytes,
                                  void* stream);

/* zha_sparse_attn_decode for callers that cannot allocate device memory -- an operator
 * hook handed only its input and output pointers, with no workspace, or a code path
 * where cudaMalloc is off limits because it synchronizes the device or because device
 * memory belongs to another allocator.  (The source pages have no counterpart: this is
 * a calling convention of this library.)  Same arguments, results and checks as
 * zha_sparse_attn_decode minus the scratch pair: the split-KV partials go to a fixed
 * device array inside this library of zha_noalloc_scratch_capacity() bytes (128 KiB),
 * which every GPU that loads the library holds until the process exits.  Shapes whose
 * partials need more return ZHA_ERR_CAPACITY (use zha_sparse_attn_decode for them).
 * The tree's device must be current (ZHA_ERR_INVALID_ARG otherwise).  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) and caches it for the
 * life of the process; make that first call before any stream capture.  A cudaDeviceReset
 * invalidates the cached address, so do not call this entry point after one.  No call allocates or frees device memory.  All calls share the one array and
 * nothing in it needs clearing between calls, so calls whose kernels overlap on the GPU
 * (other streams, other threads) race on it: order them. */
zha_status zha_sparse_attn_decode_noalloc(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype,
                                          int q_heads, int nq, const void* d_K, const void* d_V,
                                          const int* d_leaf_idx, int beam, float scale, void* d_O,
                                          zha_dtype o_dtype, void* stream);
size_t zha_noalloc_scratch_capacity(void);

/* Route + attention of a decode step in one call: the results of zha_route followed by
 * zha_sparse_attn_decode over the leaves it selected, computed by one kernel launch in
 * which each query's warps route it and then attend over its leaves' tokens (no leaf
 * list or partials pass through global memory).  Arguments as in those two calls:
 *   d_leaf_idx    out [batch, q_heads, nq, beam] int32, required: the selected leaves
 *   d_leaf_score  out, nullable: their scores
 *   d_trace       out, nullable: the nodes kept per level, as in zha_route
 *   d_O           out [batch, q_heads, nq, head_dim] in o_dtype
 * Same constraints (q_heads % kv_heads == 0, 1 <= beam <= 1024, beam * branching <= 4096,
 * non-empty tree).  Needs no scratch.  When a query's widest level is too large to
 * stage in shared memory (more than about 200 KB of summary rows), the call runs the
 * route and the attention as two launches instead, with the same results; it returns
 * ZHA_ERR_UNSUPPORTED if that attention would need scratch (use the two calls then). */
zha_status zha_decode(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                      int beam, const void* d_K, const void* d_V, float scale, int* d_leaf_idx,
                      float* d_leaf_score, int* d_trace, void* d_O, zha_dtype o_dtype,
                      void* stream);

/* One decode step: zha_tree_append(tree, d_K, new_seq_len) followed by zha_decode(...) over
 * the extended cache, with the same results.  When the appended tokens all fall into one
 * leaf (a step of one token, say) and the decode runs one query per CTA (at most two queries
 * per SM), both happen in a single kernel launch: every CTA recomputes the leaf-to-root path
 * of its unit with the append's arithmetic, one CTA per unit stores it, and the route uses
 * the recomputed rows.  Otherwise the append and the decode are launched one after the other.
 * The caller has written rows [seq_len, new_seq_len) of K and V.  Argument checks as in both
 * calls (new_seq_len >= seq_len, <= capacity_tokens, > 0); on a host-side error nothing is
 * launched and the tree is unchanged. */
zha_status zha_decode_step(zha_tree* tree, const void* d_K, const void* d_V, long long new_seq_len,
                           const void* d_Q, zha_dtype q_dtype, int q_heads, int nq, int beam,
                           float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                           zha_dtype o_dtype, void* stream);

/* Causal (per-position) routing, as a prefill visits every position: query i of every
 * (batch, query head) routes over the tree of the prefix of tokens 0 .. d_positions[i] -- the
 * tree zha_tree_build would make over those tokens alone -- with the rules of zha_route.
 * That tree shares every node with the stored tree except its right edge (the ancestors of
 * the leaf holding token d_positions[i]), which each query recomputes on chip from the
 * cache and the stored rows; the stored tree is not changed.
 *   d_K          the cache the tree was built over (the prefix's last leaf is re-read)
 *   d_positions  [nq] int64, device: 0 <= position < seq_len; a position outside the tree
 *                sets ZHA_ERR_DEVICE in the error word and that query routes nowhere
 *                (leaves all -1)
 *   d_trace      nullable: [batch, q_heads, nq, L, beam] with L = zha_tree_levels of the
 *                whole tree; rows of levels at or above the prefix tree's depth are -1
 * Other arguments, layouts and limits as in zha_route; nothing is allocated.
 * ZHA_ERR_UNSUPPORTED when a query's widest level and the path do not fit shared memory. */
zha_status zha_route_causal(const zha_tree* tree, const void* d_K, const void* d_Q, zha_dtype q_dtype,
                            int q_heads, int nq, const long long* d_positions, int beam, int* d_leaf_idx,
                            float* d_leaf_score, int* d_trace, void* stream);

/* zha_route_causal followed by exact softmax attention of each query over the tokens of its
 * leaves that lie in its prefix (t <= position), in one launch; O as in zha_decode.
 * ZHA_ERR_UNSUPPORTED when the shape does not fit the fused kernel. */
zha_status zha_decode_causal(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                             const long long* d_positions, int beam, const void* d_K, const void* d_V,
                             float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                             zha_dtype o_dtype, void* stream);

/* Decode with an append buffer ("Louver" explainer, dynamic updates: keys produced during
 * decoding wait in a small buffer that every query reads directly, and a full buffer is
 * merged into the index in the background, concurrently with the attention).  Each query
 * routes over the tree of the first n_routed tokens (the prefix of zha_route_causal at
 * position n_routed - 1) and attends, exactly, over the tokens of its leaves together with
 * every buffered token n_routed .. n_tokens - 1 of the cache; O as in zha_decode.
 *   n_routed   a multiple of the leaf block, 1 <= n_routed <= zha_tree_seq_len: the tree
 *              must summarise the first n_routed tokens, through calls ordered before this
 *              one on `stream`
 *   n_tokens   n_routed <= n_tokens <= capacity; tokens n_routed .. n_tokens - 1 of d_K and
 *              d_V written by the caller before the call
 * The call reads no summary that an append of tokens at or after n_routed writes, so the
 * caller may commit the buffer (zha_tree_append to n_tokens) on another stream while it
 * keeps decoding with the old n_routed, and switch n_routed once that append has completed.
 * d_leaf_idx / d_leaf_score / d_trace describe the routed leaves only (as in
 * zha_route_causal).  ZHA_ERR_UNSUPPORTED when the shape does not fit the fused kernel. */
zha_status zha_decode_buffered(const zha_tree* tree, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                               int beam, const void* d_K, const void* d_V, long long n_routed,
                               long long n_tokens, float scale, int* d_leaf_idx, float* d_leaf_score,
                               int* d_trace, void* d_O, zha_dtype o_dtype, void* stream);

/* Bounding spheres for threshold descent ("Louver" explainer: every cluster of keys is
 * enclosed in a sphere, a center and a radius).  The center of a node is its summary; the
 * radius covers every key of its subtree (leaf: its farthest token; node: its farthest
 * child sphere, ||c_child - c|| + r_child), stored as fp32 rounded up.  The radii live in a
 * caller-owned device buffer of zha_tree_radii_bytes(tree) bytes ([units][unit_rows] fp32,
 * rows as in zha_tree_summaries), 16-byte aligned.  zha_tree_attach_radii computes them for
 * the current tree (d_K: the cache it was built over; may be NULL while the tree is empty);
 * afterwards zha_tree_build, zha_tree_append and zha_decode_step keep them current (the
 * latter then appends and decodes in two launches).  d_radii = NULL detaches. */
size_t zha_tree_radii_bytes(const zha_tree* tree);
zha_status zha_tree_attach_radii(zha_tree* tree, float* d_radii, size_t bytes, const void* d_K, void* stream);

/* Threshold (halfspace) descent: for every query, all tokens t < seq_len with
 * q . K[t] >= tau (unscaled dot product), found by descending the tree and pruning a node
 * whose sphere cannot reach the threshold (q . c + ||q|| r < tau), then checking the tokens
 * of the surviving leaves exactly (fp64).  No key with q . k >= tau is missed.
 *   d_tau      [batch, q_heads, nq] fp32 thresholds, device
 *   d_tokens   out [batch, q_heads, nq, max_tokens] int32: the tokens found, ascending, -1 after
 *   d_count    out [batch, q_heads, nq] int32: how many were found (may exceed max_tokens; the
 *              list then holds the first max_tokens); -1 when a level kept more than 8,192 nodes
 *              (the descent stops; widen the threshold or route with zha_route)
 *   d_stats    out, nullable: [batch, q_heads, nq, 2] int32: spheres tested, tokens checked
 * Requires radii attached (zha_tree_attach_radii) and a non-empty tree. */
zha_status zha_threshold_route(const zha_tree* tree, const void* d_K, const void* d_Q, zha_dtype q_dtype,
                               int q_heads, int nq, const float* d_tau, int max_tokens, int* d_tokens,
                               int* d_count, int* d_stats, void* stream);

/* Synchronizes `stream`, then reads and clears the device error word:
 * ZHA_OK, ZHA_ERR_TIMEOUT or ZHA_ERR_DEVICE (or ZHA_ERR_CUDA if the stream failed). */
zha_status zha_tree_check(zha_tree* tree, void* stream);

/* Getters.  Levels are numbered from the leaves (0) to the root (zha_tree_levels). */
long long zha_tree_seq_len(const zha_tree* tree);
int zha_tree_levels(const zha_tree* tree);                        /* L; 0 when empty   */
long long zha_tree_level_nodes(const zha_tree* tree, int level);  /* n_level now       */
long long zha_tree_level_offset(const zha_tree* tree, int level); /* row offset in unit */
long long zha_tree_unit_rows(const zha_tree* tree);               /* rows per unit      */
/* device: [units, unit_rows, head_dim] of the desc's summary_dtype (fp32, or bf16 bits) */
const void* zha_tree_summaries(const zha_tree* tree);
/* Kernel launches issued through this handle since zha_tree_init (all calls). */
long long zha_tree_launch_count(const zha_tree* tree);
/* Copies the geometry the tree was created with into *out (bindings use it to check
 * buffer shapes before a call).  ZHA_ERR_INVALID_ARG on a null argument. */
zha_status zha_tree_get_desc(const zha_tree* tree, zha_tree_desc* out);
/* The CUDA device that was current when the tree was created; -1 on a null handle. */
int zha_tree_device(const zha_tree* tree);

/* Failure-path testing (the source pages have no counterpart).  Every kernel that waits for
 * its own bulk copies bounds that wait (about a second of SM clock); a wait that runs out
 * records ZHA_ERR_TIMEOUT in the device error word, waits for the copies it issued with the
 * same default bound, marks the affected queries' outputs as lost (leaf indices -1, scores
 * and O NaN) and returns; the context stays usable.  This call lowers the first of those two
 * bounds to `cycles` SM clock cycles for every later call on this tree, so a test can make a
 * wait run out on demand; 0 restores the default.  After a call whose wait ran out, the
 * summaries that call was writing (a build or append) are unspecified until the tree is
 * rebuilt.  ZHA_ERR_INVALID_ARG on a null tree or negative cycles. */
zha_status zha_tree_set_wait_limit(zha_tree* tree, long long cycles);

const char* zha_status_string(zha_status status);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */

// Shared pieces of the routing kernels: arguments, per-query shared-memory layout, the
// packed candidate keys and the top-B selections.  Top-down beam routing follows
// "Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (abstract: queries
// traverse the tree of key summaries from the top down to retrieve a sparse subset of
// keys); every survivor's children are scored by q . S_l[c] in fp32 and the
// top-min(beam, #candidates) are kept, lower node index first on equal scores.
#pragma once

#include <algorithm>
#include <type_traits>

#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

constexpr int kRouteMaxWarps = 16;

struct RouteArgs {
  const void* Q;
  int q_bf16;
  int q_heads, nq, group, kv_heads;
  int head_dim;
  const void* pyr;            // summaries (the kernel's summary type)
  long long pyr_unit_stride;  // elements
  long long off[kMaxLevels];
  long long n[kMaxLevels];
  int L, b, beam, cmax;
  int wpq, qpc;           // warps per query, queries per CTA
  int query_smem_words;   // 8-byte words of shared memory per query
  int* leaf_idx;
  float* leaf_score;
  int* trace;
  long long total_queries;
  unsigned* err;           // device error word (bounded waits)
  int query_smem_bytes;    // shared memory per query (staged kernel)
  int rows_bytes;          // bytes of the candidate-row region per query
  // fused attention (route_tma_kernel with TKV != NoKV)
  const char* K;
  const char* V;
  long long kv_unit_stride;  // bytes
  long long lb, N;
  float qk_scale;            // scale * log2(e)
  int stage_tokens;          // tokens per stage buffer
  int attn_nbuf;             // stage buffers in the row region (2 or 3)
  void* O;
  int o_bf16;
  // fused one-leaf append (route_tma_kernel with APPEND)
  long long path_leaf;       // the leaf that received the new tokens
  int path_tokens;           // its tokens after the append
  long long path_smem_off;   // byte offset of the path region in a query's shared memory
  // causal routing (kPathPrefix): query qg routes over tokens 0 .. positions[qg % nq], or
  // over tokens 0 .. prefix_pos when positions is null
  const long long* positions;
  long long prefix_pos;
  // append buffer: the attention also covers buf_tokens tokens from leaf buf_leaf0 on (the
  // tokens after the routed prefix, which then ends on a leaf boundary)
  long long buf_leaf0;
  int buf_tokens;
  long long first_wait;      // bound of a first wait for copies (kCopyWaitCycles unless testing)
  // the route's first scored level over the whole tree (levels above it are kept whole) and
  // the number of its parents, every node of the level above
  int l_first, m_first;
  // fused append: the path's node at each level 0 .. L (path_leaf, its parent, ...)
  long long path_node[kMaxLevels];
};

struct NoKV {};  // route only: no attention epilogue

// What the route kernel does besides routing the stored tree (decode_append.cuh).
enum : int { kPathNone = 0, kPathAppend = 1, kPathPrefix = 2 };

struct RouteArgs;
// Launch route_tma_kernel for one KV type and summary type (route_tma_*.cu): route only
// (nokv), or route and attention / path with bf16 or fp32 K rows; fp32 summaries, or bf16
// summaries (the _s16 forms).  narrow / grouped pick the launch shape.
#define ZHA_ROUTE_LAUNCH_DECL(name)                                                                    \
  cudaError_t name(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks, int threads, \
                   size_t smem, cudaStream_t s, int path)
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_nokv);
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_bf16);
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_f32);
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_nokv_s16);
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_bf16_s16);
ZHA_ROUTE_LAUNCH_DECL(route_tma_launch_f32_s16);
#undef ZHA_ROUTE_LAUNCH_DECL


constexpr long long kRouteWaitCycles = kCopyWaitCycles;  // ~1 s at 1.9 GHz

// CTA-per-query kernel (route_group.cuh) for launches with at most two queries per SM: one
// CTA of nw (8 or 16) warps routes a query, every level's rows loaded straight into
// registers by all its warps, and attends over its leaves the same way; optionally with the
// one-leaf append path.  route_group_launch_* (route_group_{nokv,bf16,f32}.cu) launch it for
// one K/V type (s16: bf16 summaries); smem is group_smem_layout's total.
#define ZHA_GROUP_LAUNCH_DECL(name) \
  cudaError_t name(int D, bool s16, int nw, bool append, const RouteArgs& a, size_t smem, cudaStream_t s)
ZHA_GROUP_LAUNCH_DECL(route_group_launch_nokv);
ZHA_GROUP_LAUNCH_DECL(route_group_launch_bf16);
ZHA_GROUP_LAUNCH_DECL(route_group_launch_f32);
#undef ZHA_GROUP_LAUNCH_DECL

// Warp-per-query kernel (route_warp.cu) for launches with many queries: each warp routes one
// query with its candidate rows loaded straight into registers and, when attending, reads
// its leaves' K/V rows the same way.  It fits when its per-warp shared memory (candidate ids,
// keys, survivors) stays small and a query attends to at most kWarpMaxTokens tokens.
constexpr int kWarpMaxTokens = 256;
bool route_warp_fits(const zha_tree* t, int cmax, int beam);
cudaError_t launch_route_warp(zha_tree* t, const RouteArgs& a, bool attend, cudaStream_t s);

// Shared-memory layout of one query in the staged kernel.
struct RouteSmem {
  size_t rows, keys, cand, surv_a, surv_b, leaf_sc, red, hist, pw, bar, total;
};
__host__ __device__ inline size_t route_align(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline size_t route_rows_bytes(int D, int cmax, int sum_bytes) {
  return (size_t)cmax * D * sum_bytes;
}
// rows_bytes >= route_rows_bytes(D, cmax, sum_bytes); a fused decode may ask for more room to stage
// K/V, and for 16 floats of softmax weights per attending warp (pw_warps).
__host__ __device__ inline RouteSmem route_smem_layout(int D, int cmax, int beam, size_t rows_bytes,
                                                       int pw_warps) {
  RouteSmem s;
  size_t o = 0;
  s.rows = o;   // candidate summary rows [cmax][D]; K/V stage buffers after the route
  o += rows_bytes;
  s.keys = o;   // candidate keys [cmax]
  o += (size_t)cmax * 8;
  s.cand = o;   // candidate node ids [cmax]
  o += (size_t)cmax * 4;
  s.surv_a = o;
  o += (size_t)beam * 4;
  s.surv_b = o;
  o += (size_t)beam * 4;
  s.leaf_sc = o;
  o += (size_t)beam * 4;
  o = route_align(o, 16);
  s.red = o;  // per-warp partial results of the group selections [3][16]
  o += 3 * 16 * 4;
  s.hist = o;  // radix selection histogram [256]
  o += 256 * 4;
  s.pw = o;   // fused attention: per-warp softmax weights of one round [pw_warps][16]
  o += (size_t)pw_warps * 16 * 4;
  o = route_align(o, 8);
  s.bar = o;  // mbarriers: level copies / stage buffer 0 "full", buffers 1 and 2 "full",
              // then the three buffers' "empty"
  o += 48;
  s.total = route_align(o, 128);
  return s;
}

// The scoring order every route kernel uses, so that all of them give the same fp32 score
// for a (query, row) pair bit for bit: eight lanes share a row, lane l8 takes the row's
// 16-byte chunks l8, l8 + 8, ... in that order; within a chunk, elements 4i and 4i + 1 go to
// one packed accumulator and 4i + 2, 4i + 3 to another (score_fma); the lane's partial is
// (acc0.x + acc0.y) + (acc1.x + acc1.y), and the eight partials are summed by xor shuffles
// over lane distances 4, 2, 1 (score_reduce8).
__device__ __forceinline__ void score_fma(const float* q, const float* v, float2& acc0, float2& acc1) {
  acc0 = __ffma2_rn(make_float2(q[0], q[1]), make_float2(v[0], v[1]), acc0);
  acc1 = __ffma2_rn(make_float2(q[2], q[3]), make_float2(v[2], v[3]), acc1);
}
__device__ __forceinline__ float score_reduce8(float2 acc0, float2 acc1) {
  float s = (acc0.x + acc0.y) + (acc1.x + acc1.y);
  s += __shfl_xor_sync(0xffffffffu, s, 4);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  return s;
}

__device__ __forceinline__ unsigned long long route_key(float s, int node) {
  s = s + 0.0f;  // -0 -> +0 so equal scores tie exactly
  const uint32_t u = __float_as_uint(s);
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)ord << 32) | (uint32_t)(~(uint32_t)node);
}
__device__ __forceinline__ int key_node(unsigned long long k) { return (int)(~(uint32_t)k); }
__device__ __forceinline__ float key_score(unsigned long long k) {
  const uint32_t ord = (uint32_t)(k >> 32);
  const uint32_t u = (ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord;
  return __uint_as_float(u);
}

// Threshold T with exactly `beam` of keys[0, C) >= T (C > beam; keys distinct), found by
// one warp.  kr holds this lane's keys k = lane + 32 i (i < R; 0 past C), keys beyond 32 R
// are read from shared memory.  Binary search on the score word, one bit per step, with
// the warp-wide count taken from ballots; it starts below the common prefix of the
// largest and smallest score word and stops as soon as exactly `beam` keys remain.  If
// the whole score word ties at the boundary, the same search runs on the index word of
// the tied keys (larger index word = lower node index = kept first).
template <int R>
__device__ unsigned long long select_threshold(const unsigned long long (&kr)[R],
                                               const unsigned long long* keys, int C, int beam,
                                               int lane) {
  uint32_t h[R];
  uint32_t lmax = 0u, lmin = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    h[i] = (uint32_t)(kr[i] >> 32);
    if (lane + 32 * i < C) {
      lmax = max(lmax, h[i]);
      lmin = min(lmin, h[i]);
    }
  }
  const bool tail = C > 32 * R;
  for (int k = lane + 32 * R; k < C; k += 32) {
    const uint32_t x = (uint32_t)(keys[k] >> 32);
    lmax = max(lmax, x);
    lmin = min(lmin, x);
  }
  const uint32_t hmax = __reduce_max_sync(0xffffffffu, lmax);
  const uint32_t hmin = __reduce_min_sync(0xffffffffu, lmin);
  const uint32_t diff = hmax ^ hmin;
  const int top = diff ? 31 - __clz(diff) : -1;
  // T <= hmin, so count(>= T) == C > beam holds before the first step.
  uint32_t T = top < 0 ? hmax : (top >= 31 ? 0u : (hmax & ~((2u << top) - 1u)));
#pragma unroll 1
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    unsigned cnt = 0;
#pragma unroll
    for (int i = 0; i < R; ++i) cnt += __popc(__ballot_sync(0xffffffffu, h[i] >= cand));
    if (tail) {
      unsigned t = 0;
      for (int k = lane + 32 * R; k < C; k += 32) t += (uint32_t)(keys[k] >> 32) >= cand ? 1u : 0u;
      cnt += __reduce_add_sync(0xffffffffu, t);
    }
    if (cnt >= (unsigned)beam) {
      T = cand;
      if (cnt == (unsigned)beam) return (unsigned long long)T << 32;
    }
  }
  // Ties on the score word T: keep every larger score and the `need` tied keys with the
  // largest index words.
  unsigned gt = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) gt += __popc(__ballot_sync(0xffffffffu, h[i] > T));
  if (tail) {
    unsigned t = 0;
    for (int k = lane + 32 * R; k < C; k += 32) t += (uint32_t)(keys[k] >> 32) > T ? 1u : 0u;
    gt += __reduce_add_sync(0xffffffffu, t);
  }
  const unsigned need = (unsigned)beam - gt;
  uint32_t Tl = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = Tl | (1u << bit);
    unsigned cnt = 0;
#pragma unroll
    for (int i = 0; i < R; ++i)
      cnt += __popc(__ballot_sync(0xffffffffu, h[i] == T && (uint32_t)kr[i] >= cand && lane + 32 * i < C));
    if (tail) {
      unsigned t = 0;
      for (int k = lane + 32 * R; k < C; k += 32) {
        const unsigned long long key = keys[k];
        t += ((uint32_t)(key >> 32) == T && (uint32_t)key >= cand) ? 1u : 0u;
      }
      cnt += __reduce_add_sync(0xffffffffu, t);
    }
    if (cnt >= need) {
      Tl = cand;
      if (cnt == need) break;
    }
  }
  return ((unsigned long long)T << 32) | Tl;
}

// The beam-th largest of keys[0, C) (C > beam; keys distinct).  Binary search on the
// score word first (cached in registers, one bit per step, warp-wide counts), stopping as
// soon as exactly `beam` keys are at or above the threshold; only when scores tie at the
// threshold does it continue on the index word, read from shared memory.
__device__ inline unsigned long long kth_largest_key(const unsigned long long* keys, int C, int beam,
                                              int lane) {
  constexpr int R = 8;  // score words cached per lane (C <= 256 needs no shared reads)
  uint32_t hi[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int k = lane + 32 * i;
    hi[i] = k < C ? (uint32_t)(keys[k] >> 32) : 0u;
  }
  // Every key's score word lies in [hmin, hmax]; their common leading bits are fixed.
  uint32_t lmax = 0u, lmin = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (lane + 32 * i < C) {
      lmax = max(lmax, hi[i]);
      lmin = min(lmin, hi[i]);
    }
  for (int k = lane + 32 * R; k < C; k += 32) {
    const uint32_t h = (uint32_t)(keys[k] >> 32);
    lmax = max(lmax, h);
    lmin = min(lmin, h);
  }
  const uint32_t hmax = __reduce_max_sync(0xffffffffu, lmax);
  const uint32_t hmin = __reduce_min_sync(0xffffffffu, lmin);
  const uint32_t diff = hmax ^ hmin;
  const int top = diff ? 31 - __clz(diff) : -1;  // highest bit where scores differ
  // T <= hmin, so count(>= T) == C > beam holds before the first step.
  uint32_t T = top < 0 ? hmax : (top >= 31 ? 0u : (hmax & ~((2u << top) - 1u)));
#pragma unroll 1
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    unsigned cnt = 0;
#pragma unroll
    for (int i = 0; i < R; ++i) cnt += hi[i] >= cand ? 1u : 0u;
    for (int k = lane + 32 * R; k < C; k += 32) cnt += (uint32_t)(keys[k] >> 32) >= cand ? 1u : 0u;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= (unsigned)beam) {
      T = cand;
      if (cnt == (unsigned)beam) return (unsigned long long)T << 32;
    }
  }
  // Scores tie at T: keep every key with a larger score and the `need` tied keys with
  // the largest index words (= lowest node indices).
  unsigned gt = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) gt += hi[i] > T ? 1u : 0u;
  for (int k = lane + 32 * R; k < C; k += 32) gt += (uint32_t)(keys[k] >> 32) > T ? 1u : 0u;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const unsigned need = (unsigned)beam - gt;
  uint32_t Tl = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = Tl | (1u << bit);
    unsigned cnt = 0;
    for (int k = lane; k < C; k += 32) {
      const unsigned long long key = keys[k];
      cnt += ((uint32_t)(key >> 32) == T && (uint32_t)key >= cand) ? 1u : 0u;
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= need) {
      Tl = cand;
      if (cnt == need) break;
    }
  }
  return ((unsigned long long)T << 32) | Tl;
}

// One warp: keep the top-min(beam, C) of keys[0, C) and write their node ids (cand) to
// nxt in candidate order (and their scores to leaf_sc when `leaf`).  Keys and ids for
// k = lane + 32 i, i < R, are held in registers; candidates past 32 R come from shared
// memory.  Returns the number kept.
template <int R>
__device__ __forceinline__ int select_compact(const unsigned long long* keys, const int* cand, int C,
                                              int beam, int lane, int* nxt, float* leaf_sc,
                                              bool leaf) {
  unsigned long long kr[R];
  int cr[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int k = lane + 32 * i;
    kr[i] = k < C ? keys[k] : 0ull;
    cr[i] = k < C ? cand[k] : 0;
  }
  const unsigned long long T = C > beam ? select_threshold<R>(kr, keys, C, beam, lane) : 0ull;
  int kept = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const bool keep = lane + 32 * i < C && kr[i] >= T;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = kept + __popc(bal & ((1u << lane) - 1u));
      nxt[pos] = cr[i];
      if (leaf) leaf_sc[pos] = key_score(kr[i]);
    }
    kept += __popc(bal);
  }
  for (int k0 = 32 * R; k0 < C; k0 += 32) {
    const int k = k0 + lane;
    const unsigned long long key = k < C ? keys[k] : 0ull;
    const bool keep = k < C && key >= T;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = kept + __popc(bal & ((1u << lane) - 1u));
      nxt[pos] = cand[k];
      if (leaf) leaf_sc[pos] = key_score(key);
    }
    kept += __popc(bal);
  }
  return kept;
}

// One warp: top-min(beam, C) of keys[0, C) for C <= 64 (two keys per lane), by rounds that
// each take the largest remaining key (warp max of the score words, then of the index words
// when several keys share the top score: keys are distinct, so exactly one lane holds it).
// When fewer keys are dropped than kept (C - beam < beam) it takes the C - beam smallest keys
// instead, the same way, and keeps the rest.  The kept candidates are compacted in candidate
// order as in select_compact.  Fewer steps than the bit search when beam or C - beam is small.
// Returns the number kept.
__device__ __forceinline__ int select_extract(const unsigned long long* keys, const int* cand, int C, int beam,
                                              int lane, int* nxt, float* leaf_sc, bool leaf) {
  const unsigned long long k0 = lane < C ? keys[lane] : 0ull;
  const unsigned long long k1 = lane + 32 < C ? keys[lane + 32] : 0ull;
  bool keep0 = lane < C, keep1 = lane + 32 < C;
  if (C > beam && C - beam < beam) {
    // drop the C - beam smallest: rounds of warp min, absent keys count as the largest
    unsigned long long r0 = keep0 ? k0 : ~0ull, r1 = keep1 ? k1 : ~0ull;
    for (int it = 0; it < C - beam; ++it) {
      const unsigned long long low = r0 < r1 ? r0 : r1;
      const uint32_t hi = (uint32_t)(low >> 32);
      const uint32_t mh = __reduce_min_sync(0xffffffffu, hi);
      const unsigned at = __ballot_sync(0xffffffffu, hi == mh);
      uint32_t ml;
      if (__builtin_expect((at & (at - 1u)) == 0u, 1)) {
        ml = __shfl_sync(0xffffffffu, (uint32_t)low, __ffs(at) - 1);
      } else {
        ml = __reduce_min_sync(0xffffffffu, hi == mh ? (uint32_t)low : 0xFFFFFFFFu);
      }
      const unsigned long long T = ((unsigned long long)mh << 32) | ml;
      if (r0 == T) {
        r0 = ~0ull;
        keep0 = false;
      } else if (r1 == T) {
        r1 = ~0ull;
        keep1 = false;
      }
    }
  } else if (C > beam) {
    // each lane's two keys, larger first; a taken key is replaced by the lane's other one
    unsigned long long r0 = k0 > k1 ? k0 : k1, r1 = k0 > k1 ? k1 : k0;
    unsigned long long T = 0ull;
    for (int it = 0; it < beam; ++it) {
      const uint32_t hi = (uint32_t)(r0 >> 32);
      const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
      const unsigned at = __ballot_sync(0xffffffffu, hi == mh);
      uint32_t ml;
      if (__builtin_expect((at & (at - 1u)) == 0u, 1)) {  // one lane holds the top score
        ml = __shfl_sync(0xffffffffu, (uint32_t)r0, __ffs(at) - 1);
      } else {  // equal scores: the largest index word among them
        ml = __reduce_max_sync(0xffffffffu, hi == mh ? (uint32_t)r0 : 0u);
      }
      T = ((unsigned long long)mh << 32) | ml;
      if (r0 == T) {
        r0 = r1;
        r1 = 0ull;
      }
    }
    keep0 = keep0 && k0 >= T;
    keep1 = keep1 && k1 >= T;
  }
  int kept = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int k = lane + 32 * i;
    const unsigned long long key = i == 0 ? k0 : k1;
    const bool keep = i == 0 ? keep0 : keep1;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = kept + __popc(bal & ((1u << lane) - 1u));
      nxt[pos] = cand[k];
      if (leaf) leaf_sc[pos] = key_score(key);
    }
    kept += __popc(bal);
  }
  return kept;
}

// One warp's exact top-min(beam, C) selection, compacted in candidate order: the extract
// rounds for small levels and beams, else the bit search.
__device__ __forceinline__ int select_warp(const unsigned long long* keys, const int* cand, int C, int beam,
                                           int lane, int* nxt, float* leaf_sc, bool leaf) {
  if (C <= 64 && (beam <= 16 || C - beam <= 16)) return select_extract(keys, cand, C, beam, lane, nxt, leaf_sc, leaf);
  return C <= 64    ? select_compact<2>(keys, cand, C, beam, lane, nxt, leaf_sc, leaf)
         : C <= 128 ? select_compact<4>(keys, cand, C, beam, lane, nxt, leaf_sc, leaf)
                    : select_compact<8>(keys, cand, C, beam, lane, nxt, leaf_sc, leaf);
}

// Rank selection for small levels (C <= 64 nw, at most two candidates per thread of the
// query's nw warps): a key is kept iff fewer than `beam` keys of the level are greater
// (keys are distinct, so exactly min(C, beam) are kept).  Each thread counts for its
// candidates k = t and t + 32 nw against every key, reading two keys per 16-byte
// shared-memory load; no barrier per bit, and every warp of the query takes part.  The
// kept candidates are compacted in candidate order by per-warp ballots.  keys must be
// 16-byte aligned.  Every thread of the group must call it.  Returns the number kept.
__device__ __forceinline__ int select_rank_group(const unsigned long long* keys, const int* cand,
                                                 int C, int beam, int* nxt, float* leaf_sc,
                                                 bool leaf, unsigned* red, int wq, int lane, int nw,
                                                 int bar_id) {
  const int nt = 32 * nw;
  int kept_before = 0;  // kept candidates of earlier passes
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int k = 32 * wq + lane + pass * nt;
    if (pass == 1 && C <= nt) break;  // C is the same for the whole group
    const bool have = k < C;
    const unsigned long long key = have ? keys[k] : 0ull;
    int rank = 0;
    if (have && C > beam) {
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys);
      int j = 0;
#pragma unroll 4
      for (; j + 1 < C; j += 2) {
        const ulonglong2 v = k2[j >> 1];
        rank += (v.x > key ? 1 : 0) + (v.y > key ? 1 : 0);
      }
      if (j < C) rank += keys[j] > key ? 1 : 0;
    }
    const bool keep = have && rank < beam;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (nw > 1) {
      if (lane == 0) red[32 + wq] = __popc(bal);
      group_sync(bar_id, nt);
    }
    int pre = kept_before, all = kept_before;
    for (int w = 0; w < nw; ++w) {
      const int c = nw > 1 ? (int)red[32 + w] : __popc(bal);
      if (w < wq) pre += c;
      all += c;
    }
    if (keep) {
      const int pos = pre + __popc(bal & ((1u << lane) - 1u));
      nxt[pos] = cand[k];
      if (leaf) leaf_sc[pos] = key_score(key);
    }
    if (nw > 1) group_sync(bar_id, nt);  // red is reused by the next pass
    kept_before = all;
  }
  return min(C, beam);
}

// Radix variant for a query owning nw warps (C <= 32 nw): thread t = 32 wq + lane holds
// candidate t.  The threshold T (the beam-th largest key) is found eight key bits at a time
// from the top: a pass counts, in a 256-bin shared histogram, the next digit of every key
// that matches the digits fixed so far, and one warp scans the bins from the top digit down
// to find the digit holding the beam-th key.  It stops as soon as exactly `beam` keys are
// at or above the fixed prefix (usually after three or four passes; keys are distinct, so
// eight passes always settle it).  Three group barriers per pass.  The kept candidates
// are compacted in candidate order with per-warp ballots.  hist: 256 words of shared
// memory; red: 48 words.  Every thread of the group must call it.  Returns the number kept.
__device__ __forceinline__ int select_radix_group(const unsigned long long* keys, const int* cand,
                                                  int C, int beam, int* nxt, float* leaf_sc,
                                                  bool leaf, unsigned* red, unsigned* hist, int wq,
                                                  int lane, int nw, int bar_id) {
  const int t = 32 * wq + lane, nt = 32 * nw;
  const bool have = t < C;
  const unsigned long long key = have ? keys[t] : 0ull;
  const int node = have ? cand[t] : 0;
  unsigned long long T = 0ull;
  if (C > beam) {
    unsigned long long prefix = 0ull;  // the key digits above `shift` fixed so far
    int need = beam;                   // keys still to take among those matching prefix
    int shift = 56;
    for (;;) {
      for (int i = t; i < 256; i += nt) hist[i] = 0u;
      group_sync(bar_id, nt);
      const bool match = have && (shift == 56 || (key >> (shift + 8)) == prefix);
      if (match) atomicAdd(&hist[(unsigned)(key >> shift) & 255u], 1u);
      group_sync(bar_id, nt);
      if (wq == 0) {
        // lane l scans digits 255 - 8 l down to 248 - 8 l
        unsigned c[8], sum = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          c[i] = hist[255 - 8 * lane - i];
          sum += c[i];
        }
        unsigned incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)need);
        if (lane == __ffs(hit) - 1) {
          unsigned above = incl - sum;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (above + c[i] >= (unsigned)need) {
              red[0] = (unsigned)(255 - 8 * lane - i);
              red[1] = above;
              red[2] = c[i];
              break;
            }
            above += c[i];
          }
        }
      }
      group_sync(bar_id, nt);
      prefix = (prefix << 8) | red[0];
      need -= (int)red[1];
      if ((int)red[2] == need || shift == 0) break;  // exactly `need` keys carry the prefix
      shift -= 8;
    }
    T = prefix << shift;
  }
  const bool keep = have && key >= T;
  const unsigned bal = __ballot_sync(0xffffffffu, keep);
  group_sync(bar_id, nt);  // red[0..2] are read by every thread before red is reused
  if (lane == 0) red[32 + wq] = __popc(bal);
  group_sync(bar_id, nt);
  int pre = 0;
  for (int w = 0; w < wq; ++w) pre += (int)red[32 + w];
  if (keep) {
    const int pos = pre + __popc(bal & ((1u << lane) - 1u));
    nxt[pos] = node;
    if (leaf) leaf_sc[pos] = key_score(key);
  }
  return min(C, beam);
}

}  // namespace zha

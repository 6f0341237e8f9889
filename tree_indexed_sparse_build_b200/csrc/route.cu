// Top-down beam routing ("Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", abstract: future queries traverse the tree of key summaries from the top
// down to retrieve a sparse subset of keys).
//
// Survivors start as {root}.  For l = L-1 .. 0 every existing child c of a survivor is
// scored by q . S_l[c] in fp32, and the top-min(beam, #candidates) are kept, ordered by
// score descending with the lower node index first on equal scores.
//
// GPU mapping.  A candidate's key packs (order-preserving score bits, inverted node
// index) into 64 bits, so "greater key" is exactly "ranks first".  Candidates are the
// children of the survivors in ascending node order (survivors ascend, the children of
// a node are contiguous rows), so candidate k belongs to survivor k / b.
//
// Main kernel (route_tma_kernel): each level's candidate rows are staged in shared
// memory by one 1-D bulk copy (non-multicast TMA) per survivor -- its b children are
// one contiguous run of rows -- all completing on the query's mbarrier, so a level costs
// one memory round trip whatever its width and holds no registers while in flight.
// Few queries ("wide"): one query per CTA with up to 16 warps scoring from shared memory.
// Many queries ("narrow"): several queries per CTA, one warp each, no CTA barriers.
// Four lanes score one row from shared memory against q held in registers (each lane a
// quarter of the dims; the chunk order alternates between neighbouring rows so the two
// rows of a shared-memory phase use opposite bank halves), two rows per lane in flight.
// One warp per query then holds the candidate keys in registers, finds the B-th largest
// by a binary search on the key bits with ballot-based warp counts (starting below the
// common prefix of the largest and smallest score, stopping as soon as exactly B keys
// remain), and compacts the kept candidates with ballots in candidate order, which keeps
// the survivors ascending without a sort.
//
// Fallback kernel (route_reg_kernel) for levels too wide to stage in shared memory:
// the same selection, with candidate rows loaded into registers in batches.
#include <algorithm>
#include <type_traits>

#include "attn_core.cuh"
#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

constexpr int kRouteMaxWarps = 16;

struct RouteArgs {
  const void* Q;
  int q_bf16;
  int q_heads, nq, group, kv_heads;
  const float* pyr;
  long long pyr_unit_stride;  // floats
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
  int stage_tokens;          // tokens per stage buffer (two buffers in the row region)
  void* O;
  int o_bf16;
};

struct NoKV {};  // route only: no attention epilogue

constexpr long long kRouteWaitCycles = 2000000000LL;  // ~1 s at 1.9 GHz

// Shared-memory layout of one query in the staged kernel.
struct RouteSmem {
  size_t rows, keys, cand, surv_a, surv_b, leaf_sc, red, pw, bar, total;
};
__host__ __device__ inline size_t route_align(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline size_t route_rows_bytes(int D, int cmax) { return (size_t)cmax * D * 4; }
// rows_bytes >= route_rows_bytes(D, cmax); a fused decode may ask for more room to stage
// K/V, and for 16 floats of softmax weights per attending warp (pw_warps).
__host__ __device__ inline RouteSmem route_smem_layout(int D, int cmax, int beam, size_t rows_bytes,
                                                       int pw_warps) {
  RouteSmem s;
  size_t o = 0;
  s.rows = o;   // candidate summary rows, fp32 [cmax][D]; K/V stage buffers after the route
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
  s.red = o;  // per-warp partial results of the CTA-wide selection [3][16]
  o += 3 * 16 * 4;
  s.pw = o;   // fused attention: per-warp softmax weights of one round [pw_warps][16]
  o += (size_t)pw_warps * 16 * 4;
  o = route_align(o, 8);
  s.bar = o;  // two mbarriers: level copies / stage buffer 0, stage buffer 1
  o += 16;
  s.total = route_align(o, 128);
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
__device__ unsigned long long kth_largest_key(const unsigned long long* keys, int C, int beam,
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

template <int D, int U>
__global__ void __launch_bounds__(kRouteMaxWarps * 32) route_reg_kernel(const RouteArgs a) {
  constexpr int NJ = D / 32;  // 16-byte chunks per lane per row
  extern __shared__ unsigned long long route_smem[];
  __shared__ int s_m[kRouteMaxWarps];  // survivors per query of the CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = warp / a.wpq, wq = warp - qi * a.wpq;
  const long long qg = (long long)blockIdx.x * a.qpc + qi;
  const bool valid = qg < a.total_queries;
  pdl_wait();
  pdl_release();

  unsigned long long* keys = route_smem + (size_t)qi * a.query_smem_words;
  int* surv_a = reinterpret_cast<int*>(keys + a.cmax);
  int* surv_b = surv_a + a.beam;
  float* leaf_sc = reinterpret_cast<float*>(surv_b + a.beam);

  long long unit = 0;
  float q[NJ * 4];
  const int l8 = lane & 7, grp = lane >> 3;
  if (valid) {
    const long long hq_flat = qg / a.nq;  // b * q_heads + h
    const int h = (int)(hq_flat % a.q_heads);
    unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
    // This lane's slice of q: chunks c = l8 + 8j, dims 4c .. 4c+3.
    const long long qo = qg * D;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long long dim = qo + (l8 + 8 * j) * 4 + e;
        q[j * 4 + e] = a.q_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[dim])
                                : static_cast<const float*>(a.Q)[dim];
      }
  }
  if (wq == 0 && lane == 0) {
    surv_a[0] = 0;  // the root
    s_m[qi] = valid ? 1 : 0;
  }
  __syncthreads();

  const float* pyr_u = a.pyr + unit * a.pyr_unit_stride;
  int* cur = surv_a;
  int* nxt = surv_b;
  for (int l = a.L - 1; l >= 0; --l) {
    const int m = s_m[qi];
    int C = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, a.n[l] - (long long)a.b * last);
    }
    const float* S = pyr_u + a.off[l] * D;
#pragma unroll 1
    for (int k0 = wq * 4 * U; k0 < C; k0 += a.wpq * 4 * U) {
      float4 v[U][NJ];
      int node[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + 4 * u + grp;
        node[u] = -1;
        if (k < C) {
          node[u] = a.b * cur[k / a.b] + k % a.b;
          const float4* row = reinterpret_cast<const float4*>(S + (long long)node[u] * D);
#pragma unroll
          for (int j = 0; j < NJ; ++j) v[u][j] = __ldg(row + l8 + 8 * j);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float s = 0.f;
        if (node[u] >= 0) {
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            s = fmaf(q[4 * j + 0], v[u][j].x, s);
            s = fmaf(q[4 * j + 1], v[u][j].y, s);
            s = fmaf(q[4 * j + 2], v[u][j].z, s);
            s = fmaf(q[4 * j + 3], v[u][j].w, s);
          }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        const int k = k0 + 4 * u + grp;
        if (l8 == 0 && k < C) keys[k] = route_key(s, node[u]);
      }
    }
    __syncthreads();
    if (wq == 0 && C > 0) {
      // Threshold = the beam-th largest key (0 keeps everything when C <= beam).
      const unsigned long long T = C > a.beam ? kth_largest_key(keys, C, a.beam, lane) : 0ull;
      int base = 0;
      for (int k0 = 0; k0 < C; k0 += 32) {
        const int k = k0 + lane;
        const unsigned long long key = k < C ? keys[k] : 0ull;
        const bool keep = k < C && key >= T;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
          const int pos = base + __popc(bal & ((1u << lane) - 1u));
          nxt[pos] = key_node(key);
          if (l == 0) leaf_sc[pos] = key_score(key);
        }
        base += __popc(bal);
      }
      __syncwarp();
      if (a.trace) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < base ? nxt[k] : -1;
      }
      if (lane == 0) s_m[qi] = base;
    }
    __syncthreads();
    int* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  if (valid && wq == 0) {
    const int m = s_m[qi];
    int* out = a.leaf_idx + qg * a.beam;
    for (int k = lane; k < a.beam; k += 32) out[k] = k < m ? cur[k] : -1;
    if (a.leaf_score) {
      float* os = a.leaf_score + qg * a.beam;
      for (int k = lane; k < a.beam; k += 32)
        os[k] = k < m ? leaf_sc[k] : __int_as_float(0x7fc00000);
    }
  }
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

// Warp-group variant for a query owning nw warps (C <= 32 nw): thread t = 32 wq + lane of
// the group holds candidate t.  The threshold search counts with a group barrier reduction
// (named barrier bar_id over the group's 32 nw threads; one barrier per bit); the kept
// candidates are compacted in candidate order with per-warp ballots and a prefix over the
// warps' counts.  Every thread of the group must call it.  Returns the number kept.
__device__ __forceinline__ int select_compact_group(const unsigned long long* keys, const int* cand,
                                                    int C, int beam, int* nxt, float* leaf_sc,
                                                    bool leaf, unsigned* red, int wq, int lane,
                                                    int nw, int bar_id) {
  const int t = 32 * wq + lane, nt = 32 * nw;
  const bool have = t < C;
  const unsigned long long key = have ? keys[t] : 0ull;
  const int node = have ? cand[t] : 0;
  const uint32_t h = (uint32_t)(key >> 32);
  unsigned long long T = 0ull;
  if (C > beam) {
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, have ? h : 0u);
    const uint32_t wmin = __reduce_min_sync(0xffffffffu, have ? h : 0xFFFFFFFFu);
    if (lane == 0) {
      red[wq] = wmax;
      red[16 + wq] = wmin;
    }
    group_sync(bar_id, nt);
    uint32_t hmax = 0u, hmin = 0xFFFFFFFFu;
    for (int w = 0; w < nw; ++w) {
      hmax = max(hmax, red[w]);
      hmin = min(hmin, red[16 + w]);
    }
    const uint32_t diff = hmax ^ hmin;
    const int top = diff ? 31 - __clz(diff) : -1;
    uint32_t Th = top < 0 ? hmax : (top >= 31 ? 0u : (hmax & ~((2u << top) - 1u)));
    bool done = false;
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t c = Th | (1u << bit);
      const int cnt = group_count(bar_id, nt, have && h >= c);
      if (cnt >= beam) {
        Th = c;
        if (cnt == beam) {
          done = true;
          break;
        }
      }
    }
    if (done) {
      T = (unsigned long long)Th << 32;
    } else {
      const int need = beam - group_count(bar_id, nt, have && h > Th);
      uint32_t Tl = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t c = Tl | (1u << bit);
        const int cnt = group_count(bar_id, nt, have && h == Th && (uint32_t)key >= c);
        if (cnt >= need) {
          Tl = c;
          if (cnt == need) break;
        }
      }
      T = ((unsigned long long)Th << 32) | Tl;
    }
  }
  const bool keep = have && key >= T;
  const unsigned bal = __ballot_sync(0xffffffffu, keep);
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

// Staged routing.  qpc queries per CTA, wpq warps per query (blockDim.x = 32 qpc wpq).
// GROUPED (wpq > 1): the warps of query qi synchronise on named barrier 1 + qi; otherwise
// each query is one warp, synchronised only within the warp.
//
// With TKV = the KV storage type (not NoKV) the kernel is the fused decode: once the
// last level is selected, the query's warps attend over the tokens of its leaves.  The
// candidate-row region, free after the leaf-level scoring, becomes two K/V stage buffers
// filled by one bulk copy per leaf piece (K and V) on the two mbarriers; the warps run
// the online softmax of attn_core.cuh over each stage, merge their states through shared
// memory and write O.  No leaf list goes through global memory and nothing is launched
// between the route and the attention.
// NARROW instantiations are built for CTAs of at most 8 warps, three per SM (register cap).
template <int D, bool GROUPED, typename TKV, bool NARROW>
__global__ void __launch_bounds__(NARROW ? 256 : kRouteMaxWarps * 32, NARROW ? 3 : 1)
    route_tma_kernel(const RouteArgs a) {
  constexpr bool ATTEND = !std::is_same<TKV, NoKV>::value;
  constexpr int CPL = D / 16;  // 16-byte chunks of a row per lane (4 lanes per row)
  constexpr int R = 8;         // candidate keys held per lane in the selecting warp
  extern __shared__ __align__(128) unsigned char rsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = GROUPED ? a.wpq : 1;  // warps of this query
  const int qi = warp / nw;
  const int wq = warp - qi * nw;
  const int bar_id = 1 + qi, bar_n = 32 * nw;
  const long long qg = (long long)blockIdx.x * a.qpc + qi;
  const bool valid = qg < a.total_queries;
  const RouteSmem Ls =
      route_smem_layout(D, a.cmax, a.beam, (size_t)a.rows_bytes, ATTEND ? nw : 0);
  unsigned char* base = rsm + (size_t)qi * a.query_smem_bytes;
  const float* rows = reinterpret_cast<const float*>(base + Ls.rows);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(base + Ls.keys);
  int* cand = reinterpret_cast<int*>(base + Ls.cand);
  int* surv_a = reinterpret_cast<int*>(base + Ls.surv_a);
  int* surv_b = reinterpret_cast<int*>(base + Ls.surv_b);
  float* leaf_sc = reinterpret_cast<float*>(base + Ls.leaf_sc);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + Ls.bar);
  unsigned* red = reinterpret_cast<unsigned*>(base + Ls.red);

  auto qsync = [&]() {  // all warps of this query
    if (GROUPED) group_sync(bar_id, bar_n); else __syncwarp();
  };
  pdl_wait();
  pdl_release();

  long long unit = 0;
  if (valid) {
    const long long hq_flat = qg / a.nq;
    const int h = (int)(hq_flat % a.q_heads);
    unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
  }
  const float* pyr_u = a.pyr + unit * a.pyr_unit_stride;
  if (wq == 0 && lane == 0) {
    mbar_init(&bar[0], 1);
    if (ATTEND) mbar_init(&bar[1], 1);
    fence_mbar_init();
    surv_a[0] = 0;  // the root
  }
  qsync();

  // Four lanes per row: lane (rg = lane / 4, sub = lane % 4) reads chunks 4 (j ^ par) + sub,
  // par = rg & 1, so the two rows of a shared-memory phase use opposite bank halves.
  const int sub = lane & 3, rg = lane >> 2, par = rg & 1;
  float4 qv[CPL];
  int* cur = surv_a;
  int* nxt = surv_b;
  int m = valid ? 1 : 0;
  uint32_t parity = 0;
  for (int l = a.L - 1; l >= 0; --l) {
    int C = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, a.n[l] - (long long)a.b * last);
    }
    const float* S = pyr_u + a.off[l] * D;
    if (wq == 0 && C > 0) {
      // one bulk copy per survivor (its children are consecutive rows) + candidate ids
      if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)C * D * 4);
      __syncwarp();
      fence_proxy_async_smem();
      for (int j = lane; j < m; j += 32) {
        const long long node0 = (long long)a.b * cur[j];
        const int nc = (int)min((long long)a.b, a.n[l] - node0);
        bulk_copy_g2s((void*)(rows + (size_t)j * a.b * D), S + node0 * D, (uint32_t)nc * D * 4, bar);
      }
      for (int k = lane; k < C; k += 32) cand[k] = a.b * cur[k / a.b] + k % a.b;
    }
    if (l == a.L - 1 && valid) {  // load q while the first level is in flight
      const long long qo = qg * D;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = 4 * (j ^ par) + sub;
        float f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          f[e] = a.q_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[qo + 4 * c + e])
                          : static_cast<const float*>(a.Q)[qo + 4 * c + e];
        qv[j] = make_float4(f[0], f[1], f[2], f[3]);
      }
    }
    const bool ok = C == 0 || mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, kRouteWaitCycles);
    const bool failed = GROUPED ? group_any(bar_id, bar_n, !ok) : __any_sync(0xffffffffu, !ok);
    if (failed) {
      if (wq == 0 && lane == 0 && C > 0)  // let the copies land before the CTA exits
        mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, kRouteWaitCycles);
      return;  // the whole group leaves together
    }
    if (!GROUPED) __syncwarp();  // candidate ids written by other lanes
    if (C > 0) parity ^= 1u;

    // score: rows r = 8 (wq + nw t) + rg, two rows per lane in flight
    for (int r0 = 8 * wq; r0 < C; r0 += 16 * nw) {
      float acc[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = r0 + 8 * nw * u + rg;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[u][e] = 0.f;
        if (r < C) {
          const float4* row = reinterpret_cast<const float4*>(rows + (size_t)r * D);
#pragma unroll
          for (int j = 0; j < CPL; ++j) {
            const float4 v = row[4 * (j ^ par) + sub];
            acc[u][0] = fmaf(qv[j].x, v.x, acc[u][0]);
            acc[u][1] = fmaf(qv[j].y, v.y, acc[u][1]);
            acc[u][2] = fmaf(qv[j].z, v.z, acc[u][2]);
            acc[u][3] = fmaf(qv[j].w, v.w, acc[u][3]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float s = (acc[u][0] + acc[u][1]) + (acc[u][2] + acc[u][3]);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        const int r = r0 + 8 * nw * u + rg;
        if (sub == 0 && r < C) keys[r] = route_key(s, cand[r]);
      }
    }
    qsync();
    if (C > 0 && C <= 128 && C <= 64 * nw) {  // C is the same for the whole group
      const int kept =
          select_rank_group(keys, cand, C, a.beam, nxt, leaf_sc, l == 0, red, wq, lane, nw, bar_id);
      qsync();
      if (wq == 0 && a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    } else if (GROUPED && C <= 32 * nw) {
      const int kept =
          select_compact_group(keys, cand, C, a.beam, nxt, leaf_sc, l == 0, red, wq, lane, nw, bar_id);
      group_sync(bar_id, bar_n);
      if (wq == 0 && a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    } else if (wq == 0 && C > 0) {
      const int kept = C <= 64    ? select_compact<2>(keys, cand, C, a.beam, lane, nxt, leaf_sc, l == 0)
                       : C <= 128 ? select_compact<4>(keys, cand, C, a.beam, lane, nxt, leaf_sc, l == 0)
                                  : select_compact<R>(keys, cand, C, a.beam, lane, nxt, leaf_sc, l == 0);
      __syncwarp();
      if (a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    }
    m = min(C, a.beam);
    qsync();
    int* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  if (valid && wq == 0 && a.leaf_idx) {
    int* out = a.leaf_idx + qg * a.beam;
    for (int k = lane; k < a.beam; k += 32) out[k] = k < m ? cur[k] : -1;
  }
  if (valid && wq == 0 && a.leaf_score) {
    float* os = a.leaf_score + qg * a.beam;
    for (int k = lane; k < a.beam; k += 32) os[k] = k < m ? leaf_sc[k] : __int_as_float(0x7fc00000);
  }
  if constexpr (ATTEND) {
    using S = AttnShape<TKV, D>;
    constexpr int ROWB = S::ROWB;
    const int TS = a.stage_tokens;
    const int lb = (int)a.lb;
    unsigned char* sb = base + Ls.rows;  // stage buffer b: K rows at sb + 2 b TS ROWB, V after
    const size_t stage_bytes = (size_t)TS * ROWB;
    // Tokens of the selected leaves in slot order.  Only leaf n0 - 1 can hold fewer than
    // lb tokens, and survivors ascend, so it can only be the last one.
    int total = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      total = (m - 1) * lb + (int)(min(last * a.lb + a.lb, a.N) - last * a.lb);
    }
    const int nst = (total + TS - 1) / TS;
    const char* Ku = a.K + unit * a.kv_unit_stride;
    const char* Vu = a.V + unit * a.kv_unit_stride;
    // Stage st covers tokens [st TS, min(st TS + TS, total)) in buffer st & 1; the lanes of
    // warp 0 each copy the K and V pieces of some of its leaves.
    auto issue = [&](int st) {
      const int b = st & 1;
      unsigned char* kb = sb + (size_t)b * 2 * stage_bytes;
      const int w0 = st * TS, w1 = min(w0 + TS, total);
      if (lane == 0) mbar_arrive_expect_tx(&bar[b], (uint32_t)(2 * (w1 - w0) * ROWB));
      __syncwarp();
      fence_proxy_async_smem();
      for (int j = w0 / lb + lane; j <= (w1 - 1) / lb; j += 32) {
        const int p0 = j * lb;
        const int a0 = max(p0, w0), a1 = min(p0 + lb, w1);
        const long long row = (long long)cur[j] * a.lb + (a0 - p0);
        const uint32_t bytes = (uint32_t)((a1 - a0) * ROWB);
        bulk_copy_g2s(kb + (size_t)(a0 - w0) * ROWB, Ku + row * ROWB, bytes, &bar[b]);
        bulk_copy_g2s(kb + stage_bytes + (size_t)(a0 - w0) * ROWB, Vu + row * ROWB, bytes, &bar[b]);
      }
    };
    // phase of the wait for stage st: bar[0] carries on from the route's level copies
    auto phase = [&](int st) -> uint32_t { return ((st & 1) ? 0u : parity) ^ (uint32_t)((st >> 1) & 1); };
    if (wq == 0 && nst > 0) {
      issue(0);
      if (nst > 1) issue(1);
    }
    float qa[S::CPL][S::VEC];
    if (valid) attn_load_q<TKV, D>(a.Q, a.q_bf16 != 0, qg, lane, qa);
    float* pw = reinterpret_cast<float*>(base + Ls.pw) + wq * 16;
    float m_w = -INFINITY, l_w = 0.f;
    float acc[S::DPL];
#pragma unroll
    for (int e = 0; e < S::DPL; ++e) acc[e] = 0.f;
    int fail_st = -1;
    for (int st = 0; st < nst; ++st) {
      const int b = st & 1;
      const bool ok = mbar_wait_bounded(&bar[b], phase(st), a.err, kDevErrTimeout, kRouteWaitCycles);
      // the stage is visible to every warp, and every warp is done with stage st - 1, whose
      // buffer the copy of stage st + 1 now reuses
      const bool bad = GROUPED ? group_any(bar_id, bar_n, !ok) : __any_sync(0xffffffffu, !ok);
      if (bad) {
        fail_st = st;
        break;
      }
      if (wq == 0 && st >= 1 && st + 1 < nst) issue(st + 1);
      const unsigned char* Ks = sb + (size_t)b * 2 * stage_bytes;
      attn_tokens<TKV, D>(Ks, Ks + stage_bytes, min(TS, total - st * TS), 8 * wq, 8 * nw, 16 * nw, qa,
                          a.qk_scale, pw, m_w, l_w, acc, lane);
    }
    if (fail_st >= 0) {
      // let the copies in flight land before the CTA's shared memory is released; the
      // query's output is poisoned so the failure shows besides the error word
      // (stages 0 and 1 are issued up front, stage st + 1 only after stage st's barrier)
      const int last_issued = min(max(fail_st, 1), nst - 1);
      if (wq == 0 && lane == 0)
        for (int st = fail_st; st <= last_issued; ++st)
          mbar_wait_bounded(&bar[st & 1], phase(st), a.err, kDevErrTimeout, kRouteWaitCycles);
      if (valid && wq == 0)
        for (int e = lane; e < D; e += 32) {
          if (a.o_bf16)
            static_cast<uint16_t*>(a.O)[qg * D + e] = 0x7FC0u;
          else
            static_cast<float*>(a.O)[qg * D + e] = __int_as_float(0x7fc00000);
        }
      return;
    }
    l_w = warp_sum(l_w);
    if (GROUPED) {
      // merge the warps' states; the accumulators reuse the stage buffers
      float* accr = reinterpret_cast<float*>(sb);
      float* redf = reinterpret_cast<float*>(red);
      group_sync(bar_id, bar_n);
#pragma unroll
      for (int e = 0; e < S::DPL; ++e) accr[wq * D + lane * S::DPL + e] = acc[e];
      if (lane == 0) {
        redf[wq] = m_w;
        redf[16 + wq] = l_w;
      }
      group_sync(bar_id, bar_n);
      for (int d = 32 * wq + lane; d < D && valid; d += bar_n) {
        float M = -INFINITY;
        for (int w = 0; w < nw; ++w) M = fmaxf(M, redf[w]);
        float o = 0.f, l = 0.f;
        for (int w = 0; w < nw; ++w) {
          const float sw = redf[w] == -INFINITY ? 0.f : exp2f(redf[w] - M);
          o = fmaf(sw, accr[w * D + d], o);
          l = fmaf(sw, redf[16 + w], l);
        }
        const float r = l > 0.f ? o / l : 0.f;
        if (a.o_bf16)
          static_cast<uint16_t*>(a.O)[qg * D + d] = f32_to_bf16_bits(r);
        else
          static_cast<float*>(a.O)[qg * D + d] = r;
      }
    } else if (valid) {
#pragma unroll
      for (int e = 0; e < S::DPL; ++e) {
        const float r = l_w > 0.f ? acc[e] / l_w : 0.f;
        const long long o = qg * D + lane * S::DPL + e;
        if (a.o_bf16)
          static_cast<uint16_t*>(a.O)[o] = f32_to_bf16_bits(r);
        else
          static_cast<float*>(a.O)[o] = r;
      }
    }
  }
}

namespace {
template <int D, bool GROUPED, typename TKV, bool NARROW>
cudaError_t run_route_tma(const RouteArgs& a, unsigned blocks, int threads, size_t smem,
                          cudaStream_t s) {
  auto kern = route_tma_kernel<D, GROUPED, TKV, NARROW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TKV>
cudaError_t run_route_tma_d(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks,
                            int threads, size_t smem, cudaStream_t s) {
  if (narrow) {
    if (grouped)
      return D == 128 ? run_route_tma<128, true, TKV, true>(a, blocks, threads, smem, s)
                      : run_route_tma<64, true, TKV, true>(a, blocks, threads, smem, s);
    return D == 128 ? run_route_tma<128, false, TKV, true>(a, blocks, threads, smem, s)
                    : run_route_tma<64, false, TKV, true>(a, blocks, threads, smem, s);
  }
  if (grouped)
    return D == 128 ? run_route_tma<128, true, TKV, false>(a, blocks, threads, smem, s)
                    : run_route_tma<64, true, TKV, false>(a, blocks, threads, smem, s);
  return D == 128 ? run_route_tma<128, false, TKV, false>(a, blocks, threads, smem, s)
                  : run_route_tma<64, false, TKV, false>(a, blocks, threads, smem, s);
}

template <int D, int U>
cudaError_t run_route(const RouteArgs& a, unsigned blocks, int threads, size_t smem,
                      cudaStream_t s) {
  auto kern = route_reg_kernel<D, U>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

constexpr size_t kRouteSmemCap = 200 * 1024;  // staged kernel: shared memory per query

// Arguments common to the route and the fused decode.
RouteArgs route_args(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                     int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace) {
  RouteArgs a{};
  const int D = t->desc.head_dim;
  a.Q = d_Q;
  a.q_bf16 = q_dtype == ZHA_BF16;
  a.q_heads = q_heads;
  a.nq = nq;
  a.kv_heads = t->desc.kv_heads;
  a.group = q_heads / t->desc.kv_heads;
  a.pyr = t->pyr;
  a.pyr_unit_stride = t->unit_rows * D;
  for (int l = 0; l <= t->L; ++l) {
    a.off[l] = t->off[l];
    a.n[l] = t->n[l];
  }
  a.L = t->L;
  a.b = t->desc.branching;
  a.beam = beam;
  long long cmax = 1;
  for (int l = 0; l < t->L; ++l)
    cmax = std::max(cmax, std::min(std::min((long long)beam, t->n[l + 1]) * a.b, t->n[l]));
  a.cmax = (int)cmax;
  a.total_queries = (long long)t->desc.batch * q_heads * nq;
  a.leaf_idx = d_leaf_idx;
  a.leaf_score = d_leaf_score;
  a.trace = d_trace;
  a.err = t->d_err;
  return a;
}

// Warps per query in narrow launches: enough that each warp scores about 16 rows of the
// widest level (at most 4).
#ifndef ZHA_NARROW_WPQ
#define ZHA_NARROW_WPQ 0  // 0: by the widest level; else a fixed count (1, 2 or 4)
#endif
int narrow_wpq(long long cmax) {
  if (ZHA_NARROW_WPQ > 0) return ZHA_NARROW_WPQ;
  return (int)std::min<long long>(4, std::max<long long>(1, (cmax + 15) / 16));
}

// Launch shape of the staged kernel.  Wide (at most two queries per SM): one query per
// CTA, enough warps for the widest level (and, fused, for the attention tokens).
// Narrow: up to 8 warps per CTA, narrow_wpq warps per query.
struct StagedShape {
  bool wide, grouped;
  unsigned blocks;
  int threads;
  size_t smem;
};
StagedShape staged_shape(const zha_tree* t, RouteArgs& a, size_t per_query, int attn_warps) {
  StagedShape sh{};
  sh.wide = a.total_queries <= 2LL * t->sms;
  if (sh.wide) {
    const long long want = std::max<long long>((a.cmax + 31) / 32, attn_warps);
    a.wpq = (int)std::max(1LL, std::min<long long>(kRouteMaxWarps, want));
    a.qpc = 1;
    sh.blocks = (unsigned)a.total_queries;
    sh.smem = per_query;
  } else {
    a.wpq = narrow_wpq(a.cmax);
    a.qpc = (int)std::max<size_t>(1, std::min<size_t>(8 / a.wpq, (96 * 1024) / per_query));
    sh.blocks = (unsigned)((a.total_queries + a.qpc - 1) / a.qpc);
    sh.smem = per_query * a.qpc;
  }
  sh.threads = 32 * a.wpq * a.qpc;
  sh.grouped = a.wpq > 1;
  return sh;
}
}  // namespace

cudaError_t launch_route(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads,
                         int nq, int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                         cudaStream_t stream) {
  RouteArgs a = route_args(t, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace);
  const int D = t->desc.head_dim;
  const long long cmax = a.cmax;
  cudaError_t e;

  // Staged kernel when a query's widest level fits in shared memory.
  a.rows_bytes = (int)route_rows_bytes(D, a.cmax);
  const size_t per_query = route_smem_layout(D, a.cmax, beam, a.rows_bytes, 0).total;
  if (per_query <= kRouteSmemCap) {
    a.query_smem_bytes = (int)per_query;
    // 8 rows per warp step, two steps in flight
    const StagedShape sh = staged_shape(t, a, per_query, 0);
    e = run_route_tma_d<NoKV>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream);
    ++t->launches;
    return e;
  }

  // Register kernel.  Warps per query: enough to cover the widest level in one batch, but
  // no more than the SMs can hold for this many queries.
  constexpr int kU128 = 2, kU64 = 4;
  const int rows_per_batch = 4 * (D == 128 ? kU128 : kU64);
  const long long need = (cmax + rows_per_batch - 1) / rows_per_batch;
  const long long room = std::max(1LL, (long long)t->sms * 32 / std::max(1LL, a.total_queries));
  int wpq = (int)std::min<long long>(kRouteMaxWarps, std::min(need, room));
  wpq = std::max(wpq, 1);
  const int cta_warps = wpq > 8 ? kRouteMaxWarps : 8;
  a.wpq = wpq;
  a.qpc = std::max(1, cta_warps / wpq);
  // keys (8 B each) + two survivor lists (4 B) + leaf scores (4 B), rounded to 8 B words
  const long long words = cmax + (3LL * beam * 4 + 7) / 8;
  a.query_smem_words = (int)words;
  const size_t smem = (size_t)words * 8 * a.qpc;
  const int threads = a.qpc * a.wpq * 32;
  const unsigned blocks = (unsigned)((a.total_queries + a.qpc - 1) / a.qpc);
  e = D == 128 ? run_route<128, kU128>(a, blocks, threads, smem, stream)
               : run_route<64, kU64>(a, blocks, threads, smem, stream);
  ++t->launches;
  return e;
}

// Fused route + attention (one launch).  Wide launches (one query per CTA): the row
// region grows up to 128 KB when the attention wants bigger stages, so a long leaf list
// streams in a few large stages.  Narrow launches (several queries per SM): the row region
// stays the route's own, since a larger one would cut the queries resident per SM, and the
// call is fused only when the query's tokens then fit in at most two stages; otherwise
// fused = false and the route and the attention run as two launches.  Stages hold at
// least 8 tokens.
DecodePlan plan_decode(const zha_tree* t, int q_heads, int nq, int beam) {
  DecodePlan p{};
  const int D = t->desc.head_dim;
  const int row = D * (t->desc.kv_dtype == ZHA_BF16 ? 2 : 4);
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  const bool wide = queries <= 2LL * t->sms;
  long long cmax = 1;
  for (int l = 0; l < t->L; ++l)
    cmax = std::max(cmax, std::min(std::min((long long)beam, t->n[l + 1]) * t->desc.branching, t->n[l]));
  const long long tokens = std::min((long long)beam * t->desc.leaf_block, t->N);
  const size_t route_rows = route_rows_bytes(D, (int)cmax);
  const size_t want = (size_t)4 * row * (size_t)((tokens + 1) / 2);  // two stages
  size_t rows = wide ? std::max(route_rows, std::min(want, (size_t)128 * 1024)) : route_rows;
  rows = std::max(rows, (size_t)4 * 8 * row);
  p.stage_tokens = (int)(rows / (4 * row)) / 8 * 8;
  p.rows_bytes = rows;
  p.attn_warps = wide ? (int)std::min<long long>(kRouteMaxWarps, (tokens + 31) / 32) : 1;
  p.smem_per_query =
      route_smem_layout(D, (int)cmax, beam, rows, wide ? kRouteMaxWarps : narrow_wpq(cmax)).total;
  p.fused = p.smem_per_query <= kRouteSmemCap && (wide || 2LL * p.stage_tokens >= tokens);
  return p;
}

cudaError_t launch_decode(zha_tree* t, const DecodePlan& p, const void* d_Q, zha_dtype q_dtype,
                          int q_heads, int nq, int beam, const void* d_K, const void* d_V,
                          float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                          void* d_O, zha_dtype o_dtype, cudaStream_t stream) {
  RouteArgs a = route_args(t, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace);
  const int D = t->desc.head_dim;
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  a.rows_bytes = (int)p.rows_bytes;
  a.K = static_cast<const char*>(d_K);
  a.V = static_cast<const char*>(d_V);
  a.kv_unit_stride = t->desc.capacity_tokens * D * (bf ? 2LL : 4LL);
  a.lb = t->desc.leaf_block;
  a.N = t->N;
  a.qk_scale = scale * 1.4426950408889634f;
  a.stage_tokens = p.stage_tokens;
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  a.query_smem_bytes = (int)p.smem_per_query;  // weight area sized for 16 warps when wide
  const StagedShape sh = staged_shape(t, a, p.smem_per_query, p.attn_warps);
  cudaError_t e;
  if (bf)
    e = run_route_tma_d<uint16_t>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream);
  else
    e = run_route_tma_d<float>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream);
  ++t->launches;
  return e;
}

}  // namespace zha

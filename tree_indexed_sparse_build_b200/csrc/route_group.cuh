// CTA-per-query routing (and route + attention, optionally with the one-leaf append) for
// launches with at most two queries per SM.
//
// Top-down beam routing ("Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", abstract: future queries traverse the tree of key summaries from the top down
// to retrieve a sparse subset of keys, and attention runs over that subset).
//
// With few queries per SM a query's time is a chain of dependent steps: each level's rows,
// its selection, then the attended tokens.  Here one CTA of NW warps owns the query and
// every step uses all of them: a level's candidate rows are loaded straight into registers,
// 4 P rows per warp per round (P row passes of 16-byte loads in flight per lane), so a level
// of up to 4 P NW candidates is one memory round trip; the attention splits the leaves'
// tokens over the warps the same way (attn_regs.cuh) and merges their softmax states
// through shared memory.  Nothing is staged in shared memory, so no bytes cross it twice
// and no copy has to be waited for, except the append path's (below).
//
// Scoring follows the order all route kernels share (score_fma / score_reduce8,
// route_common.cuh: eight lanes per row, lane l8 takes 16-byte chunks l8 + 8 j; the four
// rows of a pass group are summed by one transposed butterfly), so scores, leaves, survivors
// and leaf scores are bit-identical to the other kernels'.  The keys stay in the registers
// of the lanes that scored them, and the selection (select_regs) keeps the same exact
// top-min(beam, C) over the packed (score, inverted node index) keys in three barriers.
//
// The setup is kept off the chain as far as it goes: the host passes the first scored level
// and the path's nodes, the query is loaded while the path's copies are in flight, and the
// first level's rows are prefetched into L2 meanwhile.
//
// APPEND (fused decode step): the tokens appended to one leaf change only the path from that
// leaf to the root.  Thread 0 issues bulk copies of the leaf's tokens and of each level's
// children of the path node (decode_append.cuh) before anything else; the CTA recomputes
// the path rows with the stand-alone append's arithmetic, the unit's first query stores
// them, and each CTA scores the path node's row from its own recomputed copy, so no CTA
// waits for another.  That copy wait is bounded like every other (first_wait, then the
// drain bound): a wait that runs out marks the query's results lost.
#pragma once

#include <algorithm>
#include <type_traits>

#include "attn_regs.cuh"
#include "decode_append.cuh"
#include "device_common.cuh"
#include "route_common.cuh"
#include "zha_internal.h"

namespace zha {

// Shared memory of one query (one CTA of nw warps).
struct GroupSmem {
  size_t keys, sk, sr, hw, surv_a, surv_b, leaf_sc, am, al, aw, aacc, path, total;
};
__host__ __device__ inline GroupSmem group_smem_layout(int D, int cmax, int beam, int nw, size_t path_bytes) {
  GroupSmem s;
  size_t o = 0;
  s.keys = o;  // candidate keys [cmax]
  o = route_align(o + (size_t)cmax * 8, 16);
  s.sk = o;  // the selection's surviving keys [cmax], in candidate order
  o = route_align(o + (size_t)cmax * 8, 16);
  s.sr = o;  // their candidate slots [cmax]
  o = route_align(o + (size_t)cmax * 4, 16);
  s.hw = o;  // the selection's lane maxima (score words) [32]
  o += 32 * 4;
  s.surv_a = o;
  o += (size_t)beam * 4;
  s.surv_b = o;
  o += (size_t)beam * 4;
  s.leaf_sc = o;
  o += (size_t)beam * 4;
  s.am = o;  // attention: per-warp running max [nw]
  o += (size_t)nw * 4;
  s.al = o;  // per-warp softmax sums [nw]
  o += (size_t)nw * 4;
  s.aw = o;  // per-warp merge weights [nw], then 1 / the merged sum
  o += (size_t)(nw + 1) * 4;
  o = route_align(o, 16);
  s.aacc = o;  // per-warp output rows [nw][D]
  o += (size_t)nw * D * 4;
  o = route_align(o, 128);
  s.path = o;  // the append path (decode_append.cuh)
  o += path_bytes;
  s.total = route_align(o, 128);
  return s;
}

// Node id of candidate slot r: the first scored level's candidates are all its nodes (cur
// null); below, survivor j's children are slots j b .. j b + b - 1.
__device__ __forceinline__ int cand_node(const int* cur, int b, int r) {
  if (cur == nullptr) return r;
  const int j = r / b;
  return b * cur[j] + (r - j * b);
}

// One warp: exact top-min(beam, C) of keys[0, C) (C <= 32 R; keys distinct), written to
// nxt as node ids in candidate order (scores to leaf_sc when `leaf`).  Lane holds keys
// lane + 32 i.  The steps are kept short and independent, and no step shuffles more than
// once: a lone warp pays every latency.
//  1. Threshold on the score words: T = the beam-th largest of the 32 lanes' largest score
//     words (counted with ties).  At least beam lanes hold a key whose score word is >= T,
//     so the beam-th largest key's score word is >= T and every kept key passes.
//  2. The keys with score word >= T (usually a few times beam) are compacted in candidate
//     order.
//  3. A survivor is kept when fewer than beam survivors are above it; the kept ones keep
//     their candidate order, so a ballot places them.
// When only a few candidates are dropped (C - beam <= 2, C <= 64) they are found directly:
// the smallest key (two warp minimum reductions, score word then index word), C - beam times.
// No CTA barrier: the caller synchronises before keys are read and after nxt is written.
template <int R>
__device__ __forceinline__ int select_lanes(const unsigned long long* keys, int C, int beam, const int* cur, int b,
                                            int* nxt, float* leaf_sc, bool leaf, unsigned long long* sk, int* sr,
                                            uint32_t* hw) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  unsigned long long k[R];
#pragma unroll
  for (int i = 0; i < R; ++i) k[i] = lane + 32 * i < C ? keys[lane + 32 * i] : 0ull;
  if (C <= beam || (R == 2 && C - beam <= 2)) {
    // drop the C - beam smallest keys (none when C <= beam), keep the rest in place order
    bool drop[R];
#pragma unroll
    for (int i = 0; i < R; ++i) drop[i] = lane + 32 * i >= C;
    for (int d = 0; d < C - beam; ++d) {  // the smallest remaining key: score word, then index word
      unsigned long long mn = ~0ull;
#pragma unroll
      for (int i = 0; i < R; ++i) mn = !drop[i] && k[i] < mn ? k[i] : mn;
      const uint32_t mh = __reduce_min_sync(0xffffffffu, (uint32_t)(mn >> 32));
      const uint32_t ml = __reduce_min_sync(0xffffffffu, (uint32_t)(mn >> 32) == mh ? (uint32_t)mn : 0xffffffffu);
      const unsigned long long m = ((unsigned long long)mh << 32) | ml;
#pragma unroll
      for (int i = 0; i < R; ++i) drop[i] = drop[i] || k[i] == m;  // keys are distinct
    }
    int base = 0;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const unsigned kb = __ballot_sync(0xffffffffu, !drop[i]);
      if (!drop[i]) {
        const int pos = base + __popc(kb & lt);
        nxt[pos] = cand_node(cur, b, lane + 32 * i);
        if (leaf) leaf_sc[pos] = key_score(k[i]);
      }
      base += __popc(kb);
    }
    return base;
  }
  uint32_t h[R];
#pragma unroll
  for (int i = 0; i < R; ++i) h[i] = (uint32_t)(k[i] >> 32);  // empty slots: 0
  uint32_t hm = 0u;
#pragma unroll
  for (int i = 0; i < R; ++i) hm = max(hm, h[i]);
  hw[lane] = hm;  // every lane reads all 32 words back (broadcast loads, no shuffles)
  __syncwarp();
  int gt0 = 0, gt1 = 0, ge0 = 0, ge1 = 0;
  const uint4* h4 = reinterpret_cast<const uint4*>(hw);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 v = h4[q];
    gt0 += (v.x > hm ? 1 : 0) + (v.y > hm ? 1 : 0);
    ge0 += (v.x >= hm ? 1 : 0) + (v.y >= hm ? 1 : 0);
    gt1 += (v.z > hm ? 1 : 0) + (v.w > hm ? 1 : 0);
    ge1 += (v.z >= hm ? 1 : 0) + (v.w >= hm ? 1 : 0);
  }
  // the lanes holding the beam-th largest word (none when beam > 32: every key survives)
  const unsigned qb = __ballot_sync(0xffffffffu, gt0 + gt1 < beam && ge0 + ge1 >= beam);
  const uint32_t T = qb ? __shfl_sync(0xffffffffu, hm, __ffs(qb) - 1) : 0u;
  unsigned bal[R];
#pragma unroll
  for (int i = 0; i < R; ++i) bal[i] = __ballot_sync(0xffffffffu, lane + 32 * i < C && h[i] >= T);
  int S = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if ((bal[i] >> lane) & 1u) {
      sk[S + __popc(bal[i] & lt)] = k[i];
      sr[S + __popc(bal[i] & lt)] = lane + 32 * i;
    }
    S += __popc(bal[i]);
  }
  __syncwarp();
  const ulonglong2* s2 = reinterpret_cast<const ulonglong2*>(sk);
  int kept = 0;
  for (int j0 = 0; j0 < S; j0 += 32) {
    const int j = j0 + lane;
    const unsigned long long key = j < S ? sk[j] : ~0ull;
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
    if (S <= 32) {  // one survivor per lane: every comparison unrolled
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        if (i < S) {
          const ulonglong2 v = s2[i >> 1], w = s2[(i >> 1) + 1];
          c0 += v.x > key && i < S ? 1 : 0;
          c1 += v.y > key && i + 1 < S ? 1 : 0;
          c2 += w.x > key && i + 2 < S ? 1 : 0;
          c3 += w.y > key && i + 3 < S ? 1 : 0;
        }
      }
    } else {
      for (int i = 0; i < S; ++i) c0 += sk[i] > key ? 1 : 0;
    }
    const bool keep = j < S && c0 + c1 + c2 + c3 < beam;
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = kept + __popc(kb & lt);
      nxt[pos] = cand_node(cur, b, sr[j]);
      if (leaf) leaf_sc[pos] = key_score(key);
    }
    kept += __popc(kb);
  }
  return beam;
}

// select_lanes with the fewest registers for C.  Each width is compiled as a function of its
// own: inlined side by side into one body they share a register allocation and run about
// three times slower.
template <int R>
__device__ __noinline__ int select_lanes_fn(const unsigned long long* keys, int C, int beam, const int* cur, int b,
                                            int* nxt, float* leaf_sc, bool leaf, unsigned long long* sk, int* sr,
                                            uint32_t* hw) {
  return select_lanes<R>(keys, C, beam, cur, b, nxt, leaf_sc, leaf, sk, sr, hw);
}
__device__ __forceinline__ int select_one_warp(const unsigned long long* keys, int C, int beam, const int* cur, int b,
                                               int* nxt, float* leaf_sc, bool leaf, unsigned long long* sk, int* sr,
                                               uint32_t* hw) {
  if (C <= 64) return select_lanes_fn<2>(keys, C, beam, cur, b, nxt, leaf_sc, leaf, sk, sr, hw);
  if (C <= 128) return select_lanes_fn<4>(keys, C, beam, cur, b, nxt, leaf_sc, leaf, sk, sr, hw);
  if (C <= 256) return select_lanes_fn<8>(keys, C, beam, cur, b, nxt, leaf_sc, leaf, sk, sr, hw);
  return select_lanes_fn<16>(keys, C, beam, cur, b, nxt, leaf_sc, leaf, sk, sr, hw);
}

// A query whose path copies did not arrive: no leaves, NaN scores and output.
template <bool ATTEND, int D>
__device__ __forceinline__ void group_poison(const RouteArgs& a, long long qg, int tid, int nt) {
  for (int k = tid; k < a.beam; k += nt) {
    if (a.leaf_idx) a.leaf_idx[qg * a.beam + k] = -1;
    if (a.leaf_score) a.leaf_score[qg * a.beam + k] = __int_as_float(0x7fc00000);
  }
  if (ATTEND && a.O != nullptr)
    for (int e = tid; e < D; e += nt) {
      if (a.o_bf16) static_cast<uint16_t*>(a.O)[qg * D + e] = 0x7FC0u;
      else static_cast<float*>(a.O)[qg * D + e] = __int_as_float(0x7fc00000);
    }
}

// Query qg = blockIdx.x.  TS: summary storage; TKV: K/V storage (NoKV: route only).
template <int D, typename TS, typename TKV, int NW, bool APPEND>
__global__ void __launch_bounds__(NW * 32, 16 / NW) route_group_kernel(const RouteArgs a) {
  constexpr bool ATTEND = !std::is_same<TKV, NoKV>::value;
  static_assert(!APPEND || ATTEND, "the path reads K rows of type TKV");
  constexpr int NT = NW * 32;
  constexpr int EPC = 16 / (int)sizeof(TS);       // summary elements per 16-byte chunk
  constexpr int CPL = D * (int)sizeof(TS) / 128;  // 16-byte chunks of a row per lane (8 lanes a row)
  constexpr int P = 16 / CPL;                     // row passes per round: 16 loads in flight per lane
  static_assert(P % 4 == 0 && 16 % P == 0, "passes go four at a time through the butterfly");
  extern __shared__ __align__(128) unsigned char gsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qg = blockIdx.x;  // grid = the call's queries (< 2^31)
  PathSmem Ps{};
  size_t path_bytes = 0;
  if constexpr (APPEND) {
    Ps = path_smem_layout(D, D * (int)sizeof(TKV), (int)sizeof(TS), (int)a.lb, a.b, a.L);
    path_bytes = Ps.total;
  }
  const GroupSmem Ls = group_smem_layout(D, a.cmax, a.beam, NW, path_bytes);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(gsm + Ls.keys);
  unsigned long long* sk = reinterpret_cast<unsigned long long*>(gsm + Ls.sk);
  int* sr = reinterpret_cast<int*>(gsm + Ls.sr);
  uint32_t* hw = reinterpret_cast<uint32_t*>(gsm + Ls.hw);
  int* surv_a = reinterpret_cast<int*>(gsm + Ls.surv_a);
  int* surv_b = reinterpret_cast<int*>(gsm + Ls.surv_b);
  float* leaf_sc = reinterpret_cast<float*>(gsm + Ls.leaf_sc);
  unsigned char* pb = gsm + Ls.path;
  uint64_t* pbar = reinterpret_cast<uint64_t*>(pb + Ps.bar);
  pdl_wait();
  pdl_release();

  const int hq_flat = qg / a.nq;
  const int h = hq_flat % a.q_heads;
  const long long unit = (long long)(hq_flat / a.q_heads) * a.kv_heads + h / a.group;
  const TS* pyr_u = static_cast<const TS*>(a.pyr) + unit * a.pyr_unit_stride;
  if constexpr (APPEND) {
    if (tid == 0) {  // the path's copies first: they are the longest wait
      mbar_init(pbar, 1);
      fence_mbar_init();
      path_issue<TKV, TS, D>(Ps, pb, a.K + unit * a.kv_unit_stride, pyr_u, a.off, a.n, a.b, a.L, a.path_leaf,
                             a.path_tokens, a.lb, pbar, a.path_node);
    }
  }
  const int l8 = lane & 7, rg = lane >> 3;
  float qv[CPL][EPC];
#pragma unroll
  for (int j = 0; j < CPL; ++j)
#pragma unroll
    for (int e = 0; e < EPC; ++e) qv[j][e] = load_elem(a.Q, a.q_bf16 != 0, (long long)qg * D + EPC * (l8 + 8 * j) + e);
  // Levels with at most `beam` nodes below the root are kept whole (as in the other kernels):
  // the first scored level's candidates are all its nodes.
  const int l_first = a.l_first;
  if (a.trace)
    for (int l = l_first + 1; l < a.L; ++l) {
      int* tr = a.trace + ((long long)qg * a.L + (a.L - 1 - l)) * a.beam;
      for (int k = tid; k < a.beam; k += NT) tr[k] = k < a.n[l] ? k : -1;
    }

  const int* cur = nullptr;  // survivors of the level above (null: every node)
  int* nxt = surv_a;
  int m = 0;
  for (int l = l_first; l >= 0; --l) {
    const bool first = l == l_first;
    int C = (int)a.n[l];
    if (!first) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, a.n[l] - (long long)a.b * last);
    }
    const TS* S = pyr_u + a.off[l] * D;
    // The path node's row: recomputed (below the first level, where the path is ready);
    // the first level is scored from the stored rows while the path is computed, and its
    // path node rescored afterwards.
    const int pn = (APPEND && !first) ? (int)a.path_node[l] : -1;
    const uint4* pf = APPEND ? reinterpret_cast<const uint4*>(pb + Ps.pf + (size_t)l * D * sizeof(TS)) : nullptr;
    for (int R0 = 0; R0 < C; R0 += 4 * P * NW) {  // rows R0 + 4 (p NW + warp) + rg
      uint4 v[P][CPL];
      int nd[P];
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int r = R0 + 4 * (p * NW + warp) + rg;
        nd[p] = -1;
        if (r < C) {
          const int node = cand_node(cur, a.b, r);
          nd[p] = node;
          if (APPEND && node == pn) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) v[p][j] = pf[l8 + 8 * j];
          } else {
            const uint4* row = reinterpret_cast<const uint4*>(S + (size_t)node * D);
#pragma unroll
            for (int j = 0; j < CPL; ++j) v[p][j] = ldg16(row + l8 + 8 * j);
          }
        } else {
#pragma unroll
          for (int j = 0; j < CPL; ++j) v[p][j] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // Four passes at a time: each lane forms its partial of each pass's row, and one
      // transposed butterfly over the eight lanes of a row (distances 4, 2, 1) sums all
      // four rows with four shuffles, associating as score_reduce8 does: lane l8 ends with
      // the sum of pass l8 / 2.
#pragma unroll
      for (int p4 = 0; p4 < P; p4 += 4) {
        float part[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < CPL; ++j) {
            float f[EPC];
            Vec16<TS>::to_f32(v[p4 + u][j], f);
#pragma unroll
            for (int e = 0; e < EPC; e += 4) score_fma(qv[j] + e, f + e, acc0, acc1);
          }
          part[u] = (acc0.x + acc0.y) + (acc1.x + acc1.y);
        }
        const bool hi4 = (l8 & 4) != 0, hi2 = (l8 & 2) != 0;
        const float send0 = hi4 ? part[0] : part[2], send1 = hi4 ? part[1] : part[3];
        const float keep0 = hi4 ? part[2] : part[0], keep1 = hi4 ? part[3] : part[1];
        const float b0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 4);
        const float b1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 4);
        float sc = (hi2 ? b1 : b0) + __shfl_xor_sync(0xffffffffu, hi2 ? b0 : b1, 2);
        sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        // lane l8 holds pass p4 + l8 / 2; its node id is in nd of that pass (same lane group)
        int node = nd[p4];
#pragma unroll
        for (int u = 1; u < 4; ++u)
          if ((l8 >> 1) == u) node = nd[p4 + u];
        const int r = R0 + 4 * ((p4 + (l8 >> 1)) * NW + warp) + rg;
        if ((l8 & 1) == 0 && r < C) keys[r] = route_key(sc, node);
      }
    }
    bool synced = false;
    if constexpr (APPEND) {
      if (first) {
        // the path: its copies were issued first; one thread waits, the CTA computes the rows
        const bool pok = tid != 0 || mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, a.first_wait);
        if (__syncthreads_or(!pok)) {
          if (tid == 0) mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, kRouteWaitCycles);  // let the copies land
          group_poison<ATTEND, D>(a, qg, tid, NT);
          return;
        }
        // the unit's first query stores the path
        const bool writer = (qg % a.nq) == 0 && ((qg / a.nq) % a.q_heads) % a.group == 0;
        path_compute<TKV, TS, D>(Ps, pb, const_cast<TS*>(pyr_u), a.off, a.n, a.b, a.L, a.path_tokens, writer, tid,
                                 NT, []() { __syncthreads(); });
        synced = true;
      }
    }
    if (!synced) __syncthreads();  // every key of the level
    if (warp == 0) {
      if (APPEND && first) {  // rescore the path node from its recomputed row (8 lanes, the shared order)
        const int pn0 = (int)a.path_node[l];
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          float f[EPC];
          Vec16<TS>::to_f32(pf[l8 + 8 * j], f);
#pragma unroll
          for (int e = 0; e < EPC; e += 4) score_fma(qv[j] + e, f + e, acc0, acc1);
        }
        const float sc = score_reduce8(acc0, acc1);
        if (lane == 0) keys[pn0] = route_key(sc, pn0);
        __syncwarp();
      }
      const int kept = select_one_warp(keys, C, a.beam, cur, a.b, nxt, leaf_sc, l == 0, sk, sr, hw);
      __syncwarp();
      if (a.trace) {
        int* tr = a.trace + ((long long)qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    }
    __syncthreads();  // the survivors
    m = min(C, a.beam);
    cur = nxt;
    nxt = nxt == surv_a ? surv_b : surv_a;
  }
  if (a.leaf_idx)
    for (int k = tid; k < a.beam; k += NT) a.leaf_idx[(long long)qg * a.beam + k] = k < m ? cur[k] : -1;
  if (a.leaf_score)
    for (int k = tid; k < a.beam; k += NT)
      a.leaf_score[(long long)qg * a.beam + k] = k < m ? leaf_sc[k] : __int_as_float(0x7fc00000);
  if constexpr (ATTEND) {
    if (a.O == nullptr) return;
    using A = RegAttn<TKV, D>;
    constexpr int PP = 8;
    float* am = reinterpret_cast<float*>(gsm + Ls.am);
    float* al = reinterpret_cast<float*>(gsm + Ls.al);
    float* aw = reinterpret_cast<float*>(gsm + Ls.aw);
    float* aacc = reinterpret_cast<float*>(gsm + Ls.aacc);
    float qc[A::VEC];
    reg_attn_load_q<TKV, D>(a.Q, a.q_bf16 != 0, qg, lane, qc);
    const int total = leaf_token_count(cur, m, a.lb, a.N);
    float m_w = -INFINITY, l_w = 0.f;
    float acc[A::VEC];
#pragma unroll
    for (int e = 0; e < A::VEC; ++e) acc[e] = 0.f;
    reg_attn_tokens<TKV, D, PP>(cur, total, a.lb, a.K + unit * a.kv_unit_stride, a.V + unit * a.kv_unit_stride, qc,
                                a.qk_scale, warp, NW, lane, m_w, l_w, acc);
    reg_attn_fold<TKV, D>(l_w, acc);
    if (lane == 0) {
      am[warp] = m_w;
      al[warp] = l_w;
    }
    if (lane < A::LPT)
#pragma unroll
      for (int e = 0; e < A::VEC; ++e) aacc[warp * D + lane * A::VEC + e] = acc[e];
    __syncthreads();
    // merge the warps' states: weight 2^(m_w - M) on each warp's sum and output row
    if (warp == 0) {
      const float mw = lane < NW ? am[lane] : -INFINITY;
      float M = mw;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float w = mw == -INFINITY ? 0.f : exp2f(mw - M);
      float L = lane < NW ? al[lane] * w : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
      if (lane < NW) aw[lane] = w;
      if (lane == 0) aw[NW] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < D; e += NT) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) o += aacc[w * D + e] * aw[w];
      const float val[1] = {o};
      store_out(a.O, a.o_bf16 != 0, qg, D, e, val, aw[NW]);
    }
  }
}

template <int D, typename TS, typename TKV, int NW, bool APPEND>
cudaError_t run_group(const RouteArgs& a, size_t smem, cudaStream_t s) {
  auto kern = route_group_kernel<D, TS, TKV, NW, APPEND>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)a.total_queries), dim3(NW * 32), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TS, typename TKV, bool APPEND>
cudaError_t run_group_nw(int D, int nw, const RouteArgs& a, size_t smem, cudaStream_t s) {
  if (nw == 16)
    return D == 128 ? run_group<128, TS, TKV, 16, APPEND>(a, smem, s) : run_group<64, TS, TKV, 16, APPEND>(a, smem, s);
  return D == 128 ? run_group<128, TS, TKV, 8, APPEND>(a, smem, s) : run_group<64, TS, TKV, 8, APPEND>(a, smem, s);
}

// Every shape of one K/V type: head_dim 64 or 128, 8 or 16 warps, summaries fp32 or bf16,
// with or without the append path (which needs a K type).
template <typename TKV>
cudaError_t run_group_kv(int D, bool s16, int nw, bool append, const RouteArgs& a, size_t smem, cudaStream_t s) {
  if constexpr (std::is_same<TKV, NoKV>::value) {
    if (append) return cudaErrorInvalidValue;
    return s16 ? run_group_nw<uint16_t, TKV, false>(D, nw, a, smem, s)
               : run_group_nw<float, TKV, false>(D, nw, a, smem, s);
  } else {
    if (append)
      return s16 ? run_group_nw<uint16_t, TKV, true>(D, nw, a, smem, s)
                 : run_group_nw<float, TKV, true>(D, nw, a, smem, s);
    return s16 ? run_group_nw<uint16_t, TKV, false>(D, nw, a, smem, s)
               : run_group_nw<float, TKV, false>(D, nw, a, smem, s);
  }
}

}  // namespace zha

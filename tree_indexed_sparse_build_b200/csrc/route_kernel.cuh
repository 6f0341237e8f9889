// The staged route kernel (route_tma_kernel) and its launch helpers.  Its instantiations
// are spread over route_tma_{nokv,bf16,f32}{,_s16}.cu (one per KV type and summary type),
// which compile in parallel; route.cu plans the launches and calls them through
// route_tma_launch_* (route_common.cuh).
#pragma once

#include <algorithm>
#include <type_traits>

#include "attn_core.cuh"
#include "decode_append.cuh"
#include "decode_attn.cuh"
#include "device_common.cuh"
#include "route_common.cuh"
#include "zha_internal.h"

namespace zha {

// Staged routing.  qpc queries per CTA, wpq warps per query (blockDim.x = 32 qpc wpq).
// GROUPED (wpq > 1): the warps of query qi synchronise on named barrier 1 + qi; otherwise
// each query is one warp, synchronised only within the warp.
//
// With TKV = the KV storage type (not NoKV) the kernel is the fused decode: once the
// last level is selected, the query's warps attend over the tokens of its leaves.  The
// candidate-row region, free after the leaf-level scoring, becomes two or three K/V stage
// buffers filled by one bulk copy per leaf piece (K and V) on their "full" mbarriers and
// refilled as the warps release them (decode_attn.cuh); the warps run the online softmax
// of attn_core.cuh over each stage, merge their states through shared memory and write O.
// No leaf list goes through global memory and nothing is launched between the route and
// the attention.  With buf_tokens the attention also covers the append buffer's tokens.
// NARROW instantiations are built for CTAs of at most 8 warps, three per SM (register cap).
// PATH (decode_append.cuh; needs TKV, the type of the K rows the path reads):
//  kPathAppend (fused decode, one query per CTA) -- the kernel first extends the tree by
//    the tokens appended to one leaf, and stores the path (one CTA per unit);
//  kPathPrefix (causal routing, append-buffer decode) -- query qg routes over the tree of
//    tokens 0 .. p, p = positions[qg % nq] (or prefix_pos): its own depth and node counts,
//    and its prefix's right edge recomputed into shared memory (never stored).
// With a KV type, the query then attends over its leaves unless O is null.
// TS: the summaries' storage (float, or bf16 bits in uint16_t); rows are staged as stored
// and widened to fp32 as they are scored.
// A query whose copies did not arrive (a bounded wait ran out, the error word is set): no
// leaves, NaN scores and output, so the loss shows in the results as well.  Called by one warp.
template <bool ATTEND, int D>
__device__ __forceinline__ void route_poison(const RouteArgs& a, long long qg, int lane) {
  for (int k = lane; k < a.beam; k += 32) {
    if (a.leaf_idx) a.leaf_idx[qg * a.beam + k] = -1;
    if (a.leaf_score) a.leaf_score[qg * a.beam + k] = __int_as_float(0x7fc00000);
  }
  if (ATTEND && a.O != nullptr)
    for (int e = lane; e < D; e += 32) {
      if (a.o_bf16) static_cast<uint16_t*>(a.O)[qg * D + e] = 0x7FC0u;
      else static_cast<float*>(a.O)[qg * D + e] = __int_as_float(0x7fc00000);
    }
}

template <int D, bool GROUPED, typename TKV, bool NARROW, int PATH, typename TS>
__global__ void __launch_bounds__(NARROW ? 256 : kRouteMaxWarps * 32, NARROW ? 3 : 1)
    route_tma_kernel(const RouteArgs a) {
  constexpr bool ATTEND = !std::is_same<TKV, NoKV>::value;
  constexpr bool APPEND = PATH == kPathAppend;
  constexpr bool PREFIX = PATH == kPathPrefix;
  constexpr bool HASPATH = PATH != kPathNone;
  static_assert(!HASPATH || ATTEND, "the path reads K rows of type TKV");
  constexpr int EPC = 16 / (int)sizeof(TS);       // summary elements per 16-byte chunk
  constexpr int CPL = D * (int)sizeof(TS) / 128;  // 16-byte chunks of a row per lane (8 lanes per row)
  constexpr uint32_t SROW = D * (uint32_t)sizeof(TS);  // bytes of a summary row
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
  const TS* rows = reinterpret_cast<const TS*>(base + Ls.rows);
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
  const TS* pyr_u = static_cast<const TS*>(a.pyr) + unit * a.pyr_unit_stride;
  // the path region (fused append or causal prefix)
  unsigned char* pb = base + a.path_smem_off;
  PathSmem Ps{};
  if (HASPATH) Ps = path_smem_layout(D, D * (int)sizeof(TKV), (int)sizeof(TS), (int)a.lb, a.b, a.L);
  uint64_t* pbar = reinterpret_cast<uint64_t*>(pb + Ps.bar);
  // this query's tree: the whole tree, or (PREFIX) the tree of its prefix
  long long Nq = a.N;
  bool live = valid;  // a query with a position outside the tree routes nowhere
  if constexpr (PREFIX) {
    const long long pos = !valid ? 0 : a.positions ? a.positions[qg % a.nq] : a.prefix_pos;
    if (valid && (pos < 0 || pos >= a.N)) {
      if (wq == 0 && lane == 0) atomicOr(a.err, kDevErrBadLeaf);
      live = false;
    }
    Nq = live ? pos + 1 : 1;
    if (wq == 0 && lane == 0) {
      long long* qn = reinterpret_cast<long long*>(pb + Ps.qn);
      qn[0] = (Nq + a.lb - 1) / a.lb;
      int L = 0;
      do {  // L = smallest L >= 1 with b^L >= n0
        qn[L + 1] = (qn[L] + a.b - 1) / a.b;
        ++L;
      } while (qn[L] > 1);
      qn[kMaxLevels - 1] = L;
    }
    qsync();
  }
  const long long* nl = PREFIX ? reinterpret_cast<const long long*>(pb + Ps.qn) : a.n;
  const int Lq = PREFIX ? (int)nl[kMaxLevels - 1] : a.L;
  // A level with at most `beam` nodes is kept whole once every node above it is: starting
  // from the root, such levels need no scoring, and routing begins at the highest level
  // l_first >= 1 with more than `beam` nodes (else at the leaves), from every node of the
  // level above it.  The leaves are always scored (their scores are an output).
  int l_first = Lq - 1;
  while (l_first >= 1 && nl[l_first] <= a.beam) --l_first;
  const int m_first = (int)nl[l_first + 1];
  if (wq == 0 && lane == 0) {
    mbar_init(&bar[0], 1);
    if (ATTEND)
      for (int i = 0; i < a.attn_nbuf; ++i) {
        if (i > 0) mbar_init(&bar[i], 1);  // "full" (bar[0] serves the route first)
        mbar_init(&bar[3 + i], nw);        // "empty": one arrival per warp
      }
    if (HASPATH) mbar_init(pbar, 1);
    fence_mbar_init();
    if constexpr (HASPATH) {
      if (live) {
        fence_proxy_async_smem();
        const long long leaf = APPEND ? a.path_leaf : (Nq - 1) / a.lb;
        const int ntok = APPEND ? a.path_tokens : (int)(Nq - leaf * a.lb);
        path_issue<TKV, TS, D>(Ps, pb, a.K + unit * a.kv_unit_stride, pyr_u, a.off, nl, a.b, Lq, leaf,
                           ntok, a.lb, pbar);
      }
    }
  }
  if (wq == 0) {
    for (int k = lane; k < m_first; k += 32) surv_a[k] = k;  // every node of level l_first + 1
    if (a.trace && valid)
      for (int l = l_first + 1; l < Lq; ++l) {  // the levels kept whole: all their nodes
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = (live && k < nl[l]) ? k : -1;
      }
  }
  qsync();

  // Eight lanes per row, in the scoring order of score_fma / score_reduce8 (route_common.cuh):
  // lane (rg = lane / 8, l8 = lane % 8) reads chunks l8 + 8 j, so each row of a shared-memory
  // phase is one 128-byte run.
  const int l8 = lane & 7, rg = lane >> 3;
  float qv[CPL][EPC];
  int* cur = surv_a;
  int* nxt = surv_b;
  int m = live ? m_first : 0;
  uint32_t parity = 0;
  for (int l = l_first; l >= 0; --l) {
    int C = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, nl[l] - (long long)a.b * last);
    }
    const TS* S = pyr_u + a.off[l] * D;
    if (wq == 0 && C > 0) {
      // one bulk copy per survivor (its children are consecutive rows) + candidate ids
      if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)C * SROW);
      __syncwarp();
      fence_proxy_async_smem();
      for (int j = lane; j < m; j += 32) {
        const long long node0 = (long long)a.b * cur[j];
        const int nc = (int)min((long long)a.b, nl[l] - node0);
        bulk_copy_g2s((void*)(rows + (size_t)j * a.b * D), S + node0 * D, (uint32_t)nc * SROW, bar);
      }
      for (int j = lane; j < m; j += 32) {  // survivor j's children are candidates j b ..
        const int node0 = a.b * cur[j];
        const int nc = min(a.b, C - j * a.b);
        for (int i = 0; i < nc; ++i) cand[j * a.b + i] = node0 + i;
      }
    }
    if (HASPATH && wq == 0) {
      // candidate slot of the path node at this level: its parent is a survivor j, and the
      // parent's children are candidates j b .. j b + b - 1
      const long long* node = reinterpret_cast<const long long*>(pb + Ps.node);
      int* kpos = reinterpret_cast<int*>(pb + Ps.kpos);
      int found = -1;
      for (int j0 = 0; j0 < m; j0 += 32) {
        const int j = j0 + lane;
        const unsigned hit = __ballot_sync(0xffffffffu, j < m && live && cur[j] == node[l + 1]);
        if (hit && found < 0) found = j0 + __ffs(hit) - 1;
      }
      if (lane == 0) kpos[0] = found < 0 ? -1 : (int)(found * a.b + (node[l] - a.b * node[l + 1]));
    }
    if (l == l_first && valid) {  // load q while the first level is in flight
      const long long qo = qg * D;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = l8 + 8 * j;
#pragma unroll
        for (int e = 0; e < EPC; ++e)
          qv[j][e] = a.q_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[qo + EPC * c + e])
                              : static_cast<const float*>(a.Q)[qo + EPC * c + e];
      }
    }
    if (HASPATH && l == l_first) {
      // the path rows, while the first level's copies are in flight
      const bool pok = !live || mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, a.first_wait);
      const bool pfail = GROUPED ? group_any(bar_id, bar_n, !pok) : __any_sync(0xffffffffu, !pok);
      if (pfail) {
        if (wq == 0 && lane == 0) {  // let all copies land before the CTA exits
          if (live) mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, kRouteWaitCycles);
          if (C > 0) mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, kRouteWaitCycles);
        }
        if (wq == 0 && valid) route_poison<ATTEND, D>(a, qg, lane);
        return;
      }
      // every thread has seen the path's copies land: the path barrier's life ends here, as
      // its memory may later hold the attention's stages
      if (wq == 0 && lane == 0) mbar_inval(pbar);
      if constexpr (HASPATH) {
        if (live) {
          // fused append: the first query of each unit stores the path
          const bool writer = APPEND && (qg % a.nq) == 0 && ((qg / a.nq) % a.q_heads) % a.group == 0;
          const int ntok = APPEND ? a.path_tokens : (int)(Nq - ((Nq - 1) / a.lb) * a.lb);
          path_compute<TKV, TS, D>(Ps, pb, const_cast<TS*>(pyr_u), a.off, nl, a.b, Lq, ntok, writer,
                               32 * wq + lane, bar_n, qsync);
        }
      }
    }
    const bool ok = C == 0 || mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, a.first_wait);
    const bool failed = GROUPED ? group_any(bar_id, bar_n, !ok) : __any_sync(0xffffffffu, !ok);
    if (failed) {
      if (wq == 0 && lane == 0 && C > 0)  // let the copies land before the CTA exits
        mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, kRouteWaitCycles);
      if (wq == 0 && valid) route_poison<ATTEND, D>(a, qg, lane);
      return;  // the whole group leaves together
    }
    if (!GROUPED) __syncwarp();  // candidate ids written by other lanes
    if (C > 0) parity ^= 1u;
    if (HASPATH) {
      // the staged row of the path node may predate the append, or (prefix) cover tokens
      // past the query's prefix: use the recomputed one
      const int k = *reinterpret_cast<const int*>(pb + Ps.kpos);
      if (k >= 0) {
        const TS* pf = reinterpret_cast<const TS*>(pb + Ps.pf) + (size_t)l * D;
        TS* dst = const_cast<TS*>(rows) + (size_t)k * D;
        for (int e = 32 * wq + lane; e < D; e += bar_n) dst[e] = pf[e];
        qsync();
      }
    }

    // score: rows r0 + 4 nw u + rg (u = 0 .. 3) per iteration, r0 = 4 (wq + 4 nw t).  Each
    // lane forms its partial of the four rows, and one transposed butterfly over the eight
    // lanes of a row (distances 4, 2, 1) sums all four with four shuffles, associating
    // exactly as score_reduce8 does: lane l8 ends with the sum of row u = l8 / 2.
    for (int r0 = 4 * wq; r0 < C; r0 += 16 * nw) {
      float part[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + 4 * nw * u + rg;
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        if (r < C) {
          const uint4* row = reinterpret_cast<const uint4*>(rows + (size_t)r * D);
#pragma unroll
          for (int j = 0; j < CPL; ++j) {
            float v[EPC];
            Vec16<TS>::to_f32(row[l8 + 8 * j], v);
#pragma unroll
            for (int e = 0; e < EPC; e += 4) score_fma(qv[j] + e, v + e, acc0, acc1);
          }
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
      const int r = r0 + 4 * nw * (l8 >> 1) + rg;
      if ((l8 & 1) == 0 && r < C) keys[r] = route_key(sc, cand[r]);
    }
    qsync();
    // C is the same for the whole group.  Up to 64 candidates: one warp's register selection
    // (no shared-memory ranks, no group barriers inside); up to 128: ranks over the group;
    // wider: the group's radix selection, or one warp's register selection.
    if (C > 64 && C <= 128 && C <= 64 * nw) {
      const int kept =
          select_rank_group(keys, cand, C, a.beam, nxt, leaf_sc, l == 0, red, wq, lane, nw, bar_id);
      qsync();
      if (wq == 0 && a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    } else if (GROUPED && C > 64 && C <= 32 * nw) {  // radix selection over the group
      const int kept = select_radix_group(keys, cand, C, a.beam, nxt, leaf_sc, l == 0, red,
                                          reinterpret_cast<unsigned*>(base + Ls.hist), wq, lane, nw, bar_id);
      group_sync(bar_id, bar_n);
      if (wq == 0 && a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    } else if (wq == 0 && C > 0) {
      const int kept = select_warp(keys, cand, C, a.beam, lane, nxt, leaf_sc, l == 0);
      __syncwarp();
      if (a.trace && valid) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
    }
    m = min(C, a.beam);
    // This level's generic shared-memory writes (the path's rows and values, the patched
    // candidate row) lie where bulk copies land next: the next level's rows, or the
    // attention's stages.  Each thread orders its own writes before those copies (a proxy
    // fence by the writing thread, then the barrier the copies follow).
    fence_proxy_async_smem();
    qsync();
    int* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  if (PREFIX && valid && wq == 0 && a.trace)  // levels above this query's tree
    for (int l = Lq; l < a.L; ++l) {
      int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
      for (int k = lane; k < a.beam; k += 32) tr[k] = -1;
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
    if (a.O == nullptr) return;  // route only (the path needed the K type)
    using S = AttnShape<TKV, D>;
    StagedAttn sa;
    sa.leaves = cur;
    sa.m = m;
    sa.buf_leaf0 = a.buf_leaf0;
    sa.lb = (int)a.lb;
    sa.total = leaf_tokens(cur, m, a.lb, Nq) + (live ? a.buf_tokens : 0);
    sa.TS = a.stage_tokens;
    sa.nbuf = a.attn_nbuf;
    sa.sb = base + Ls.rows;  // the candidate rows (and the append path) are no longer needed
    sa.bars = bar;
    sa.empty = bar + 3;
    sa.ph0 = parity;  // bar[0] carries on from the route's level copies
    sa.Ku = a.K + unit * a.kv_unit_stride;
    sa.Vu = a.V + unit * a.kv_unit_stride;
    sa.qk_scale = a.qk_scale;
    sa.O = a.O;
    sa.o_bf16 = a.o_bf16;
    sa.err = a.err;
    sa.wait_cycles = a.first_wait;
    sa.drain_cycles = kRouteWaitCycles;
    const int nst = (sa.total + sa.TS - 1) / sa.TS;
    if (wq == 0)
      for (int st = 0; st < min(nst, sa.nbuf); ++st)
        attn_issue_stage<S::ROWB>(cur, m, sa.buf_leaf0, sa.lb, sa.total, sa.TS, st, sa.nbuf, sa.sb, sa.Ku, sa.Vu,
                                  bar, lane);
    float qa[S::CPL][S::VEC];
    if (valid) attn_load_q<TKV, D>(a.Q, a.q_bf16 != 0, qg, lane, qa);
    float* pw = reinterpret_cast<float*>(base + Ls.pw) + wq * 16;
    attend_staged<TKV, D>(sa, qg, valid, qa, pw, reinterpret_cast<float*>(red), wq, nw, lane, bar_id);
  }
}

template <int D, bool GROUPED, typename TKV, bool NARROW, int PATH, typename TS>
cudaError_t run_route_tma(const RouteArgs& a, unsigned blocks, int threads, size_t smem,
                          cudaStream_t s) {
  auto kern = route_tma_kernel<D, GROUPED, TKV, NARROW, PATH, TS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TKV, int PATH, typename TS>
cudaError_t run_shape(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks, int threads,
                      size_t smem, cudaStream_t s) {
  if constexpr (PATH != kPathAppend) {  // the fused append runs in wide launches only
    if (narrow) {
      if (grouped)
        return D == 128 ? run_route_tma<128, true, TKV, true, PATH, TS>(a, blocks, threads, smem, s)
                        : run_route_tma<64, true, TKV, true, PATH, TS>(a, blocks, threads, smem, s);
      return D == 128 ? run_route_tma<128, false, TKV, true, PATH, TS>(a, blocks, threads, smem, s)
                      : run_route_tma<64, false, TKV, true, PATH, TS>(a, blocks, threads, smem, s);
    }
  } else if (narrow) {
    return cudaErrorNotSupported;
  }
  if (grouped)
    return D == 128 ? run_route_tma<128, true, TKV, false, PATH, TS>(a, blocks, threads, smem, s)
                    : run_route_tma<64, true, TKV, false, PATH, TS>(a, blocks, threads, smem, s);
  return D == 128 ? run_route_tma<128, false, TKV, false, PATH, TS>(a, blocks, threads, smem, s)
                  : run_route_tma<64, false, TKV, false, PATH, TS>(a, blocks, threads, smem, s);
}

template <typename TKV, typename TS>
cudaError_t run_route_tma_d_impl(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks,
                                 int threads, size_t smem, cudaStream_t s, int path = kPathNone) {
  if constexpr (!std::is_same<TKV, NoKV>::value) {
    if (path == kPathAppend)
      return run_shape<TKV, kPathAppend, TS>(D, grouped, narrow, a, blocks, threads, smem, s);
    if (path == kPathPrefix)
      return run_shape<TKV, kPathPrefix, TS>(D, grouped, narrow, a, blocks, threads, smem, s);
  }
  return run_shape<TKV, kPathNone, TS>(D, grouped, narrow, a, blocks, threads, smem, s);
}

}  // namespace zha

// Top-down beam routing ("Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", abstract: future queries traverse the tree of key summaries from the top
// down to retrieve a sparse subset of keys).
//
// Survivors start as {root}.  For l = L-1 .. 0 every existing child c of a survivor is
// scored by q . S_l[c] in fp32, and the top-min(beam, #candidates) are kept, ordered by
// score descending with the lower node index first on equal scores.  Levels with at most
// beam nodes below the root are kept whole without scoring (the route starts at the
// highest level with more than beam nodes, from every node of the level above it).
//
// GPU mapping.  A candidate's key packs (order-preserving score bits, inverted node
// index) into 64 bits, so "greater key" is exactly "ranks first".  Candidates are the
// children of the survivors in ascending node order (survivors ascend, the children of
// a node are contiguous rows), so candidate k belongs to survivor k / b.
//
// Kernels, by how many queries a call carries per SM:
//  - at most two (route_group.cuh, route_group_kernel): one CTA of 8 or 16 warps per query;
//    every level's candidate rows are loaded straight into registers by all the warps (one
//    memory round trip for up to 64 NW candidates), the keys are gathered in shared memory
//    and one warp selects; the attention splits the leaves' tokens over the warps and
//    merges their softmax states; the one-leaf append of a decode step rides along.
//  - more (route_warp.cu, route_warp_kernel): one warp per query, rows into registers, up
//    to sixteen queries in flight per SM.
//  - the causal and buffered calls, and shapes the two above do not take
//    (route_kernel.cuh, route_tma_kernel): each level's rows staged in shared memory by one
//    1-D bulk copy (non-multicast TMA) per survivor, scored by the query's warps.
// Every kernel scores in one shared order (eight lanes per row, route_common.cuh), so
// scores, survivors and leaves are bit-identical across them.  Selections: exact top-B by
// thresholds, ranks and ballots (route_common.cuh, route_group.cuh).
//
// Fallback kernel (route_reg_kernel) for levels too wide to stage in shared memory:
// the same selection, with candidate rows loaded into registers in batches.
//
// Summaries are stored in fp32 or bf16 (the tree's summary type, TS in the kernels); rows
// are read as stored and widened to fp32 for scoring.
//
// Files: route_tma_kernel and its launch helpers are in route_kernel.cuh, instantiated per
// KV type and summary type in route_tma_{nokv,bf16,f32}{,_s16}.cu; route_group_kernel in
// route_group.cuh, instantiated per KV type in route_group_{nokv,bf16,f32}.cu;
// route_warp_kernel in route_warp.cu; this file holds the register kernel and the host-side
// plans (launch_route, plan_decode, launch_decode, launch_causal).
#include <algorithm>
#include <type_traits>

#include "attn_core.cuh"
#include "decode_append.cuh"
#include "decode_attn.cuh"
#include "device_common.cuh"
#include "route_common.cuh"
#include "route_group.cuh"
#include "zha_internal.h"

namespace zha {

template <int D, int U, typename TS>
__global__ void __launch_bounds__(kRouteMaxWarps * 32) route_reg_kernel(const RouteArgs a) {
  constexpr int EPC = 16 / (int)sizeof(TS);  // summary elements per 16-byte chunk
  constexpr int NJ = D / (8 * EPC);          // 16-byte chunks per lane per row (8 lanes a row)
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
  float q[NJ * EPC];
  const int l8 = lane & 7, grp = lane >> 3;
  if (valid) {
    const long long hq_flat = qg / a.nq;  // b * q_heads + h
    const int h = (int)(hq_flat % a.q_heads);
    unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
    // This lane's slice of q: chunks c = l8 + 8j, dims EPC c .. EPC c + EPC - 1.
    const long long qo = qg * D;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        const long long dim = qo + (l8 + 8 * j) * EPC + e;
        q[j * EPC + e] = a.q_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[dim])
                                  : static_cast<const float*>(a.Q)[dim];
      }
  }
  if (wq == 0 && lane == 0) {
    surv_a[0] = 0;  // the root
    s_m[qi] = valid ? 1 : 0;
  }
  __syncthreads();

  const TS* pyr_u = static_cast<const TS*>(a.pyr) + unit * a.pyr_unit_stride;
  int* cur = surv_a;
  int* nxt = surv_b;
  for (int l = a.L - 1; l >= 0; --l) {
    const int m = s_m[qi];
    int C = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, a.n[l] - (long long)a.b * last);
    }
    const TS* S = pyr_u + a.off[l] * D;
#pragma unroll 1
    for (int k0 = wq * 4 * U; k0 < C; k0 += a.wpq * 4 * U) {
      uint4 v[U][NJ];
      int node[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + 4 * u + grp;
        node[u] = -1;
        if (k < C) {
          node[u] = a.b * cur[k / a.b] + k % a.b;
          const uint4* row = reinterpret_cast<const uint4*>(S + (long long)node[u] * D);
#pragma unroll
          for (int j = 0; j < NJ; ++j) v[u][j] = __ldg(row + l8 + 8 * j);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        if (node[u] >= 0) {
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            float f[EPC];
            Vec16<TS>::to_f32(v[u][j], f);
#pragma unroll
            for (int e = 0; e < EPC; e += 4) score_fma(q + EPC * j + e, f + e, acc0, acc1);
          }
        }
        const float s = score_reduce8(acc0, acc1);
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

namespace {
template <int D, int U, typename TS>
cudaError_t run_route(const RouteArgs& a, unsigned blocks, int threads, size_t smem,
                      cudaStream_t s) {
  auto kern = route_reg_kernel<D, U, TS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

constexpr size_t kRouteSmemCap = 200 * 1024;  // staged kernel: shared memory per query
constexpr size_t kCtaSmemCap = 227 * 1024;    // dynamic shared memory of one CTA

// The staged kernel's instantiation set for this tree: route only (kv false) or with the
// cache's K/V type, over its summary type.
using RouteLaunch = cudaError_t (*)(int, bool, bool, const RouteArgs&, unsigned, int, size_t, cudaStream_t, int);
RouteLaunch staged_launch(const zha_tree* t, bool kv) {
  const bool s16 = sum_bf16(t);
  if (!kv) return s16 ? route_tma_launch_nokv_s16 : route_tma_launch_nokv;
  if (t->desc.kv_dtype == ZHA_BF16) return s16 ? route_tma_launch_bf16_s16 : route_tma_launch_bf16;
  return s16 ? route_tma_launch_f32_s16 : route_tma_launch_f32;
}

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
  a.head_dim = D;
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
  a.first_wait = first_wait_cycles(t);
  a.l_first = t->L - 1;
  while (a.l_first >= 1 && t->n[a.l_first] <= beam) --a.l_first;
  a.m_first = (int)t->n[a.l_first + 1];
  return a;
}

// Narrow launches: CTAs of at most 8 warps, three resident per SM (the NARROW kernels'
// register cap), in the 228 KB of shared memory an SM holds (1 KB of it reserved per CTA).
// Each level of a route is one memory round trip, so throughput follows the number of
// queries resident per SM: the launch takes the warps per query (4, 2 or 1; at most enough
// that each warp scores about 16 rows of the widest level) and queries per CTA that keep
// the most queries resident, preferring more warps per query, then fewer queries per CTA.
constexpr int kNarrowMaxWpq = 4;
constexpr int kNarrowCtasPerSm = 3;
constexpr size_t kSmSmem = 228 * 1024, kCtaReserved = 1024;
#ifndef ZHA_NARROW_WPQ
#define ZHA_NARROW_WPQ 0  // 0: by the rule above; else a fixed count (1, 2 or 4)
#endif
int narrow_qpc(int wpq, size_t per_query, long long* resident = nullptr) {
  int best = 1;
  long long best_r = -1;
  for (int q = 1; q <= 8 / wpq; ++q) {
    const size_t cta = (size_t)q * per_query;
    if (cta > kCtaSmemCap) break;
    const long long r = (long long)q * std::min<long long>(kNarrowCtasPerSm, kSmSmem / (cta + kCtaReserved));
    if (r > best_r) {
      best_r = r;
      best = q;
    }
  }
  if (resident) *resident = best_r;
  return best;
}
int narrow_wpq(long long cmax, size_t per_query) {
  if (ZHA_NARROW_WPQ > 0) return ZHA_NARROW_WPQ;
  const int want = (int)std::min<long long>(kNarrowMaxWpq, std::max<long long>(1, (cmax + 15) / 16));
  int best = want;
  long long best_r;
  narrow_qpc(want, per_query, &best_r);
  for (int w = want / 2; w >= 1; w /= 2) {
    long long r;
    narrow_qpc(w, per_query, &r);
    if (r > best_r) {
      best_r = r;
      best = w;
    }
  }
  return best;
}

// Launch shape of the staged kernel.  Wide (at most two queries per SM): one query per
// CTA, enough warps for the widest level (and, fused, for the attention tokens).
// Narrow: up to 8 warps per CTA, narrow_wpq warps per query, narrow_qpc queries per CTA
// (per_query sized with the per-warp weight area of kNarrowMaxWpq warps).
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
    a.wpq = narrow_wpq(a.cmax, per_query);
    a.qpc = narrow_qpc(a.wpq, per_query);
    sh.blocks = (unsigned)((a.total_queries + a.qpc - 1) / a.qpc);
    sh.smem = per_query * a.qpc;
  }
  sh.threads = 32 * a.wpq * a.qpc;
  sh.grouped = a.wpq > 1;
  return sh;
}
// CTA-per-query kernel (route_group.cuh): 16 warps when every query has an SM to itself,
// else 8 (two CTAs per SM).  It fits when every candidate of a level has a thread (the
// selection holds one key per thread) and its shared memory (keys, ids, the attention's
// per-warp states and, appending, the path) fits one CTA.
int group_warps(const zha_tree* t, long long queries) { return queries <= t->sms ? 16 : 8; }
size_t group_smem(const zha_tree* t, int cmax, int beam, int nw, bool append) {
  const int D = t->desc.head_dim;
  const int row = D * (t->desc.kv_dtype == ZHA_BF16 ? 2 : 4);
  const size_t path =
      append ? path_smem_layout(D, row, sum_bytes(t), (int)t->desc.leaf_block, t->desc.branching, t->L).total : 0;
  return group_smem_layout(D, cmax, beam, nw, path).total;
}
bool group_fits(const zha_tree* t, int cmax, int beam, int nw, bool append) {
  return cmax <= 32 * nw && group_smem(t, cmax, beam, nw, append) <= kCtaSmemCap;
}
cudaError_t launch_route_group(zha_tree* t, const RouteArgs& a, int nw, bool attend, bool append, cudaStream_t s) {
  const int D = t->desc.head_dim;
  const bool s16 = sum_bf16(t);
  const size_t smem = group_smem(t, a.cmax, a.beam, nw, append);
  if (!attend) return route_group_launch_nokv(D, s16, nw, false, a, smem, s);
  if (t->desc.kv_dtype == ZHA_BF16) return route_group_launch_bf16(D, s16, nw, append, a, smem, s);
  return route_group_launch_f32(D, s16, nw, append, a, smem, s);
}
}  // namespace

cudaError_t launch_route(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads,
                         int nq, int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                         cudaStream_t stream) {
  RouteArgs a = route_args(t, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace);
  const int D = t->desc.head_dim;
  const long long cmax = a.cmax;
  cudaError_t e;

  // Many queries: one warp per query, rows loaded into registers.
  if (a.total_queries > 2LL * t->sms && route_warp_fits(t, a.cmax, beam)) {
    e = launch_route_warp(t, a, false, stream);
    ++t->launches;
    return e;
  }
  // Few queries: one CTA per query, rows loaded into registers by all its warps.
  if (a.total_queries <= 2LL * t->sms) {
    const int nw = group_warps(t, a.total_queries);
    if (group_fits(t, a.cmax, beam, nw, false)) {
      e = launch_route_group(t, a, nw, false, false, stream);
      ++t->launches;
      return e;
    }
  }
  a.rows_bytes = (int)route_rows_bytes(D, a.cmax, sum_bytes(t));
  // Staged kernel when a query's widest level fits in shared memory.
  const size_t per_query = route_smem_layout(D, a.cmax, beam, a.rows_bytes, 0).total;
  if (per_query <= kRouteSmemCap) {
    a.query_smem_bytes = (int)per_query;
    // 8 rows per warp step, two steps in flight
    const StagedShape sh = staged_shape(t, a, per_query, 0);
    e = staged_launch(t, false)(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream, kPathNone);
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
  if (sum_bf16(t))
    e = D == 128 ? run_route<128, kU128, uint16_t>(a, blocks, threads, smem, stream)
                 : run_route<64, kU64, uint16_t>(a, blocks, threads, smem, stream);
  else
    e = D == 128 ? run_route<128, kU128, float>(a, blocks, threads, smem, stream)
                 : run_route<64, kU64, float>(a, blocks, threads, smem, stream);
  ++t->launches;
  return e;
}

// Fused route + attention (one launch).  Wide launches (one query per CTA): the row region
// grows so that the attention streams its leaves through up to three large stages in
// flight together -- up to 192 KB when every CTA has an SM to itself, 96 KB when two share
// one -- and, with an SM to itself, also holds the one-leaf append's path after the route's
// rows (decode_append.cuh).  Narrow launches (several queries per SM): the row region
// stays the route's own, since a larger one would cut the queries resident per SM, and the
// call is fused only when the query's tokens then fit in at most two stages; otherwise
// fused = false and the route and the attention run as two launches.  Stages hold a
// multiple of 16 tokens (the attention's rounds), at least 16.
DecodePlan plan_decode(const zha_tree* t, int q_heads, int nq, int beam, bool allow_warp) {
  DecodePlan p{};
  const int D = t->desc.head_dim;
  const int row = D * (t->desc.kv_dtype == ZHA_BF16 ? 2 : 4);
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  const bool wide = queries <= 2LL * t->sms;
  long long cmax = 1;
  for (int l = 0; l < t->L; ++l)
    cmax = std::max(cmax, std::min(std::min((long long)beam, t->n[l + 1]) * t->desc.branching, t->n[l]));
  const long long tokens = std::min((long long)beam * t->desc.leaf_block, t->N);
  const size_t route_rows = route_rows_bytes(D, (int)cmax, sum_bytes(t));
  if (allow_warp && !wide && route_warp_fits(t, (int)cmax, beam)) {  // one warp per query (route_warp.cu)
    p.warp = true;
    p.fused = true;
    return p;
  }
  if (allow_warp && wide) {  // one CTA per query (route_group.cuh)
    const int nw = group_warps(t, queries);
    if (group_fits(t, (int)cmax, beam, nw, false)) {
      p.group = true;
      p.group_warps = nw;
      p.fused = true;
      p.append_ok = group_fits(t, (int)cmax, beam, nw, true);
      return p;
    }
  }
  if (!wide) {
    p.nbuf = 2;
    p.rows_bytes = std::max(route_rows, (size_t)4 * 16 * row);  // two stages of 16 tokens at least
    p.stage_tokens = (int)(p.rows_bytes / (4 * row)) / 16 * 16;
    p.attn_warps = 1;
    p.smem_per_query = route_smem_layout(D, (int)cmax, beam, p.rows_bytes, kNarrowMaxWpq).total;
    p.fused = p.smem_per_query <= kRouteSmemCap && p.stage_tokens >= 16 && 2LL * p.stage_tokens >= tokens;
    return p;
  }
  const bool own_sm = queries <= t->sms;
  const size_t cap = own_sm ? 192 * 1024 : 96 * 1024;
  size_t rows = std::min((size_t)2 * row * (size_t)tokens, cap);  // all the tokens, if they fit
  rows = std::max(std::max(rows, route_rows), (size_t)4 * 16 * row);
  p.path_bytes = path_smem_layout(D, row, sum_bytes(t), (int)t->desc.leaf_block, t->desc.branching, t->L).total;
  p.path_off = route_align(route_rows, 128);
  if (own_sm) rows = std::max(rows, p.path_off + p.path_bytes);
  p.nbuf = rows >= (size_t)3 * 2 * 16 * row ? 3 : 2;
  p.stage_tokens = (int)(rows / ((size_t)p.nbuf * 2 * row)) / 16 * 16;
  p.rows_bytes = rows;
  p.attn_warps = (int)std::min<long long>(kRouteMaxWarps, (tokens + 31) / 32);
  p.smem_per_query = route_smem_layout(D, (int)cmax, beam, rows, kRouteMaxWarps).total;
  p.fused = p.smem_per_query <= kCtaSmemCap;
  p.append_ok = p.fused && own_sm;
  return p;
}

cudaError_t launch_decode(zha_tree* t, const DecodePlan& p, const void* d_Q, zha_dtype q_dtype,
                          int q_heads, int nq, int beam, const void* d_K, const void* d_V,
                          float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                          void* d_O, zha_dtype o_dtype, cudaStream_t stream, long long append_leaf) {
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
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  if (p.warp) {
    const cudaError_t e = launch_route_warp(t, a, true, stream);
    ++t->launches;
    return e;
  }
  const bool append = append_leaf >= 0;
  if (append) {  // the tree already has its new shape
    a.path_leaf = append_leaf;
    a.path_tokens = (int)(std::min(append_leaf * a.lb + a.lb, t->N) - append_leaf * a.lb);
    a.path_node[0] = append_leaf;
    for (int l = 1; l <= t->L; ++l) a.path_node[l] = a.path_node[l - 1] / t->desc.branching;
  }
  if (p.group) {
    const cudaError_t e = launch_route_group(t, a, p.group_warps, true, append, stream);
    ++t->launches;
    return e;
  }
  a.stage_tokens = p.stage_tokens;
  a.attn_nbuf = p.nbuf;
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  a.query_smem_bytes = (int)p.smem_per_query;  // weight area sized for 16 warps when wide
  StagedShape sh = staged_shape(t, a, p.smem_per_query, p.attn_warps);
  if (append) a.path_smem_off = (long long)p.path_off;  // inside the row region, after the route's rows
  const cudaError_t e = staged_launch(t, true)(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream,
                                               append ? kPathAppend : kPathNone);
  ++t->launches;
  return e;
}

// Causal routing (and, with d_O, attention): query qg routes over the tree of tokens
// 0 .. positions[qg % nq] (kPathPrefix).  Each query's shared memory holds the route's region
// (grown for the attention's stages when attending, as planned by plan_decode) and the path
// region of its prefix's right edge: inside the row region after the route's candidate rows
// when it fits there, else after the route's region.
cudaError_t launch_causal(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq, int beam,
                          const long long* d_positions, const void* d_K, const void* d_V, float scale,
                          int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                          zha_dtype o_dtype, cudaStream_t stream, bool* unsupported, long long prefix_pos,
                          int buf_tokens) {
  *unsupported = false;
  RouteArgs a = route_args(t, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace);
  const int D = t->desc.head_dim;
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  const int row = D * (bf ? 2 : 4);
  const bool attend = d_O != nullptr;
  const DecodePlan dp = plan_decode(t, q_heads, nq, beam, false);
  const bool wide = a.total_queries <= 2LL * t->sms;
  // Route only: the route's rows.  Attending: the decode plan's row region; in narrow
  // launches grown up to 64 KB, and any number of stages is accepted (the attention
  // pipelines them), since a causal pass has no two-launch fallback.
  size_t rows = std::max(route_rows_bytes(D, a.cmax, sum_bytes(t)), (size_t)4 * 16 * row);
  int nbuf = 2, stage_tokens = (int)(rows / (4 * row)) / 16 * 16;
  if (attend) {
    rows = dp.rows_bytes;
    nbuf = dp.nbuf;
    stage_tokens = dp.stage_tokens;
    if (!wide) {
      const long long tokens = std::min((long long)beam * t->desc.leaf_block, t->N) + buf_tokens;
      rows = std::max(rows, std::min((size_t)2 * row * (size_t)tokens, (size_t)64 * 1024));
      stage_tokens = (int)(rows / (4 * row)) / 16 * 16;
    }
  }
  a.rows_bytes = (int)rows;
  a.K = static_cast<const char*>(d_K);
  a.V = static_cast<const char*>(d_V);
  a.kv_unit_stride = t->desc.capacity_tokens * D * (bf ? 2LL : 4LL);
  a.lb = t->desc.leaf_block;
  a.N = t->N;
  a.qk_scale = scale * 1.4426950408889634f;
  a.stage_tokens = stage_tokens;
  a.attn_nbuf = nbuf;
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  a.positions = d_positions;
  a.prefix_pos = prefix_pos;
  a.buf_leaf0 = (prefix_pos + 1) / t->desc.leaf_block;
  a.buf_tokens = buf_tokens;
  const int pw_warps = wide ? kRouteMaxWarps : kNarrowMaxWpq;
  const size_t route_part = route_smem_layout(D, a.cmax, beam, (size_t)a.rows_bytes, pw_warps).total;
  const size_t path_bytes = path_smem_layout(D, row, sum_bytes(t), (int)a.lb, a.b, t->L).total;
  // The path is needed during the route only, so it goes inside the row region after the
  // route's candidate rows when it fits there (the attention's stages overwrite it once the
  // route is done), else after the query's route layout.
  const size_t path_in_rows = route_align(route_rows_bytes(D, a.cmax, sum_bytes(t)), 128);
  const bool inside = path_in_rows + path_bytes <= (size_t)a.rows_bytes;
  a.path_smem_off = (long long)(inside ? path_in_rows : route_align(route_part, 128));
  const size_t per_query = inside ? route_part : (size_t)a.path_smem_off + path_bytes;
  if ((attend && stage_tokens < 16) || per_query > (wide ? kCtaSmemCap : kRouteSmemCap)) {
    *unsupported = true;
    return cudaSuccess;
  }
  a.query_smem_bytes = (int)per_query;
  const StagedShape sh = staged_shape(t, a, per_query, attend ? dp.attn_warps : 0);
  const cudaError_t e =
      staged_launch(t, true)(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream, kPathPrefix);
  ++t->launches;
  return e;
}

}  // namespace zha

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
#include "decode_append.cuh"
#include "decode_attn.cuh"
#include "device_common.cuh"
#include "route_common.cuh"
#include "zha_internal.h"

namespace zha {

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
// PATH (decode_append.cuh; needs TKV, the type of the K rows the path reads):
//  kPathAppend (fused decode, one query per CTA) -- the kernel first extends the tree by
//    the tokens appended to one leaf, and stores the path (one CTA per unit);
//  kPathPrefix (causal routing) -- query qg routes over the tree of tokens 0 .. p, p =
//    positions[qg % nq]: its own depth and node counts, and its prefix's right edge
//    recomputed into shared memory (never stored).
// With a KV type, the query then attends over its leaves unless O is null.
template <int D, bool GROUPED, typename TKV, bool NARROW, int PATH = kPathNone>
__global__ void __launch_bounds__(NARROW ? 256 : kRouteMaxWarps * 32, NARROW ? 3 : 1)
    route_tma_kernel(const RouteArgs a) {
  constexpr bool ATTEND = !std::is_same<TKV, NoKV>::value;
  constexpr bool APPEND = PATH == kPathAppend;
  constexpr bool PREFIX = PATH == kPathPrefix;
  constexpr bool HASPATH = PATH != kPathNone;
  static_assert(!HASPATH || ATTEND, "the path reads K rows of type TKV");
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
  // the path region (fused append or causal prefix)
  unsigned char* pb = base + a.path_smem_off;
  PathSmem Ps{};
  if (HASPATH) Ps = path_smem_layout(D, D * (int)sizeof(TKV), (int)a.lb, a.b, a.L);
  uint64_t* pbar = reinterpret_cast<uint64_t*>(pb + Ps.bar);
  // this query's tree: the whole tree, or (PREFIX) the tree of its prefix
  long long Nq = a.N;
  bool live = valid;  // a query with a position outside the tree routes nowhere
  if constexpr (PREFIX) {
    const long long pos = valid ? a.positions[qg % a.nq] : 0;
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
  if (wq == 0 && lane == 0) {
    mbar_init(&bar[0], 1);
    if (ATTEND)
      for (int i = 0; i < a.attn_nbuf; ++i) {
        if (i > 0) mbar_init(&bar[i], 1);  // "full" (bar[0] serves the route first)
        mbar_init(&bar[3 + i], nw);        // "empty": one arrival per warp
      }
    if (HASPATH) mbar_init(pbar, 1);
    fence_mbar_init();
    surv_a[0] = 0;  // the root
    if constexpr (HASPATH) {
      if (live) {
        fence_proxy_async_smem();
        const long long leaf = APPEND ? a.path_leaf : (Nq - 1) / a.lb;
        const int ntok = APPEND ? a.path_tokens : (int)(Nq - leaf * a.lb);
        path_issue<TKV, D>(Ps, pb, a.K + unit * a.kv_unit_stride, pyr_u, a.off, nl, a.b, Lq, leaf,
                           ntok, a.lb, pbar);
      }
    }
  }
  qsync();

  // Four lanes per row: lane (rg = lane / 4, sub = lane % 4) reads chunks 4 (j ^ par) + sub,
  // par = rg & 1, so the two rows of a shared-memory phase use opposite bank halves.
  const int sub = lane & 3, rg = lane >> 2, par = rg & 1;
  float4 qv[CPL];
  int* cur = surv_a;
  int* nxt = surv_b;
  int m = live ? 1 : 0;
  uint32_t parity = 0;
  for (int l = Lq - 1; l >= 0; --l) {
    int C = 0;
    if (m > 0) {
      const long long last = cur[m - 1];
      C = (m - 1) * a.b + (int)min((long long)a.b, nl[l] - (long long)a.b * last);
    }
    const float* S = pyr_u + a.off[l] * D;
    if (wq == 0 && C > 0) {
      // one bulk copy per survivor (its children are consecutive rows) + candidate ids
      if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)C * D * 4);
      __syncwarp();
      fence_proxy_async_smem();
      for (int j = lane; j < m; j += 32) {
        const long long node0 = (long long)a.b * cur[j];
        const int nc = (int)min((long long)a.b, nl[l] - node0);
        bulk_copy_g2s((void*)(rows + (size_t)j * a.b * D), S + node0 * D, (uint32_t)nc * D * 4, bar);
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
    if (l == Lq - 1 && valid) {  // load q while the first level is in flight
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
    if (HASPATH && l == Lq - 1) {
      // the path rows, while the first level's copies are in flight
      const bool pok = !live || mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, kRouteWaitCycles);
      const bool pfail = GROUPED ? group_any(bar_id, bar_n, !pok) : __any_sync(0xffffffffu, !pok);
      if (pfail) {
        if (wq == 0 && lane == 0) {  // let all copies land before the CTA exits
          if (live) mbar_wait_bounded(pbar, 0, a.err, kDevErrTimeout, kRouteWaitCycles);
          if (C > 0) mbar_wait_bounded(bar, parity, a.err, kDevErrTimeout, kRouteWaitCycles);
        }
        return;
      }
      if constexpr (HASPATH) {
        if (live) {
          // fused append: the first query of each unit stores the path
          const bool writer = APPEND && (qg % a.nq) == 0 && ((qg / a.nq) % a.q_heads) % a.group == 0;
          const int ntok = APPEND ? a.path_tokens : (int)(Nq - ((Nq - 1) / a.lb) * a.lb);
          path_compute<TKV, D>(Ps, pb, const_cast<float*>(pyr_u), a.off, nl, a.b, Lq, ntok, writer,
                               32 * wq + lane, bar_n, qsync);
        }
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
    if (HASPATH) {
      // the staged row of the path node may predate the append, or (prefix) cover tokens
      // past the query's prefix: use the recomputed one
      const int k = *reinterpret_cast<const int*>(pb + Ps.kpos);
      if (k >= 0) {
        const float* pf = reinterpret_cast<const float*>(pb + Ps.pf) + (size_t)l * D;
        float* dst = const_cast<float*>(rows) + (size_t)k * D;
        for (int e = 32 * wq + lane; e < D; e += bar_n) dst[e] = pf[e];
        qsync();
      }
    }

    // score: rows r = 8 (wq + nw t) + rg, two rows per lane in flight
    for (int r0 = 8 * wq; r0 < C; r0 += 16 * nw) {
      // four running sums per row (dims 4c + e for e = 0..3), updated pairwise by packed FMAs
      float2 acc[2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = r0 + 8 * nw * u + rg;
        acc[u][0] = make_float2(0.f, 0.f);
        acc[u][1] = make_float2(0.f, 0.f);
        if (r < C) {
          const float4* row = reinterpret_cast<const float4*>(rows + (size_t)r * D);
#pragma unroll
          for (int j = 0; j < CPL; ++j) {
            const float4 v = row[4 * (j ^ par) + sub];
            acc[u][0] = __ffma2_rn(make_float2(qv[j].x, qv[j].y), make_float2(v.x, v.y), acc[u][0]);
            acc[u][1] = __ffma2_rn(make_float2(qv[j].z, qv[j].w), make_float2(v.z, v.w), acc[u][1]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float s = (acc[u][0].x + acc[u][0].y) + (acc[u][1].x + acc[u][1].y);
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
    } else if (GROUPED && C <= 32 * nw) {  // radix selection over the group
      const int kept = select_radix_group(keys, cand, C, a.beam, nxt, leaf_sc, l == 0, red,
                                          reinterpret_cast<unsigned*>(base + Ls.hist), wq, lane, nw, bar_id);
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
    sa.lb = (int)a.lb;
    sa.total = leaf_tokens(cur, m, a.lb, Nq);
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
    sa.wait_cycles = kRouteWaitCycles;
    const int nst = (sa.total + sa.TS - 1) / sa.TS;
    if (wq == 0)
      for (int st = 0; st < min(nst, sa.nbuf); ++st)
        attn_issue_stage<S::ROWB>(cur, sa.lb, sa.total, sa.TS, st, sa.nbuf, sa.sb, sa.Ku, sa.Vu, bar, lane);
    float qa[S::CPL][S::VEC];
    if (valid) attn_load_q<TKV, D>(a.Q, a.q_bf16 != 0, qg, lane, qa);
    float* pw = reinterpret_cast<float*>(base + Ls.pw) + wq * 16;
    attend_staged<TKV, D>(sa, qg, valid, qa, pw, reinterpret_cast<float*>(red), wq, nw, lane, bar_id);
  }
}

namespace {
template <int D, bool GROUPED, typename TKV, bool NARROW, int PATH = kPathNone>
cudaError_t run_route_tma(const RouteArgs& a, unsigned blocks, int threads, size_t smem,
                          cudaStream_t s) {
  auto kern = route_tma_kernel<D, GROUPED, TKV, NARROW, PATH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(blocks), dim3(threads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TKV, int PATH>
cudaError_t run_shape(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks, int threads,
                      size_t smem, cudaStream_t s) {
  if constexpr (PATH != kPathAppend) {  // the fused append runs in wide launches only
    if (narrow) {
      if (grouped)
        return D == 128 ? run_route_tma<128, true, TKV, true, PATH>(a, blocks, threads, smem, s)
                        : run_route_tma<64, true, TKV, true, PATH>(a, blocks, threads, smem, s);
      return D == 128 ? run_route_tma<128, false, TKV, true, PATH>(a, blocks, threads, smem, s)
                      : run_route_tma<64, false, TKV, true, PATH>(a, blocks, threads, smem, s);
    }
  } else if (narrow) {
    return cudaErrorNotSupported;
  }
  if (grouped)
    return D == 128 ? run_route_tma<128, true, TKV, false, PATH>(a, blocks, threads, smem, s)
                    : run_route_tma<64, true, TKV, false, PATH>(a, blocks, threads, smem, s);
  return D == 128 ? run_route_tma<128, false, TKV, false, PATH>(a, blocks, threads, smem, s)
                  : run_route_tma<64, false, TKV, false, PATH>(a, blocks, threads, smem, s);
}

template <typename TKV>
cudaError_t run_route_tma_d(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks,
                            int threads, size_t smem, cudaStream_t s, int path = kPathNone) {
  if constexpr (!std::is_same<TKV, NoKV>::value) {
    if (path == kPathAppend) return run_shape<TKV, kPathAppend>(D, grouped, narrow, a, blocks, threads, smem, s);
    if (path == kPathPrefix) return run_shape<TKV, kPathPrefix>(D, grouped, narrow, a, blocks, threads, smem, s);
  }
  return run_shape<TKV, kPathNone>(D, grouped, narrow, a, blocks, threads, smem, s);
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
constexpr size_t kCtaSmemCap = 227 * 1024;    // dynamic shared memory of one CTA

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

  a.rows_bytes = (int)route_rows_bytes(D, a.cmax);
  // Staged kernel when a query's widest level fits in shared memory.
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

// Fused route + attention (one launch).  Wide launches (one query per CTA): the row region
// grows so that the attention streams its leaves through up to three large stages in
// flight together -- up to 192 KB when every CTA has an SM to itself, 96 KB when two share
// one -- and, with an SM to itself, also holds the one-leaf append's path after the route's
// rows (decode_append.cuh).  Narrow launches (several queries per SM): the row region
// stays the route's own, since a larger one would cut the queries resident per SM, and the
// call is fused only when the query's tokens then fit in at most two stages; otherwise
// fused = false and the route and the attention run as two launches.  Stages hold a
// multiple of 16 tokens (the attention's rounds), at least 16.
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
  if (!wide) {
    p.nbuf = 2;
    p.rows_bytes = std::max(route_rows, (size_t)4 * 16 * row);  // two stages of 16 tokens at least
    p.stage_tokens = (int)(p.rows_bytes / (4 * row)) / 16 * 16;
    p.attn_warps = 1;
    p.smem_per_query = route_smem_layout(D, (int)cmax, beam, p.rows_bytes, narrow_wpq(cmax)).total;
    p.fused = p.smem_per_query <= kRouteSmemCap && p.stage_tokens >= 16 && 2LL * p.stage_tokens >= tokens;
    return p;
  }
  const bool own_sm = queries <= t->sms;
  const size_t cap = own_sm ? 192 * 1024 : 96 * 1024;
  size_t rows = std::min((size_t)2 * row * (size_t)tokens, cap);  // all the tokens, if they fit
  rows = std::max(std::max(rows, route_rows), (size_t)4 * 16 * row);
  p.path_bytes = path_smem_layout(D, row, (int)t->desc.leaf_block, t->desc.branching, t->L).total;
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
  a.stage_tokens = p.stage_tokens;
  a.attn_nbuf = p.nbuf;
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  a.query_smem_bytes = (int)p.smem_per_query;  // weight area sized for 16 warps when wide
  StagedShape sh = staged_shape(t, a, p.smem_per_query, p.attn_warps);
  const bool append = append_leaf >= 0;
  if (append) {  // the tree already has its new shape; the path region follows the route's
    a.path_leaf = append_leaf;
    a.path_tokens = (int)(std::min(append_leaf * a.lb + a.lb, t->N) - append_leaf * a.lb);
    a.path_smem_off = (long long)p.path_off;  // inside the row region, after the route's rows
  }
  cudaError_t e;
  if (bf)
    e = run_route_tma_d<uint16_t>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream,
                                  append ? kPathAppend : kPathNone);
  else
    e = run_route_tma_d<float>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem, stream,
                               append ? kPathAppend : kPathNone);
  ++t->launches;
  return e;
}

// Causal routing (and, with d_O, attention): query qg routes over the tree of tokens
// 0 .. positions[qg % nq] (kPathPrefix).  Each query's shared memory holds the route's region
// (grown for the attention's stages when attending, as planned by plan_decode) followed by
// the path region of its prefix's right edge.
cudaError_t launch_causal(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq, int beam,
                          const long long* d_positions, const void* d_K, const void* d_V, float scale,
                          int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                          zha_dtype o_dtype, cudaStream_t stream, bool* unsupported) {
  *unsupported = false;
  RouteArgs a = route_args(t, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace);
  const int D = t->desc.head_dim;
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  const int row = D * (bf ? 2 : 4);
  const bool attend = d_O != nullptr;
  const DecodePlan dp = plan_decode(t, q_heads, nq, beam);
  const bool wide = a.total_queries <= 2LL * t->sms;
  // Route only: the route's rows.  Attending: the decode plan's row region; in narrow
  // launches grown up to 64 KB, and any number of stages is accepted (the attention
  // pipelines them), since a causal pass has no two-launch fallback.
  size_t rows = std::max(route_rows_bytes(D, a.cmax), (size_t)4 * 16 * row);
  int nbuf = 2, stage_tokens = (int)(rows / (4 * row)) / 16 * 16;
  if (attend) {
    rows = dp.rows_bytes;
    nbuf = dp.nbuf;
    stage_tokens = dp.stage_tokens;
    if (!wide) {
      const long long tokens = std::min((long long)beam * t->desc.leaf_block, t->N);
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
  const int pw_warps = wide ? kRouteMaxWarps : narrow_wpq(a.cmax);
  const size_t route_part = route_smem_layout(D, a.cmax, beam, (size_t)a.rows_bytes, pw_warps).total;
  const size_t path_bytes = path_smem_layout(D, row, (int)a.lb, a.b, t->L).total;
  a.path_smem_off = (long long)route_align(route_part, 128);
  const size_t per_query = (size_t)a.path_smem_off + path_bytes;
  if ((attend && stage_tokens < 16) || per_query > (wide ? kCtaSmemCap : kRouteSmemCap)) {
    *unsupported = true;
    return cudaSuccess;
  }
  a.query_smem_bytes = (int)per_query;
  const StagedShape sh = staged_shape(t, a, per_query, attend ? dp.attn_warps : 0);
  cudaError_t e = bf ? run_route_tma_d<uint16_t>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem,
                                                 stream, kPathPrefix)
                     : run_route_tma_d<float>(D, sh.grouped, !sh.wide, a, sh.blocks, sh.threads, sh.smem,
                                              stream, kPathPrefix);
  ++t->launches;
  return e;
}

}  // namespace zha

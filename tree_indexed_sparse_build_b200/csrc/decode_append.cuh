// One-leaf append inside the fused decode kernel.
//
// When a decode step appends tokens that all fall into one leaf (the usual case: one token),
// only the path from that leaf to the root changes ("Subquadratic Attention with a
// Hierarchical Tree-Structured Indexer", abstract: the tree is updated as the cache grows).
// Every CTA that routes a query of the unit recomputes that path itself, with the same
// arithmetic and summation order as the stand-alone append kernel (leaf = fp64 sum of its
// tokens in order / count; a parent = fp64 sum of its existing children in index order /
// count, the touched child taken from its kept fp64 value, the others from their stored
// rows; SumT rounds and keeps as the append kernel does for fp32 and bf16 summaries), so the
// rows are bit-identical to what the append kernel writes.  One CTA per unit
// writes them back; every CTA patches them into its own staged candidate rows, so no CTA
// waits for another.  The path's copies (the leaf's tokens, each level's children of the
// path node) are in flight together with the route's first level.
#pragma once

#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

// Shared memory of the path, for head_dim D, token rows of row_bytes, summary elements of
// sum_bytes, leaf block lb, branching b and (at most) L levels below the root.
struct PathSmem {
  size_t tok, sib, pf, node, kpos, qn, bar, total;
};
__host__ __device__ inline size_t path_align(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline PathSmem path_smem_layout(int D, int row_bytes, int sum_bytes, int lb, int b,
                                                     int L) {
  PathSmem s;
  size_t o = 0;
  s.tok = o;   // the leaf's tokens [lb][row_bytes]
  o = path_align(o + (size_t)lb * row_bytes, 16);
  s.sib = o;   // for l = 1..L: the children of path node l, stored rows [b][D]
  o += (size_t)L * b * D * sum_bytes;
  s.pf = o;    // the stored path rows, levels 0..L [L + 1][D]
  o = path_align(o + (size_t)(L + 1) * D * sum_bytes, 8);
  s.node = o;  // path node index per level [L + 1]
  o += (size_t)(L + 1) * 8;
  s.kpos = o;  // candidate slot of the path node at the current route level
  o += 8;
  s.qn = o;    // causal routing: the prefix tree's node counts per level; its depth last
  o += (size_t)kMaxLevels * 8;
  s.bar = o;
  o += 8;
  s.total = path_align(o, 128);
  return s;
}

// One thread: path nodes, then the bulk copies of the leaf's tokens and of every level's
// children of the path node, all completing on pbar.  Ku: the unit's K rows; pyr_u: the
// unit's summaries; off / n: level offsets and node counts after the append.  nodes: the
// path's nodes at levels 0 .. L when the caller has them (else computed from leaf).
template <typename TIn, typename TS, int D>
__device__ void path_issue(const PathSmem& P, unsigned char* pb, const char* Ku, const TS* pyr_u,
                           const long long* off, const long long* n, int b, int L, long long leaf,
                           int ntok, long long lb, uint64_t* pbar, const long long* nodes = nullptr) {
  long long* node = reinterpret_cast<long long*>(pb + P.node);
  node[0] = leaf;
  for (int l = 1; l <= L; ++l) node[l] = nodes ? nodes[l] : node[l - 1] / b;
  uint32_t bytes = (uint32_t)ntok * D * sizeof(TIn);
  for (int l = 1; l <= L; ++l) {
    const long long c0 = node[l] * b, c1 = min(c0 + (long long)b, n[l - 1]);
    bytes += (uint32_t)(c1 - c0) * D * (uint32_t)sizeof(TS);
  }
  mbar_arrive_expect_tx(pbar, bytes);
  bulk_copy_g2s(pb + P.tok, Ku + leaf * lb * D * (long long)sizeof(TIn), (uint32_t)ntok * D * sizeof(TIn),
                pbar);
  for (int l = 1; l <= L; ++l) {
    const long long c0 = node[l] * b, c1 = min(c0 + (long long)b, n[l - 1]);
    bulk_copy_g2s(pb + P.sib + (size_t)(l - 1) * b * D * sizeof(TS), pyr_u + (off[l - 1] + c0) * D,
                  (uint32_t)(c1 - c0) * D * (uint32_t)sizeof(TS), pbar);
  }
}

// Threads tid < D of the group (nt threads in all): the path rows, after pbar completed.
// Each thread carries its dims e = tid, tid + nt, .. from the leaf to the root with the
// kept fp64 value in a register (a level's dim e needs only dim e of the level below), so
// the levels need no barrier; sync() once at the end makes the rows visible to the group.
// writer: also store the rows into the unit's summaries.
template <typename TIn, typename TS, int D, typename Sync>
__device__ void path_compute(const PathSmem& P, unsigned char* pb, TS* pyr_u, const long long* off,
                             const long long* n, int b, int L, int ntok, bool writer, int tid, int nt,
                             Sync sync) {
  const TIn* tok = reinterpret_cast<const TIn*>(pb + P.tok);
  TS* pf = reinterpret_cast<TS*>(pb + P.pf);
  const long long* node = reinterpret_cast<const long long*>(pb + P.node);
  for (int e = tid; e < D; e += nt) {
    double s = 0.0;
    for (int r = 0; r < ntok; ++r) {
      if constexpr (sizeof(TIn) == 2)
        s += (double)bf16_bits_to_f32(tok[(size_t)r * D + e]);
      else
        s += (double)tok[(size_t)r * D + e];
    }
    double v = s / (double)ntok;
    double kept = SumT<TS>::kept(v);
    pf[e] = SumT<TS>::store(v);
    if (writer) pyr_u[(off[0] + node[0]) * D + e] = pf[e];
    for (int l = 1; l <= L; ++l) {
      const TS* sib = reinterpret_cast<const TS*>(pb + P.sib + (size_t)(l - 1) * b * D * sizeof(TS));
      const long long c0 = node[l] * b, c1 = min(c0 + (long long)b, n[l - 1]);
      double t = 0.0;
      for (long long c = c0; c < c1; ++c)
        t += c == node[l - 1] ? kept : (double)SumT<TS>::load(sib[(c - c0) * D + e]);
      v = t / (double)(c1 - c0);
      kept = SumT<TS>::kept(v);
      pf[(size_t)l * D + e] = SumT<TS>::store(v);
      if (writer) pyr_u[(off[l] + node[l]) * D + e] = pf[(size_t)l * D + e];
    }
  }
  sync();
}

}  // namespace zha

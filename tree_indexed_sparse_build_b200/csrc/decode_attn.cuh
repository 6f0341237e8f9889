// Attention epilogue of the fused decode kernels: exact softmax attention of one query over
// the tokens of its selected leaves ("Subquadratic Attention with a Hierarchical
// Tree-Structured Indexer", abstract: the final attention runs over the sparse subset of
// keys the tree traversal retrieved), run by the warps that routed the query.
//
// The leaves' K and V rows stream through nbuf (2 or 3) stage buffers of TS tokens each
// (K rows then V rows per buffer), one 1-D bulk copy (non-multicast TMA) per leaf piece,
// completing on one mbarrier per buffer; the first nbuf stages are in flight together.  The warps run the online softmax of attn_core.cuh over each
// stage, merge their states through shared memory and write O.
#pragma once

#include "attn_core.cuh"
#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

// Tokens of the selected leaves in slot order.  Only leaf n0 - 1 can hold fewer than lb
// tokens, and leaves ascend, so it can only be the last one.
__device__ __forceinline__ int leaf_tokens(const int* leaves, int m, long long lb, long long N) {
  if (m <= 0) return 0;
  const long long last = leaves[m - 1];
  return (m - 1) * (int)lb + (int)(min(last * lb + lb, N) - last * lb);
}

// Stage st covers tokens [st TS, min(st TS + TS, total)) and goes to buffer st % nbuf of
// sb, completing on bars[st % nbuf].  Called by all lanes of one warp; each lane copies the
// K and V pieces of some of the stage's leaves.  Token slot j lb .. j lb + lb - 1 belongs to
// leaf leaves[j] for j < m and to leaf buf_leaf0 + (j - m) after them (an append buffer:
// consecutive leaves after the routed ones, the last one possibly partial).
template <int ROWB>
__device__ __forceinline__ void attn_issue_stage(const int* leaves, int m, long long buf_leaf0, int lb,
                                                 int total, int TS, int st, int nbuf, unsigned char* sb,
                                                 const char* Ku, const char* Vu, uint64_t* bars, int lane) {
  const size_t stage_bytes = (size_t)TS * ROWB;
  const int b = st % nbuf;
  unsigned char* kb = sb + (size_t)b * 2 * stage_bytes;
  const int w0 = st * TS, w1 = min(w0 + TS, total);
  if (lane == 0) mbar_arrive_expect_tx(&bars[b], (uint32_t)(2 * (w1 - w0) * ROWB));
  __syncwarp();
  fence_proxy_async_smem();
  for (int j = w0 / lb + lane; j <= (w1 - 1) / lb; j += 32) {
    const int p0 = j * lb;
    const int a0 = max(p0, w0), a1 = min(p0 + lb, w1);
    const long long leaf = j < m ? (long long)leaves[j] : buf_leaf0 + (j - m);
    const long long row = leaf * lb + (a0 - p0);
    const uint32_t bytes = (uint32_t)((a1 - a0) * ROWB);
    bulk_copy_g2s(kb + (size_t)(a0 - w0) * ROWB, Ku + row * ROWB, bytes, &bars[b]);
    bulk_copy_g2s(kb + stage_bytes + (size_t)(a0 - w0) * ROWB, Vu + row * ROWB, bytes, &bars[b]);
  }
}

// Where the attention of one query runs and what it reads.
struct StagedAttn {
  const int* leaves;     // shared memory, ascending
  int m;                 // routed leaves
  long long buf_leaf0;   // first leaf of the append buffer's tokens (slots m, m + 1, ..)
  int lb;                // tokens per leaf
  int total;             // tokens (leaf_tokens, plus the buffer's)
  int TS;                // tokens per stage buffer, a multiple of 16
  int nbuf;              // stage buffers, 2 or 3
  unsigned char* sb;     // the stage buffers; >= nw * D * 4 bytes (warp merge reuses them)
  uint64_t* bars;        // "full" mbarriers, one per buffer (arrival count 1)
  uint64_t* empty;       // "empty" mbarriers, one per buffer (arrival count nw)
  uint32_t ph0;          // phase of bars[0]'s next completion (the others start at 0)
  const char* Ku;        // this query's KV head
  const char* Vu;
  float qk_scale;        // scale * log2(e)
  void* O;               // output row qg of [queries, D]
  int o_bf16;
  unsigned* err;
  long long wait_cycles;   // bound of a first wait for a stage's copies
  long long drain_cycles;  // bound of the waits that let copies land after a failure
};

// Called by every thread of the query's nw warps (warp wq, lane), after warp 0 issued
// stages 0 .. nbuf - 1 (those that exist).  The tokens go in rounds of 16 to the warps in
// turn (round g of the whole token list to warp g mod nw), so a warp waits only for the
// stages holding its rounds.  Every warp arrives on a buffer's "empty" barrier once it is
// past that stage; warp 0 then refills the buffer with the stage nbuf further on.  No CTA
// barrier runs between stages.  Synchronises on named barrier bar_id (when nw > 1) only to
// merge the warps' states at the end.  qv: this lane's q slice (attn_load_q).  pw: 16
// floats per warp; redf: 48 floats.  Returns false after a bounded wait ran out (O is
// then NaN).
template <typename TKV, int D>
__device__ bool attend_staged(const StagedAttn& s, long long qg, bool valid,
                              const float (&qv)[AttnShape<TKV, D>::CPL][AttnShape<TKV, D>::VEC],
                              float* pw, float* redf, int wq, int nw, int lane, int bar_id) {
  using S = AttnShape<TKV, D>;
  constexpr int ROWB = S::ROWB;
  const int nt = 32 * nw;
  const size_t stage_bytes = (size_t)s.TS * ROWB;
  const int nst = (s.total + s.TS - 1) / s.TS;
  const int rps = s.TS / 16;  // rounds per full stage
  auto phase = [&](int st) -> uint32_t {
    return ((st % s.nbuf) ? 0u : s.ph0) ^ (uint32_t)((st / s.nbuf) & 1);
  };
  float m_w = -INFINITY, l_w = 0.f;
  float acc[S::DPL];
#pragma unroll
  for (int e = 0; e < S::DPL; ++e) acc[e] = 0.f;
  bool ok = true;
  int issued = min(nst, s.nbuf);  // warp 0: stages issued so far
  for (int st = 0; st < nst; ++st) {
    const int b = st % s.nbuf;
    const int cnt = min(s.TS, s.total - st * s.TS);
    const int rounds = (cnt + 15) / 16;
    const int r0 = ((wq - st * rps) % nw + nw) % nw;  // this warp's first round in the stage
    // Every warp waits for every stage, its rounds or not: a stage is full only after the
    // previous use of its buffer was released, so no warp's "empty" arrival below can count
    // toward that earlier release.
    if (ok) ok = mbar_wait_bounded(&s.bars[b], phase(st), s.err, kDevErrTimeout, s.wait_cycles);
    ok = __all_sync(0xffffffffu, ok);  // one outcome per warp before its full-warp shuffles
    if (ok && r0 < rounds) {
      const unsigned char* Ks = s.sb + (size_t)b * 2 * stage_bytes;
      attn_tokens<TKV, D>(Ks, Ks + stage_bytes, cnt, 16 * r0, 8, 16 * nw, qv, s.qk_scale, pw, m_w, l_w,
                          acc, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[b]);
    if (wq == 0 && st + s.nbuf < nst && ok) {
      // refill buffer b once every warp is past stage st
      ok = mbar_wait_bounded(&s.empty[b], (uint32_t)((st / s.nbuf) & 1), s.err, kDevErrTimeout,
                             s.drain_cycles);
      __syncwarp();
      if (ok) {
        attn_issue_stage<ROWB>(s.leaves, s.m, s.buf_leaf0, s.lb, s.total, s.TS, st + s.nbuf, s.nbuf, s.sb, s.Ku, s.Vu,
                               s.bars, lane);
        issued = st + s.nbuf + 1;
      }
    }
  }
  const bool failed = nw > 1 ? group_any(bar_id, nt, !ok) : __any_sync(0xffffffffu, !ok);
  if (failed) {
    // let the copies in flight land before the shared memory is released (bounded waits on
    // the last stages warp 0 issued); the output is poisoned so the failure shows besides
    // the error word
    if (wq == 0 && lane == 0)
      for (int st = max(0, issued - s.nbuf); st < issued; ++st)
        mbar_wait_bounded(&s.bars[st % s.nbuf], phase(st), s.err, kDevErrTimeout, s.drain_cycles);
    if (valid && wq == 0)
      for (int e = lane; e < D; e += 32) {
        if (s.o_bf16)
          static_cast<uint16_t*>(s.O)[qg * D + e] = 0x7FC0u;
        else
          static_cast<float*>(s.O)[qg * D + e] = __int_as_float(0x7fc00000);
      }
    return false;
  }
  l_w = warp_sum(l_w);
  if (nw > 1) {
    // merge the warps' states; the accumulators reuse the stage buffers (every copy has
    // landed: each stage was waited on by the warps holding its rounds)
    float* accr = reinterpret_cast<float*>(s.sb);
#pragma unroll
    for (int e = 0; e < S::DPL; ++e) accr[wq * D + lane * S::DPL + e] = acc[e];
    if (lane == 0) {
      redf[wq] = m_w;
      redf[16 + wq] = l_w;
    }
    group_sync(bar_id, nt);
    if (wq == 0 && lane < nw) {  // each warp's weight 2^(m_w - M)
      float M = -INFINITY;
      for (int w = 0; w < nw; ++w) M = fmaxf(M, redf[w]);
      redf[32 + lane] = redf[lane] == -INFINITY ? 0.f : exp2f(redf[lane] - M);
    }
    group_sync(bar_id, nt);
    for (int d = 32 * wq + lane; d < D && valid; d += nt) {
      float o = 0.f, l = 0.f;
      for (int w = 0; w < nw; ++w) {
        o = fmaf(redf[32 + w], accr[w * D + d], o);
        l = fmaf(redf[32 + w], redf[16 + w], l);
      }
      const float r = l > 0.f ? o / l : 0.f;
      if (s.o_bf16)
        static_cast<uint16_t*>(s.O)[qg * D + d] = f32_to_bf16_bits(r);
      else
        static_cast<float*>(s.O)[qg * D + d] = r;
    }
    group_sync(bar_id, nt);  // the merge buffers are free again when this returns
  } else if (valid) {
#pragma unroll
    for (int e = 0; e < S::DPL; ++e) {
      const float r = l_w > 0.f ? acc[e] / l_w : 0.f;
      const long long o = qg * D + lane * S::DPL + e;
      if (s.o_bf16)
        static_cast<uint16_t*>(s.O)[o] = f32_to_bf16_bits(r);
      else
        static_cast<float*>(s.O)[o] = r;
    }
  }
  return true;
}

}  // namespace zha

// Exact softmax attention over the tokens of the selected leaves ("Subquadratic
// Attention with a Hierarchical Tree-Structured Indexer", abstract: the final attention
// runs over the sparse subset of keys the tree traversal retrieved).
//
//   s_t = scale * q . K[t],  o = sum_t exp(s_t - max) V[t] / sum_t exp(s_t - max)
// over t < N in the union of the selected leaves' token blocks.
//
// GPU mapping: one CTA per (query, split), where a split is a contiguous run of the
// query's beam slots.  A leaf's K rows (and V rows) are contiguous in memory, so each
// leaf piece of a stage is fetched with one 1-D bulk copy (non-multicast TMA) into a
// shared-memory stage, completing on an mbarrier; the lanes of warp 0 issue the copies
// of a stage in parallel.  Splits are sized so a split is usually a single stage; when a
// split spans several stages, two stage buffers alternate so the next copy overlaps this
// stage's arithmetic.  Four lanes score a token against q held in registers (neighbouring
// tokens read their chunks in opposite orders, so the two tokens of a shared-memory phase
// hit opposite bank halves).  Each warp keeps its own online softmax (running max and sum
// in the log2 domain) over the tokens it owns; each lane accumulates head_dim/32 output
// dims; the four warps merge at the end.
//
// Splits of one query are merged in one of two ways:
//  - cluster path (at most 8 splits): the splits of a query form one thread-block cluster
//    and send their (acc, max, sum) to the rank-0 CTA's shared memory (distributed shared
//    memory); rank 0 merges and writes O.  No scratch, no second kernel.
//  - scratch path (more splits): partials go to caller scratch and combine_kernel merges.
//
// Every wait on an mbarrier is bounded by a clock budget; on expiry the kernel records
// kDevErrTimeout in the device error word and stops using the stage (no trap).
#include <cooperative_groups.h>

#include <algorithm>

#include "attn_core.cuh"
#include "device_common.cuh"
#include "zha_internal.h"

namespace cg = cooperative_groups;

namespace zha {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr long long kWaitCycles = kCopyWaitCycles;  // ~1 s at 1.9 GHz

struct AttnArgs {
  const void* Q;
  int q_bf16;
  const char* K;
  const char* V;
  long long kv_unit_stride;  // bytes
  const int* leaf_idx;
  int q_heads, nq, group, kv_heads, beam;
  long long lb, N, n0;
  float qk_scale;  // scale * log2(e)
  int lps, splits, stage_tokens, nbuf;
  void* O;
  int o_bf16;
  float* partial;  // scratch path: [queries][splits][D + 2]
  unsigned* err;
  long long total_items;
  long long first_wait;  // bound of a first wait for a stage's copies
};

// Shared-memory layout, identical on host and device.
struct AttnSmem {
  size_t red, meta, lids, lpos, pw, accr, part, kv, total;
};
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline AttnSmem attn_smem_layout(int D, int row_bytes, int lps, int stage_tokens,
                                                     int nbuf, bool cluster) {
  AttnSmem s;
  size_t o = 16;  // two mbarriers
  s.red = o;
  o += 8 * 4;
  s.meta = o;
  o += 4 * 4;
  s.lids = o;
  o += (size_t)lps * 4;
  s.lpos = o;
  o += (size_t)(lps + 1) * 4;
  s.pw = align_up(o, 16);  // per-warp softmax weights of one round [warps][16]
  o = s.pw + (size_t)kAttnWarps * 16 * 4;
  s.kv = align_up(o, 128);
  // After the last stage the stage buffers are free: the four warps' accumulators and, in
  // the cluster path (rank 0), the splits' partials [8][D + 2] reuse them.
  s.accr = s.kv;
  s.part = s.kv + align_up((size_t)kAttnWarps * D * 4, 16);
  const size_t tail = (s.part - s.kv) + (cluster ? (size_t)kMaxClusterSplits * (D + 2) * 4 : 0);
  const size_t stages = (size_t)nbuf * 2 * stage_tokens * row_bytes;
  s.total = s.kv + (stages > tail ? stages : tail);
  return s;
}

// Issue the bulk copies of stage `s` (tokens [s*TS, s*TS + TS) of the work item's token
// sequence) into buffers kbuf/vbuf.  Called by all lanes of one warp: lane 0 registers the
// stage's byte count on the barrier, then each lane copies the pieces of its leaves.
template <int ROWB>
__device__ void issue_stage(const AttnArgs& a, const char* Ku, const char* Vu, const int* lids,
                            const int* lpos, int nle, int s, unsigned char* kbuf,
                            unsigned char* vbuf, uint64_t* bar, int lane) {
  const int TS = a.stage_tokens;
  const int total = lpos[nle];
  const int w0 = s * TS, w1 = min(w0 + TS, total);
  if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(2 * (w1 - w0) * ROWB));
  __syncwarp();
  fence_proxy_async_smem();
  for (int j = lane; j < nle; j += 32) {
    const int p0 = lpos[j], p1 = lpos[j + 1];
    const int a0 = max(p0, w0), a1 = min(p1, w1);
    if (a0 >= a1) continue;
    const long long row = (long long)lids[j] * a.lb + (a0 - p0);
    const uint32_t bytes = (uint32_t)((a1 - a0) * ROWB);
    const size_t dst = (size_t)(a0 - w0) * ROWB;
    bulk_copy_g2s(kbuf + dst, Ku + row * ROWB, bytes, bar);
    bulk_copy_g2s(vbuf + dst, Vu + row * ROWB, bytes, bar);
  }
}

template <typename TKV, int D, bool CLUSTER>
__global__ void __launch_bounds__(kAttnThreads) attend_kernel(const AttnArgs a) {
  using S = AttnShape<TKV, D>;
  constexpr int ROWB = S::ROWB;
  constexpr int VEC = S::VEC;
  constexpr int CPL = S::CPL;
  constexpr int DPL = S::DPL;

  extern __shared__ __align__(128) unsigned char smem[];
  const AttnSmem L = attn_smem_layout(D, ROWB, a.lps, a.stage_tokens, a.nbuf, CLUSTER);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + L.red);
  int* meta = reinterpret_cast<int*>(smem + L.meta);
  int* lids = reinterpret_cast<int*>(smem + L.lids);
  int* lpos = reinterpret_cast<int*>(smem + L.lpos);
  float* accr = reinterpret_cast<float*>(smem + L.accr);
  float* part = reinterpret_cast<float*>(smem + L.part);
  unsigned char* kv = smem + L.kv;
  const int TS = a.stage_tokens;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* pw = reinterpret_cast<float*>(smem + L.pw) + warp * 16;
  const long long item = blockIdx.x;
  const long long qg = item / a.splits;
  const int split = (int)(item - qg * a.splits);
  const long long hq_flat = qg / a.nq;
  const int h = (int)(hq_flat % a.q_heads);
  const long long unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
  const char* Ku = a.K + unit * a.kv_unit_stride;
  const char* Vu = a.V + unit * a.kv_unit_stride;
  pdl_wait();
  pdl_release();

  // Query slice into registers (four lanes per token, see attn_core.cuh).
  float qv[CPL][VEC];
  attn_load_q<TKV, D>(a.Q, a.q_bf16 != 0, qg, lane, qv);
  // Leaf list of this split, built by warp 0: valid leaves compacted in slot order, with
  // the prefix of their token counts (their offsets in the split's token sequence).
  if (warp == 0) {
    const int s0 = split * a.lps, s1 = min(s0 + a.lps, a.beam);
    const int* li = a.leaf_idx + qg * a.beam;
    int cnt = 0, pos = 0;
    for (int c0 = s0; c0 < s1; c0 += 32) {
      const int sl = c0 + lane;
      int j = sl < s1 ? li[sl] : -1;
      if ((long long)j >= a.n0) {
        atomicOr(a.err, kDevErrBadLeaf);
        j = -1;
      }
      const bool ok = j >= 0;
      const int ntok = ok ? (int)(min((long long)j * a.lb + a.lb, a.N) - (long long)j * a.lb) : 0;
      int incl = ntok;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        const int k = cnt + __popc(bal & ((1u << lane) - 1u));
        lids[k] = j;
        lpos[k] = pos + incl - ntok;
      }
      cnt += __popc(bal);
      pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      lpos[cnt] = pos;
      meta[0] = cnt;
      mbar_init(&bar[0], 1);
      mbar_init(&bar[1], 1);
      fence_mbar_init();
    }
    __syncwarp();
    const int total0 = pos;
    const int nst0 = (total0 + TS - 1) / TS;
    for (int s = 0; s < min(a.nbuf, nst0); ++s)
      issue_stage<ROWB>(a, Ku, Vu, lids, lpos, cnt, s, kv + (size_t)s * 2 * TS * ROWB,
                        kv + (size_t)s * 2 * TS * ROWB + (size_t)TS * ROWB, &bar[s], lane);
  }
  __syncthreads();
  const int nle = meta[0];
  const int total = lpos[nle];
  const int nstages = (total + TS - 1) / TS;
  const size_t stage_bytes = (size_t)TS * ROWB;

  // this warp's running softmax state over the tokens it owns
  float m_w = -INFINITY, l_w = 0.f;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  bool failed = false;
  int failed_stage = 0;

  for (int s = 0; s < nstages; ++s) {
    const int buf = a.nbuf == 2 ? (s & 1) : 0;
    const uint32_t parity = (uint32_t)((a.nbuf == 2 ? (s >> 1) : s) & 1);
    const bool ok = mbar_wait_bounded(&bar[buf], parity, a.err, kDevErrTimeout, a.first_wait);
    // one barrier per stage: the stage's data is visible to all, every warp has finished
    // the previous stage (whose buffer the next copy may now overwrite)
    if (__syncthreads_or(!ok)) {
      failed = true;
      failed_stage = s;
      break;
    }
    if (warp == 0 && a.nbuf == 2 && s >= 1 && s + 1 < nstages) {
      const int nb = (s + 1) & 1;
      issue_stage<ROWB>(a, Ku, Vu, lids, lpos, nle, s + 1, kv + (size_t)nb * 2 * stage_bytes,
                        kv + (size_t)nb * 2 * stage_bytes + stage_bytes, &bar[nb], lane);
    }
    const unsigned char* Ks = kv + (size_t)buf * 2 * stage_bytes;
    const unsigned char* Vs = Ks + stage_bytes;
    const int cnt = min(TS, total - s * TS);

    // rounds of 64 tokens: this warp takes tokens t0 + tg and t0 + 32 + tg
    attn_tokens<TKV, D>(Ks, Vs, cnt, 8 * warp, 32, 64, qv, a.qk_scale, pw, m_w, l_w, acc, lane);
    if (a.nbuf == 1 && s + 1 < nstages) {
      __syncthreads();  // single buffer: everyone is done with it before it is refilled
      if (warp == 0)
        issue_stage<ROWB>(a, Ku, Vu, lids, lpos, nle, s + 1, kv, kv + stage_bytes, &bar[0], lane);
    }
  }

  float o = 0.f, M = -INFINITY, l = 0.f;
  // From here on this CTA no longer reads its stage buffers from the stage loop; in the
  // cluster path announce it (the rank-0 CTA receives partials into those buffers once
  // every CTA of the cluster has arrived).
  if (CLUSTER && a.splits > 1) {
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  }
  if (failed) {
    // Give copies still in flight (the stage that timed out and the one after it) a
    // second bounded wait before the CTA's shared memory is released; the output of this
    // split is poisoned so the failure is visible besides the error word.
    // (the first nbuf stages are issued up front, stage s + 1 only after stage s's barrier)
    const int last_issued = min(max(failed_stage, a.nbuf - 1), nstages - 1);
    if (tid == 0) {
      for (int s = failed_stage; s <= last_issued; ++s) {
        const int buf = a.nbuf == 2 ? (s & 1) : 0;
        const uint32_t parity = (uint32_t)((a.nbuf == 2 ? (s >> 1) : s) & 1);
        mbar_wait_bounded(&bar[buf], parity, a.err, kDevErrTimeout, kWaitCycles);
      }
    }
    __syncthreads();
    o = __int_as_float(0x7fc00000);
    M = 0.f;
    l = __int_as_float(0x7fc00000);
  } else {
    // merge the four warps' states (the accumulators reuse the stage buffers: wait until
    // every warp is done with them)
    l_w = warp_sum(l_w);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < DPL; ++e) accr[warp * D + lane * DPL + e] = acc[e];
    if (lane == 0) {
      red[warp] = m_w;
      red[4 + warp] = l_w;
    }
    __syncthreads();
    if (tid < D) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, red[w]);
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float sw = red[w] == -INFINITY ? 0.f : exp2f(red[w] - M);
        o = fmaf(sw, accr[w * D + tid], o);
        l = fmaf(sw, red[4 + w], l);
      }
    }
  }

  if (a.splits == 1) {
    if (tid < D) {
      const float r = failed ? o : (l > 0.f ? o / l : 0.f);
      if (a.o_bf16)
        static_cast<uint16_t*>(a.O)[qg * D + tid] = f32_to_bf16_bits(r);
      else
        static_cast<float*>(a.O)[qg * D + tid] = r;
    }
  } else if (CLUSTER) {
    // every split sends (acc, max, sum) to the rank-0 CTA of its cluster, which merges
    cg::cluster_group cl = cg::this_cluster();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // all past their stages
    float* dst = cl.map_shared_rank(part, 0) + (size_t)split * (D + 2);
    if (tid < D) dst[tid] = o;
    if (tid == 0) {
      dst[D] = M;
      dst[D + 1] = l;
    }
    cl.sync();
    if (split == 0 && tid < D) {
      float MM = -INFINITY;
      for (int s = 0; s < a.splits; ++s) MM = fmaxf(MM, part[s * (D + 2) + D]);
      float num = 0.f, den = 0.f;
      for (int s = 0; s < a.splits; ++s) {
        const float ms = part[s * (D + 2) + D];
        const float w = ms == -INFINITY ? 0.f : exp2f(ms - MM);
        num = fmaf(w, part[s * (D + 2) + tid], num);
        den = fmaf(w, part[s * (D + 2) + D + 1], den);
      }
      const float r = den > 0.f ? num / den : (den == den ? 0.f : den);
      if (a.o_bf16)
        static_cast<uint16_t*>(a.O)[qg * D + tid] = f32_to_bf16_bits(r);
      else
        static_cast<float*>(a.O)[qg * D + tid] = r;
    }
  } else if (tid < D) {
    float* pp = a.partial + (qg * a.splits + split) * (D + 2);
    pp[tid] = o;
    if (tid == 0) {
      pp[D] = M;
      pp[D + 1] = l;
    }
  }
}

// Merge split partials: o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.  One warp per query.
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const float* partial, int splits, void* O,
                                                       int o_bf16, long long total_q) {
  constexpr int DPL = D / 32;
  const long long qg = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_release();
  if (qg >= total_q) return;
  const float* p = partial + qg * splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, p[s * (D + 2) + D]);
  float den = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* ps = p + s * (D + 2);
    const float ms = ps[D];
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
    den = fmaf(w, ps[D + 1], den);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, ps[lane * DPL + e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    const float r = den > 0.f ? acc[e] / den : (den == den ? 0.f : den);
    const long long o = qg * D + lane * DPL + e;
    if (o_bf16)
      static_cast<uint16_t*>(O)[o] = f32_to_bf16_bits(r);
    else
      static_cast<float*>(O)[o] = r;
  }
}

// Split plan (at most max_splits splits per query).  Stages of 16 KB (K + V rows) in two buffers, so about six CTAs fit on an
// SM; a query's leaves are split so the whole grid fills one wave of such CTAs (up to 8
// splits, merged inside a cluster).  Very few queries with long leaf lists use more
// splits, merged through caller scratch by combine_kernel.
AttnPlan plan_attention(const zha_tree* t, int q_heads, int nq, int beam, int max_splits) {
  AttnPlan p{};
  const int D = t->desc.head_dim;
  const int E = t->desc.kv_dtype == ZHA_BF16 ? 2 : 4;
  const int row = D * E;
  const long long lb = t->desc.leaf_block;
  const int ts_max = std::max(8, 16384 / (2 * row));
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  const long long tok = (long long)beam * lb;
  const size_t cta_smem = attn_smem_layout(D, row, 64, ts_max, 2, true).total + 1024;
  const long long per_sm = std::max<long long>(1, std::min<long long>(16, (227 * 1024) / cta_smem));
  const long long slots = per_sm * t->sms;
  const long long want = queries > 0 ? std::max(1LL, slots / queries) : 1;
  const long long maxs = std::max(1LL, std::min((long long)beam, (tok + lb - 1) / lb));
  long long splits = std::max(1LL, std::min(std::min(want, maxs), (long long)max_splits));
  p.cluster = splits > 1 && splits <= kMaxClusterSplits;
  int lps = (int)((beam + splits - 1) / splits);
  splits = (beam + lps - 1) / lps;
  if (splits <= 1) p.cluster = false;
  const long long item_tok = (long long)lps * lb;
  const int ts = (int)std::min<long long>(ts_max, (item_tok + 7) / 8 * 8);
  p.leaves_per_split = lps;
  p.splits = (int)splits;
  p.stage_tokens = ts;
  p.stages = item_tok > ts ? 2 : 1;
  p.smem_bytes = attn_smem_layout(D, row, lps, ts, p.stages, p.cluster).total;
  p.scratch_bytes = (splits > 1 && !p.cluster) ? (size_t)queries * splits * (D + 2) * sizeof(float) : 0;
  return p;
}

namespace {
template <typename TKV, int D, bool CLUSTER>
cudaError_t run_attend(const AttnArgs& a, const AttnPlan& plan, cudaStream_t s) {
  auto kern = attend_kernel<TKV, D, CLUSTER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)plan.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.total_items);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int nattr = 1;
  if (CLUSTER) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)plan.splits;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    nattr = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TKV, int D>
cudaError_t run_attend_any(const AttnArgs& a, const AttnPlan& plan, cudaStream_t s) {
  return plan.cluster ? run_attend<TKV, D, true>(a, plan, s) : run_attend<TKV, D, false>(a, plan, s);
}
}  // namespace

cudaError_t launch_attention(zha_tree* t, const AttnPlan& plan, const void* d_Q,
                             zha_dtype q_dtype, int q_heads, int nq, const void* d_K,
                             const void* d_V, const int* d_leaf_idx, int beam, float scale,
                             void* d_O, zha_dtype o_dtype, void* d_scratch, cudaStream_t stream) {
  const int D = t->desc.head_dim;
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  AttnArgs a{};
  a.Q = d_Q;
  a.q_bf16 = q_dtype == ZHA_BF16;
  a.K = static_cast<const char*>(d_K);
  a.V = static_cast<const char*>(d_V);
  a.kv_unit_stride = t->desc.capacity_tokens * D * (bf ? 2LL : 4LL);
  a.leaf_idx = d_leaf_idx;
  a.q_heads = q_heads;
  a.nq = nq;
  a.kv_heads = t->desc.kv_heads;
  a.group = q_heads / t->desc.kv_heads;
  a.beam = beam;
  a.lb = t->desc.leaf_block;
  a.N = t->N;
  a.n0 = t->n[0];
  a.qk_scale = scale * 1.4426950408889634f;
  a.lps = plan.leaves_per_split;
  a.splits = plan.splits;
  a.stage_tokens = plan.stage_tokens;
  a.nbuf = plan.stages;
  a.O = d_O;
  a.o_bf16 = o_dtype == ZHA_BF16;
  a.partial = static_cast<float*>(d_scratch);
  a.err = t->d_err;
  a.first_wait = first_wait_cycles(t);
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  a.total_items = queries * plan.splits;
  cudaError_t e;
  if (bf)
    e = D == 128 ? run_attend_any<uint16_t, 128>(a, plan, stream)
                 : run_attend_any<uint16_t, 64>(a, plan, stream);
  else
    e = D == 128 ? run_attend_any<float, 128>(a, plan, stream)
                 : run_attend_any<float, 64>(a, plan, stream);
  ++t->launches;
  if (e != cudaSuccess || plan.splits == 1 || plan.cluster) return e;
  const unsigned blocks = (unsigned)((queries + 3) / 4);
  if (D == 128)
    e = launch_pdl(combine_kernel<128>, dim3(blocks), dim3(128), 0, stream,
                   (const float*)a.partial, plan.splits, d_O, a.o_bf16, queries);
  else
    e = launch_pdl(combine_kernel<64>, dim3(blocks), dim3(128), 0, stream,
                   (const float*)a.partial, plan.splits, d_O, a.o_bf16, queries);
  ++t->launches;
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace zha

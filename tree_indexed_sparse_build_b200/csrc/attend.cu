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
// shared-memory stage, completing on an mbarrier; two stages alternate so the next
// copy overlaps this stage's arithmetic.  Each thread scores whole tokens from shared
// memory (16-byte chunks visited in a per-row rotated order, which keeps the eight
// lanes of a shared-memory phase on distinct banks), the block keeps a running max and
// sum in the log2 domain, and each lane accumulates head_dim/32 output dims over a
// quarter of the tokens.  A split writes (acc, m, l) partials to caller scratch and a
// second kernel combines them; a single split writes O directly.
//
// Every wait on an mbarrier is bounded by a clock budget; on expiry the kernel records
// kDevErrTimeout in the device error word and stops using the stage (no trap).
#include <algorithm>

#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 1.9 GHz

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
  float* partial;  // [queries][splits][D + 2]
  unsigned* err;
  long long total_items;
};

// Shared-memory layout, identical on host and device.
struct AttnSmem {
  size_t qs, red, meta, lids, lpos, sc, accr, kv, total;
};
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline AttnSmem attn_smem_layout(int D, int row_bytes, int lps, int stage_tokens,
                                                     int nbuf) {
  AttnSmem s;
  size_t o = 16;  // two mbarriers
  s.qs = o;
  o += (size_t)D * 4;
  s.red = o;
  o += 8 * 4;
  s.meta = o;
  o += 4 * 4;
  s.lids = o;
  o += (size_t)lps * 4;
  s.lpos = o;
  o += (size_t)(lps + 1) * 4;
  s.sc = align_up(o, 16);
  o = s.sc + (size_t)stage_tokens * 4;
  s.accr = align_up(o, 16);
  o = s.accr + (size_t)kAttnWarps * D * 4;
  s.kv = align_up(o, 128);
  s.total = s.kv + (size_t)nbuf * 2 * stage_tokens * row_bytes;
  return s;
}

template <int D>
__device__ __forceinline__ void load_v(const uint16_t* p, float* o) {
  if constexpr (D / 32 == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    o[0] = __uint_as_float(v.x << 16);
    o[1] = __uint_as_float(v.x & 0xFFFF0000u);
    o[2] = __uint_as_float(v.y << 16);
    o[3] = __uint_as_float(v.y & 0xFFFF0000u);
  } else {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    o[0] = __uint_as_float(v << 16);
    o[1] = __uint_as_float(v & 0xFFFF0000u);
  }
}
template <int D>
__device__ __forceinline__ void load_v(const float* p, float* o) {
  if constexpr (D / 32 == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x;
    o[1] = v.y;
    o[2] = v.z;
    o[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x;
    o[1] = v.y;
  }
}

// Issue the bulk copies of stage `s` (tokens [s*TS, s*TS + TS) of the work item's token
// sequence) into buffer `buf`.  Called by one thread.
template <int ROWB>
__device__ void issue_stage(const AttnArgs& a, const char* Ku, const char* Vu, const int* lids,
                            const int* lpos, int nle, int s, unsigned char* kbuf,
                            unsigned char* vbuf, uint64_t* bar) {
  const int TS = a.stage_tokens;
  const int total = lpos[nle];
  const int w0 = s * TS, w1 = min(w0 + TS, total);
  mbar_arrive_expect_tx(bar, (uint32_t)(2 * (w1 - w0) * ROWB));
  for (int j = 0; j < nle; ++j) {
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

template <typename TKV, int D>
__global__ void __launch_bounds__(kAttnThreads) attend_kernel(const AttnArgs a) {
  constexpr int E = sizeof(TKV);
  constexpr int ROWB = D * E;
  constexpr int VEC = 16 / E;
  constexpr int NCH = ROWB / 16;  // 16-byte chunks per row (power of two)
  constexpr int DPL = D / 32;     // output dims per lane
  static_assert((NCH & (NCH - 1)) == 0, "chunks per row must be a power of two");

  extern __shared__ __align__(128) unsigned char smem[];
  const AttnSmem L = attn_smem_layout(D, ROWB, a.lps, a.stage_tokens, a.nbuf);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* qs = reinterpret_cast<float*>(smem + L.qs);
  float* red = reinterpret_cast<float*>(smem + L.red);
  int* meta = reinterpret_cast<int*>(smem + L.meta);
  int* lids = reinterpret_cast<int*>(smem + L.lids);
  int* lpos = reinterpret_cast<int*>(smem + L.lpos);
  float* sc = reinterpret_cast<float*>(smem + L.sc);
  float* accr = reinterpret_cast<float*>(smem + L.accr);
  unsigned char* kv = smem + L.kv;
  const int TS = a.stage_tokens;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long item = blockIdx.x;
  const long long qg = item / a.splits;
  const int split = (int)(item - qg * a.splits);
  const long long hq_flat = qg / a.nq;
  const int h = (int)(hq_flat % a.q_heads);
  const long long unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
  const char* Ku = a.K + unit * a.kv_unit_stride;
  const char* Vu = a.V + unit * a.kv_unit_stride;

  if (tid == 0) {
    int cnt = 0, pos = 0;
    const int s0 = split * a.lps, s1 = min(s0 + a.lps, a.beam);
    const int* li = a.leaf_idx + qg * a.beam;
    for (int s = s0; s < s1; ++s) {
      const int j = li[s];
      if (j < 0) continue;
      if ((long long)j >= a.n0) {
        atomicOr(a.err, kDevErrBadLeaf);
        continue;
      }
      const long long t0 = (long long)j * a.lb;
      const long long t1 = min(t0 + a.lb, a.N);
      lids[cnt] = j;
      lpos[cnt] = pos;
      pos += (int)(t1 - t0);
      ++cnt;
    }
    lpos[cnt] = pos;
    meta[0] = cnt;
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  for (int d = tid; d < D; d += kAttnThreads) {
    const long long qi = qg * D + d;
    qs[d] = a.q_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[qi])
                     : static_cast<const float*>(a.Q)[qi];
  }
  __syncthreads();
  const int nle = meta[0];
  const int total = lpos[nle];
  const int nstages = (total + TS - 1) / TS;
  const size_t stage_bytes = (size_t)TS * ROWB;
  if (tid == 0) {
    for (int s = 0; s < min(a.nbuf, nstages); ++s)
      issue_stage<ROWB>(a, Ku, Vu, lids, lpos, nle, s, kv + (size_t)s * 2 * stage_bytes,
                        kv + (size_t)s * 2 * stage_bytes + stage_bytes, &bar[s]);
  }

  float m_run = -INFINITY, l_run = 0.f;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  bool failed = false;
  int failed_stage = 0;

  for (int s = 0; s < nstages; ++s) {
    const int buf = a.nbuf == 2 ? (s & 1) : 0;
    const uint32_t parity = (uint32_t)((a.nbuf == 2 ? (s >> 1) : s) & 1);
    const bool ok = mbar_wait_bounded(&bar[buf], parity, a.err, kDevErrTimeout, kWaitCycles);
    if (__syncthreads_or(!ok)) {
      failed = true;
      failed_stage = s;
      break;
    }
    const unsigned char* Ks = kv + (size_t)buf * 2 * stage_bytes;
    const unsigned char* Vs = Ks + stage_bytes;
    const int cnt = min(TS, total - s * TS);

    // scores
    float lmax = -INFINITY;
    for (int t = tid; t < cnt; t += kAttnThreads) {
      const unsigned char* row = Ks + (size_t)t * ROWB;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int cc = (c + t) & (NCH - 1);
        const uint4 v = *reinterpret_cast<const uint4*>(row + cc * 16);
        float f[VEC];
        Vec16<TKV>::to_f32(v, f);
        const float* qq = qs + cc * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dot = fmaf(qq[e], f[e], dot);
      }
      const float sv = dot * a.qk_scale;
      sc[t] = sv;
      lmax = fmaxf(lmax, sv);
    }
    lmax = warp_max(lmax);
    if (lane == 0) red[warp] = lmax;
    __syncthreads();
    lmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float m_new = fmaxf(m_run, lmax);
    const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
    float lsum = 0.f;
    for (int t = tid; t < cnt; t += kAttnThreads) {
      const float p = exp2f(sc[t] - m_new);
      sc[t] = p;
      lsum += p;
    }
    lsum = warp_sum(lsum);
    if (lane == 0) red[4 + warp] = lsum;
    __syncthreads();
    lsum = (red[4] + red[5]) + (red[6] + red[7]);
    l_run = l_run * alpha + lsum;
    m_run = m_new;

    // weighted V: this warp takes tokens t = warp, warp + 4, ...; this lane DPL dims
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] *= alpha;
    for (int t = warp; t < cnt; t += kAttnWarps) {
      const float p = sc[t];
      float v[DPL];
      load_v<D>(reinterpret_cast<const TKV*>(Vs + (size_t)t * ROWB) + lane * DPL, v);
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(p, v[e], acc[e]);
    }
    __syncthreads();  // every read of this buffer and of sc is done
    if (tid == 0 && s + a.nbuf < nstages) {
      fence_proxy_async_smem();
      issue_stage<ROWB>(a, Ku, Vu, lids, lpos, nle, s + a.nbuf, kv + (size_t)buf * 2 * stage_bytes,
                        kv + (size_t)buf * 2 * stage_bytes + stage_bytes, &bar[buf]);
    }
  }

  if (failed) {
    // Give copies still in flight (the stage that timed out and the one after it) a
    // second bounded wait before the CTA's shared memory is released, then poison the
    // output so the failure is visible besides the error word.
    if (tid == 0) {
      for (int s = failed_stage; s < min(failed_stage + a.nbuf, nstages); ++s) {
        const int buf = a.nbuf == 2 ? (s & 1) : 0;
        const uint32_t parity = (uint32_t)((a.nbuf == 2 ? (s >> 1) : s) & 1);
        mbar_wait_bounded(&bar[buf], parity, a.err, kDevErrTimeout, kWaitCycles);
      }
    }
    __syncthreads();
    if (tid < D) {
      const float nanv = __int_as_float(0x7fc00000);
      if (a.splits == 1) {
        if (a.o_bf16)
          static_cast<uint16_t*>(a.O)[qg * D + tid] = f32_to_bf16_bits(nanv);
        else
          static_cast<float*>(a.O)[qg * D + tid] = nanv;
      } else {
        float* pp = a.partial + (qg * a.splits + split) * (D + 2);
        pp[tid] = nanv;
        if (tid == 0) {
          pp[D] = 0.f;
          pp[D + 1] = nanv;
        }
      }
    }
    return;
  }

  // cross-warp reduction of the accumulators
#pragma unroll
  for (int e = 0; e < DPL; ++e) accr[warp * D + lane * DPL + e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) o += accr[w * D + tid];
    if (a.splits == 1) {
      const float r = l_run > 0.f ? o / l_run : 0.f;
      if (a.o_bf16)
        static_cast<uint16_t*>(a.O)[qg * D + tid] = f32_to_bf16_bits(r);
      else
        static_cast<float*>(a.O)[qg * D + tid] = r;
    } else {
      float* pp = a.partial + (qg * a.splits + split) * (D + 2);
      pp[tid] = o;
      if (tid == 0) {
        pp[D] = m_run;
        pp[D + 1] = l_run;
      }
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
    const float r = den > 0.f ? acc[e] / den : 0.f;
    const long long o = qg * D + lane * DPL + e;
    if (o_bf16)
      static_cast<uint16_t*>(O)[o] = f32_to_bf16_bits(r);
    else
      static_cast<float*>(O)[o] = r;
  }
}

AttnPlan plan_attention(const zha_tree* t, int q_heads, int nq, int beam) {
  AttnPlan p{};
  const int D = t->desc.head_dim;
  const int E = t->desc.kv_dtype == ZHA_BF16 ? 2 : 4;
  const int row = D * E;
  const long long lb = t->desc.leaf_block;
  const int ts_max = std::max(8, 32768 / (2 * row));
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  const long long tok = (long long)beam * lb;
  long long want = queries > 0 ? (2LL * t->sms + queries - 1) / queries : 1;
  const long long maxs = std::max(1LL, std::min((long long)beam, (tok + ts_max - 1) / ts_max));
  long long splits = std::max(1LL, std::min(want, maxs));
  const int lps = (int)((beam + splits - 1) / splits);
  splits = (beam + lps - 1) / lps;
  const long long item_tok = (long long)lps * lb;
  const int ts = (int)std::min<long long>(ts_max, (item_tok + 7) / 8 * 8);
  p.leaves_per_split = lps;
  p.splits = (int)splits;
  p.stage_tokens = ts;
  p.stages = item_tok > ts ? 2 : 1;
  p.smem_bytes = attn_smem_layout(D, row, lps, ts, p.stages).total;
  p.scratch_bytes = splits > 1 ? (size_t)queries * splits * (D + 2) * sizeof(float) : 0;
  return p;
}

namespace {
template <typename TKV, int D>
cudaError_t run_attend(const AttnArgs& a, const AttnPlan& plan, cudaStream_t s) {
  auto kern = attend_kernel<TKV, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)plan.smem_bytes);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)a.total_items, kAttnThreads, plan.smem_bytes, s>>>(a);
  return cudaGetLastError();
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
  const long long queries = (long long)t->desc.batch * q_heads * nq;
  a.total_items = queries * plan.splits;
  cudaError_t e;
  if (bf)
    e = D == 128 ? run_attend<uint16_t, 128>(a, plan, stream) : run_attend<uint16_t, 64>(a, plan, stream);
  else
    e = D == 128 ? run_attend<float, 128>(a, plan, stream) : run_attend<float, 64>(a, plan, stream);
  ++t->launches;
  if (e != cudaSuccess || plan.splits == 1) return e;
  const unsigned blocks = (unsigned)((queries + 3) / 4);
  if (D == 128)
    combine_kernel<128><<<blocks, 128, 0, stream>>>(a.partial, plan.splits, d_O, a.o_bf16, queries);
  else
    combine_kernel<64><<<blocks, 128, 0, stream>>>(a.partial, plan.splits, d_O, a.o_bf16, queries);
  ++t->launches;
  return cudaGetLastError();
}

}  // namespace zha

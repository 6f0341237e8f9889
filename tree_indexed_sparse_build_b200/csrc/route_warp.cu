// Warp-per-query routing (and route + attention) for launches with many queries.
//
// Top-down beam routing ("Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", abstract: future queries traverse the tree of key summaries from the top down
// to retrieve a sparse subset of keys, and the final attention runs over that subset).
//
// When a call carries many more queries than the GPU has SMs, throughput follows how many
// queries are in flight per SM.  The staged kernel (route_kernel.cuh) lands each level's
// candidate rows in shared memory, which caps residency at the rows one level needs per
// query (32 KB at 64 fp32 candidates of 128 dims: six queries per SM).  Here each warp owns
// one query and loads its candidate rows straight into registers, P row-passes at a time,
// so no shared memory is held across a level and the SM keeps sixteen queries in flight,
// each with 16 16-byte loads outstanding per lane.  Shared memory holds only the query's
// candidate ids, keys and survivors (under 1 KB per warp).
//
// Scoring follows the order all route kernels share (score_fma / score_reduce8,
// route_common.cuh: eight lanes per row, lane l8 takes 16-byte chunks l8 + 8 j), so scores,
// and therefore leaves, survivors and leaf scores, are bit-identical to the staged kernel's;
// q stays in registers (D / 8 floats per lane).  The selection is the same exact
// top-min(beam, C) over the packed (score, inverted node index) keys (select_warp).
//
// Attention (TKV = the K/V storage type): the query's warp reads its leaves' K and V rows
// straight from global memory and keeps an online softmax (attn_regs.cuh).
#include <algorithm>
#include <type_traits>

#include "attn_regs.cuh"
#include "device_common.cuh"
#include "route_common.cuh"
#include "zha_internal.h"

namespace zha {

namespace {

constexpr int kWarpCtaWarps = 8;  // warps (queries in flight) per CTA

// Per-warp shared memory: candidate keys [cmax], candidate ids [cmax], two survivor lists
// and the leaf scores [beam].
struct WarpSmem {
  size_t keys, cand, surv_a, surv_b, leaf_sc, total;
};
__host__ __device__ inline WarpSmem warp_smem_layout(int cmax, int beam) {
  WarpSmem s;
  size_t o = 0;
  s.keys = o;
  o += (size_t)cmax * 8;
  s.cand = o;
  o += (size_t)cmax * 4;
  s.surv_a = o;
  o += (size_t)beam * 4;
  s.surv_b = o;
  o += (size_t)beam * 4;
  s.leaf_sc = o;
  o += (size_t)beam * 4;
  s.total = route_align(o, 16);
  return s;
}

// Exact softmax attention of query qg over the tokens of its m leaves by one warp
// (attn_regs.cuh: every token in this warp's rounds, PP passes per round).
template <typename TKV, int D, int PP>
__device__ __forceinline__ void warp_attend(const int* leaves, int m, long long lb, long long N,
                                            const char* Ku, const char* Vu, const void* Q, bool q_bf16,
                                            long long qg, float qk_scale, void* O, bool o_bf16, int lane) {
  using A = RegAttn<TKV, D>;
  float qc[A::VEC];
  reg_attn_load_q<TKV, D>(Q, q_bf16, qg, lane, qc);
  const int total = leaf_token_count(leaves, m, lb, N);
  float m_w = -INFINITY, l_w = 0.f;
  float acc[A::VEC];
#pragma unroll
  for (int e = 0; e < A::VEC; ++e) acc[e] = 0.f;
  reg_attn_tokens<TKV, D, PP>(leaves, total, lb, Ku, Vu, qc, qk_scale, 0, 1, lane, m_w, l_w, acc);
  reg_attn_fold<TKV, D>(l_w, acc);
  if (lane < A::LPT) store_out(O, o_bf16, qg, D, lane * A::VEC, acc, l_w > 0.f ? 1.f / l_w : 0.f);
}

// One warp per query, queries qg = blockIdx.x * W + warp, then every gridDim.x * W further.
// P: row passes (4 rows each) whose loads are in flight together.
template <int D, typename TS, typename TKV, int P>
__global__ void __launch_bounds__(kWarpCtaWarps * 32, 2) route_warp_kernel(const RouteArgs a) {
  constexpr bool ATTEND = !std::is_same<TKV, NoKV>::value;
  constexpr int EPC = 16 / (int)sizeof(TS);       // summary elements per 16-byte chunk
  constexpr int CPL = D * (int)sizeof(TS) / 128;  // 16-byte chunks of a row per lane (8 lanes a row)
  extern __shared__ __align__(16) unsigned char wsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  const WarpSmem Ls = warp_smem_layout(a.cmax, a.beam);
  unsigned char* base = wsm + (size_t)warp * Ls.total;
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(base + Ls.keys);
  int* cand = reinterpret_cast<int*>(base + Ls.cand);
  int* surv_a = reinterpret_cast<int*>(base + Ls.surv_a);
  int* surv_b = reinterpret_cast<int*>(base + Ls.surv_b);
  float* leaf_sc = reinterpret_cast<float*>(base + Ls.leaf_sc);
  pdl_wait();
  pdl_release();

  // Levels with at most `beam` nodes below the root are kept whole (as in the staged kernel).
  int l_first = a.L - 1;
  while (l_first >= 1 && a.n[l_first] <= a.beam) --l_first;
  const int m_first = (int)a.n[l_first + 1];
  const int l8 = lane & 7, rg = lane >> 3;

  for (long long qg = (long long)blockIdx.x * W + warp; qg < a.total_queries; qg += (long long)gridDim.x * W) {
    const long long hq_flat = qg / a.nq;
    const int h = (int)(hq_flat % a.q_heads);
    const long long unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
    const TS* pyr_u = static_cast<const TS*>(a.pyr) + unit * a.pyr_unit_stride;
    float qv[CPL][EPC];
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
      for (int e = 0; e < EPC; ++e) qv[j][e] = load_elem(a.Q, a.q_bf16 != 0, qg * D + EPC * (l8 + 8 * j) + e);
    for (int k = lane; k < m_first; k += 32) surv_a[k] = k;
    if (a.trace)
      for (int l = l_first + 1; l < a.L; ++l) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < a.n[l] ? k : -1;
      }
    __syncwarp();
    int* cur = surv_a;
    int* nxt = surv_b;
    int m = m_first;
    for (int l = l_first; l >= 0; --l) {
      int C = 0;
      if (m > 0) {
        const long long last = cur[m - 1];
        C = (m - 1) * a.b + (int)min((long long)a.b, a.n[l] - (long long)a.b * last);
      }
      const TS* S = pyr_u + a.off[l] * D;
      for (int j = lane; j < m; j += 32) {  // survivor j's children are candidates j b ..
        const int node0 = a.b * cur[j];
        const int nc = min(a.b, C - j * a.b);
        for (int i = 0; i < nc; ++i) cand[j * a.b + i] = node0 + i;
      }
      __syncwarp();
      for (int r0 = 0; r0 < C; r0 += 4 * P) {  // rows r0 + 4 p + rg, P passes in flight
        uint4 v[P][CPL];
#pragma unroll
        for (int p = 0; p < P; ++p) {  // rows past C re-read the last candidate (not scored)
          const int r = min(r0 + 4 * p + rg, C - 1);
          const uint4* row = reinterpret_cast<const uint4*>(S + (size_t)cand[r] * D);
#pragma unroll
          for (int j = 0; j < CPL; ++j) v[p][j] = ldg16(row + l8 + 8 * j);
        }
        // Four passes at a time: each lane forms its partial of each pass's row, and one
        // transposed butterfly over the eight lanes of a row (distances 4, 2, 1) sums all
        // four rows with four shuffles.  The sums associate exactly as score_reduce8's, so
        // scores equal the other kernels' bit for bit.
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
          // lanes l8 < 4 keep passes 0, 1 and lanes l8 >= 4 passes 2, 3; bit 1 of l8 then
          // keeps one of the two, bit 0 pairs lanes holding the same row: lane l8 ends with
          // the sum of pass l8 / 2
          const bool hi4 = (l8 & 4) != 0, hi2 = (l8 & 2) != 0;
          const float send0 = hi4 ? part[0] : part[2], send1 = hi4 ? part[1] : part[3];
          const float keep0 = hi4 ? part[2] : part[0], keep1 = hi4 ? part[3] : part[1];
          const float b0 = keep0 + __shfl_xor_sync(0xffffffffu, send0, 4);
          const float b1 = keep1 + __shfl_xor_sync(0xffffffffu, send1, 4);
          float sc = (hi2 ? b1 : b0) + __shfl_xor_sync(0xffffffffu, hi2 ? b0 : b1, 2);
          sc += __shfl_xor_sync(0xffffffffu, sc, 1);
          const int r = r0 + 4 * (p4 + (l8 >> 1)) + rg;
          if ((l8 & 1) == 0 && r < C) keys[r] = route_key(sc, cand[r]);
        }
      }
      __syncwarp();
      const int kept = C > 0 ? select_warp(keys, cand, C, a.beam, lane, nxt, leaf_sc, l == 0) : 0;
      __syncwarp();
      if (a.trace) {
        int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
        for (int k = lane; k < a.beam; k += 32) tr[k] = k < kept ? nxt[k] : -1;
      }
      m = min(C, a.beam);
      int* tmp = cur;
      cur = nxt;
      nxt = tmp;
    }
    if (a.leaf_idx) {
      int* out = a.leaf_idx + qg * a.beam;
      for (int k = lane; k < a.beam; k += 32) out[k] = k < m ? cur[k] : -1;
    }
    if (a.leaf_score) {
      float* os = a.leaf_score + qg * a.beam;
      for (int k = lane; k < a.beam; k += 32) os[k] = k < m ? leaf_sc[k] : __int_as_float(0x7fc00000);
    }
    if constexpr (ATTEND) {
      if (a.O != nullptr) {
        constexpr int PP = 8;
        warp_attend<TKV, D, PP>(cur, m, a.lb, a.N, a.K + unit * a.kv_unit_stride, a.V + unit * a.kv_unit_stride,
                                a.Q, a.q_bf16 != 0, qg, a.qk_scale, a.O, a.o_bf16 != 0, lane);
      }
    }
    __syncwarp();  // the next query reuses this warp's shared memory
  }
}

template <int D, typename TS, typename TKV>
cudaError_t run_warp(const RouteArgs& a, int sms, cudaStream_t s) {
  constexpr int P = 16 / (D * (int)sizeof(TS) / 128);  // 16 row loads in flight per lane
  static_assert(P % 4 == 0, "passes go four at a time through the butterfly");
  auto kern = route_warp_kernel<D, TS, TKV, P>;
  const size_t smem = (size_t)kWarpCtaWarps * warp_smem_layout(a.cmax, a.beam).total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpCtaWarps * 32, smem);
  if (e != cudaSuccess) return e;
  const long long need = (a.total_queries + kWarpCtaWarps - 1) / kWarpCtaWarps;
  const unsigned blocks = (unsigned)std::max(1LL, std::min(need, (long long)std::max(per_sm, 1) * sms));
  e = launch_pdl(kern, dim3(blocks), dim3(kWarpCtaWarps * 32), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TS, typename TKV>
cudaError_t run_warp_d(int D, const RouteArgs& a, int sms, cudaStream_t s) {
  return D == 128 ? run_warp<128, TS, TKV>(a, sms, s) : run_warp<64, TS, TKV>(a, sms, s);
}

}  // namespace

bool route_warp_fits(const zha_tree* t, int cmax, int beam) {
  return (size_t)kWarpCtaWarps * warp_smem_layout(cmax, beam).total <= 96 * 1024 &&
         (long long)beam * t->desc.leaf_block <= kWarpMaxTokens;
}

cudaError_t launch_route_warp(zha_tree* t, const RouteArgs& a, bool attend, cudaStream_t s) {
  const int D = t->desc.head_dim;
  const bool s16 = sum_bf16(t);
  if (!attend)
    return s16 ? run_warp_d<uint16_t, NoKV>(D, a, t->sms, s) : run_warp_d<float, NoKV>(D, a, t->sms, s);
  if (t->desc.kv_dtype == ZHA_BF16)
    return s16 ? run_warp_d<uint16_t, uint16_t>(D, a, t->sms, s) : run_warp_d<float, uint16_t>(D, a, t->sms, s);
  return s16 ? run_warp_d<uint16_t, float>(D, a, t->sms, s) : run_warp_d<float, float>(D, a, t->sms, s);
}

}  // namespace zha

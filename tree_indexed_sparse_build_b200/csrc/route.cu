// Top-down beam routing ("Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", abstract: future queries traverse the tree of key summaries from the top
// down to retrieve a sparse subset of keys).
//
// Survivors start as {root}.  For l = L-1 .. 0 every existing child c of a survivor is
// scored by q . S_l[c] in fp32, and the top-min(beam, #candidates) are kept, ordered by
// score descending with the lower node index first on equal scores.
//
// GPU mapping: one warp per query.  Candidates are the children of the survivors, kept
// in ascending node order (survivors ascend, children of a node are contiguous), so
// candidate k belongs to survivor k / b.  Eight lanes read one 512-byte summary row
// (d = 128) with 16-byte loads, four rows per warp step and four steps in flight.  A
// candidate's key packs (order-preserving score bits, inverted node index) into 64 bits,
// so "greater key" is exactly "ranks first".  The B-th largest key is found by a 64-step
// binary search on the key bits with a warp-wide count per step (stopping early once
// exactly B keys remain), and the kept candidates are compacted with a ballot in
// candidate order, which keeps the survivors ascending without a sort.
#include <algorithm>

#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

constexpr int kRouteWarps = 4;

struct RouteArgs {
  const void* Q;
  int q_bf16;
  int q_heads, nq, group, kv_heads;
  const float* pyr;
  long long pyr_unit_stride;  // floats
  long long off[kMaxLevels];
  long long n[kMaxLevels];
  int L, b, beam, cmax;
  int warp_smem_words;  // 8-byte words of shared memory per warp
  int* leaf_idx;
  float* leaf_score;
  int* trace;
  long long total_queries;
};

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

template <int D>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(const RouteArgs a) {
  constexpr int NJ = D / 32;  // 16-byte chunks per lane per row
  constexpr int U = 4;        // warp steps (4 rows each) in flight
  extern __shared__ unsigned long long route_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long qg = (long long)blockIdx.x * kRouteWarps + warp;
  if (qg >= a.total_queries) return;  // no block-level barrier in this kernel

  unsigned long long* keys = route_smem + (size_t)warp * a.warp_smem_words;
  int* surv_a = reinterpret_cast<int*>(keys + a.cmax);
  int* surv_b = surv_a + a.beam;
  float* leaf_sc = reinterpret_cast<float*>(surv_b + a.beam);

  const long long hq_flat = qg / a.nq;  // b * q_heads + h
  const int h = (int)(hq_flat % a.q_heads);
  const long long bb = hq_flat / a.q_heads;
  const long long unit = bb * a.kv_heads + h / a.group;
  const int l8 = lane & 7, grp = lane >> 3;

  // This lane's slice of q: chunks c = l8 + 8j, dims 4c .. 4c+3.
  float q[NJ * 4];
  {
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

  const float* pyr_u = a.pyr + unit * a.pyr_unit_stride;
  if (lane == 0) surv_a[0] = 0;  // the root
  __syncwarp();
  int* cur = surv_a;
  int* nxt = surv_b;
  int m = 1;
  for (int l = a.L - 1; l >= 0; --l) {
    const long long nl = a.n[l];
    const long long last = cur[m - 1];
    const int nc_last = (int)min((long long)a.b, nl - (long long)a.b * last);
    const int C = (m - 1) * a.b + nc_last;
    const float* S = pyr_u + a.off[l] * D;

    for (int k0 = 0; k0 < C; k0 += 4 * U) {
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
    __syncwarp();

    // Threshold T = the beam-th largest key (0 keeps everything when C <= beam).
    unsigned long long T = 0ull;
    if (C > a.beam) {
      for (int bit = 63; bit >= 0; --bit) {
        const unsigned long long cand = T | (1ull << bit);
        unsigned cnt = 0;
        for (int k = lane; k < C; k += 32) cnt += keys[k] >= cand ? 1u : 0u;
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (cnt >= (unsigned)a.beam) {
          T = cand;
          if (cnt == (unsigned)a.beam) break;
        }
      }
    }
    // Ordered compaction of the kept candidates.
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
    m = base;
    if (a.trace) {
      int* tr = a.trace + (qg * a.L + (a.L - 1 - l)) * a.beam;
      for (int k = lane; k < a.beam; k += 32) tr[k] = k < m ? nxt[k] : -1;
    }
    int* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  int* out = a.leaf_idx + qg * a.beam;
  for (int k = lane; k < a.beam; k += 32) out[k] = k < m ? cur[k] : -1;
  if (a.leaf_score) {
    float* os = a.leaf_score + qg * a.beam;
    for (int k = lane; k < a.beam; k += 32) os[k] = k < m ? leaf_sc[k] : __int_as_float(0x7fc00000);
  }
}

cudaError_t launch_route(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads,
                         int nq, int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                         cudaStream_t stream) {
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
  // keys (8 B each) + two survivor lists (4 B) + leaf scores (4 B), rounded to 8 B words
  const long long words = cmax + (3LL * beam * 4 + 7) / 8;
  a.warp_smem_words = (int)words;
  a.leaf_idx = d_leaf_idx;
  a.leaf_score = d_leaf_score;
  a.trace = d_trace;
  a.total_queries = (long long)t->desc.batch * q_heads * nq;
  const size_t smem = (size_t)words * 8 * kRouteWarps;
  const long long blocks = (a.total_queries + kRouteWarps - 1) / kRouteWarps;
  cudaError_t e;
  if (D == 128) {
    e = cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_kernel<128><<<(unsigned)blocks, kRouteWarps * 32, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_kernel<64><<<(unsigned)blocks, kRouteWarps * 32, smem, stream>>>(a);
  }
  ++t->launches;
  return cudaGetLastError();
}

}  // namespace zha

// Threshold (halfspace) descent with bounding spheres ("Louver" explainer: sparse attention
// as exact retrieval of every key whose score reaches a threshold tau, i.e. every key in
// the halfspace {p : q . p >= tau}; clusters of keys enclosed in bounding spheres are pruned
// when the sphere misses the halfspace and the keys of the others are checked exactly, so
// no key is missed).  On this tree: the spheres of radii.cu (centers = the stored
// summaries); survivors start as {root}; for l = L-1 .. 0 a child of a survivor is kept iff
// q . c + ||q|| r >= tau; the tokens of the surviving leaves are then checked exactly.
//
// Arithmetic: q . c and q . k in fp64 from the stored values (exact products); a sphere is
// pruned only when its bound is below tau by more than 1e-9 of the magnitudes involved, so
// rounding can only keep a sphere, never lose a key.  The token check is exact in fp64.
//
// GPU mapping: one CTA of 8 warps per query.  The survivors of a level live in shared
// memory (at most kFrontierCap); the children of the survivors are tested in chunks of
// kChunk candidates, one thread per candidate row: the thread sums its row's products in
// dim order with fp64 FMAs against q held in shared memory (fp64, read as a broadcast), so
// no cross-lane reduction is needed; and since a product of a stored element (bf16 or fp32)
// and a q element is exact in fp64, that sum is bit for bit the plain sequential fp64 sum.
// The kept ones are compacted in candidate order by a block-wide prefix sum, so survivors
// and the tokens found stay ascending.  The leaves' tokens go through the same chunked test.
#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

namespace {

constexpr int kThThreads = 256;
constexpr int kThWarps = kThThreads / 32;
constexpr int kChunk = 1024;        // candidates per chunk (4 per thread in the compaction)
constexpr int kFrontierCap = 8192;  // survivors of one level a query may keep

struct ThreshArgs {
  const void* Q;
  int q_bf16;
  int q_heads, nq, group, kv_heads;
  const void* pyr;            // summaries (fp32 or bf16, the kernel's TS)
  long long pyr_unit_stride;  // elements
  const float* radii;
  long long off[kMaxLevels];
  long long n[kMaxLevels];
  int L, b;
  long long lb, N;
  const char* K;
  long long k_unit_stride;  // bytes
  const float* tau;         // [queries]
  int max_tokens;
  int* tokens;              // [queries][max_tokens]
  int* count;               // [queries]
  int* stats;               // [queries][2], nullable: spheres tested, tokens checked
  long long total_queries;
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// dot = sum over dims e in order of q[e] * row[e], and (MAG) mag = sum of |q[e] * row[e]|, in
// fp64 by one thread: the row read in 16-byte pieces (four in flight), q from shared memory.
template <typename T, int D, bool MAG>
__device__ __forceinline__ void row_dot(const T* row, const double* q, double& dot, double& mag) {
  constexpr int EPC = Vec16<T>::N;
  dot = 0.0;
  mag = 0.0;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 4 * EPC) {
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = ldg16(row + c0 + i * EPC);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float f[EPC];
      Vec16<T>::to_f32(v[i], f);
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        const double qe = q[c0 + i * EPC + e], x = (double)f[e];
        dot = fma(qe, x, dot);
        if (MAG) mag += fabs(qe * x);
      }
    }
  }
}

// Block-wide ordered compaction of one chunk: flags[i] (i < n) -> positions base + prefix.
// Returns the number of set flags.  pos receives each kept item's rank (or -1).
__device__ int chunk_compact(const unsigned char* flags, int n, int* pos, int* wsum) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int c = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) c += (4 * t + i < n && flags[4 * t + i]) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kThWarps; ++w) {
    if (w < warp) before += wsum[w];
    total += wsum[w];
  }
  int p = before + incl - c;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = 4 * t + i;
    if (k < n) pos[k] = flags[k] ? p++ : -1;
  }
  __syncthreads();
  return total;
}

template <typename TK, typename TS, int D>
__global__ void __launch_bounds__(kThThreads) threshold_kernel(const ThreshArgs a) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(16) unsigned char tsm[];
  int* fa = reinterpret_cast<int*>(tsm);
  int* fb = fa + kFrontierCap;
  int* pos = fb + kFrontierCap;                                     // [kChunk]
  unsigned char* flags = reinterpret_cast<unsigned char*>(pos + kChunk);  // [kChunk]
  int* wsum = reinterpret_cast<int*>(flags + kChunk);               // [kThWarps]
  double* qs = reinterpret_cast<double*>(wsum + kThWarps + 4);      // [D], 16-byte aligned
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const long long qg = blockIdx.x;
  pdl_wait();
  pdl_release();
  if (qg >= a.total_queries) return;
  const long long hq_flat = qg / a.nq;
  const int h = (int)(hq_flat % a.q_heads);
  const long long unit = (hq_flat / a.q_heads) * a.kv_heads + h / a.group;
  const TS* pu = static_cast<const TS*>(a.pyr) + unit * a.pyr_unit_stride;
  const float* ru = a.radii + unit * (a.pyr_unit_stride / D);
  const TK* Ku = reinterpret_cast<const TK*>(a.K + unit * a.k_unit_stride);
  const double tau = (double)a.tau[qg];

  // this lane's dims of q, and ||q||
  double qv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    const long long at = qg * D + lane * DPL + e;
    qv[e] = a.q_bf16 ? (double)bf16_bits_to_f32(static_cast<const uint16_t*>(a.Q)[at])
                     : (double)static_cast<const float*>(a.Q)[at];
  }
  double qn = 0.0;
#pragma unroll
  for (int e = 0; e < DPL; ++e) qn = fma(qv[e], qv[e], qn);
  qn = sqrt(warp_sum_d(qn));
  if (warp == 0)
#pragma unroll
    for (int e = 0; e < DPL; ++e) qs[lane * DPL + e] = qv[e];

  int* cur = fa;
  int* nxt = fb;
  if (t == 0) cur[0] = 0;  // the root
  int m = 1;
  long long tested = 0, checked = 0;
  bool overflow = false;
  __syncthreads();
  for (int l = a.L - 1; l >= 0 && !overflow; --l) {
    const long long total = (long long)m * a.b;  // child slots of the survivors
    const TS* S = pu + a.off[l] * D;
    const float* R = ru + a.off[l];
    int mn = 0;
    for (long long c0 = 0; c0 < total; c0 += kChunk) {
      const int n = (int)min((long long)kChunk, total - c0);
      for (int k = t; k < n; k += kThThreads) {  // one candidate row per thread
        const long long slot = c0 + k;
        const long long node = (long long)a.b * cur[slot / a.b] + slot % a.b;
        bool keep = false;
        if (node < a.n[l]) {
          double dot, mag;
          row_dot<TS, D, true>(S + node * D, qs, dot, mag);
          const double rq = qn * (double)R[node];
          keep = dot + rq >= tau - 1e-9 * (mag + rq + fabs(tau));
        }
        flags[k] = keep ? 1 : 0;
      }
      __syncthreads();
      const int kept = chunk_compact(flags, n, pos, wsum);
      if (mn + kept > kFrontierCap) {
        overflow = true;
        break;
      }
      for (int k = t; k < n; k += kThThreads)
        if (pos[k] >= 0) {
          const long long slot = c0 + k;
          nxt[mn + pos[k]] = (int)((long long)a.b * cur[slot / a.b] + slot % a.b);
        }
      mn += kept;
      __syncthreads();
    }
    if (m > 0)  // spheres tested: only the last survivor can have fewer than b children
      tested += (long long)(m - 1) * a.b + min((long long)a.b, a.n[l] - (long long)a.b * cur[m - 1]);
    int* tmp = cur;
    cur = nxt;
    nxt = tmp;
    m = mn;
    __syncthreads();
  }

  int found = 0;
  int* out = a.tokens + qg * a.max_tokens;
  if (!overflow) {
    // the tokens of the surviving leaves, in order
    const long long total = (long long)m * a.lb;
    for (long long c0 = 0; c0 < total; c0 += kChunk) {
      const int n = (int)min((long long)kChunk, total - c0);
      for (int k = t; k < n; k += kThThreads) {  // one token per thread
        const long long slot = c0 + k;
        const long long tok = (long long)cur[slot / a.lb] * a.lb + slot % a.lb;
        bool keep = false;
        if (tok < a.N) {
          double dot, mag;
          row_dot<TK, D, false>(Ku + tok * D, qs, dot, mag);
          keep = dot >= tau;
        }
        flags[k] = keep ? 1 : 0;
      }
      __syncthreads();
      const int kept = chunk_compact(flags, n, pos, wsum);
      for (int k = t; k < n; k += kThThreads)
        if (pos[k] >= 0 && found + pos[k] < a.max_tokens) {
          const long long slot = c0 + k;
          out[found + pos[k]] = (int)((long long)cur[slot / a.lb] * a.lb + slot % a.lb);
        }
      found += kept;
      __syncthreads();
    }
    if (m > 0)  // tokens checked: only leaf n0 - 1 can be short, and it can only be last
      checked = (long long)(m - 1) * a.lb + (min((long long)cur[m - 1] * a.lb + a.lb, a.N) - (long long)cur[m - 1] * a.lb);
  }
  for (int k = (overflow ? 0 : found) + t; k < a.max_tokens; k += kThThreads) out[k] = -1;
  if (t == 0) {
    a.count[qg] = overflow ? -1 : found;
    if (a.stats) {
      a.stats[qg * 2] = (int)tested;
      a.stats[qg * 2 + 1] = (int)checked;
    }
  }
}

template <typename TK, typename TS, int D>
cudaError_t run_threshold(const ThreshArgs& a, size_t smem, cudaStream_t s) {
  auto kern = threshold_kernel<TK, TS, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)a.total_queries), dim3(kThThreads), smem, s, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_threshold(zha_tree* t, const void* d_K, const void* d_Q, zha_dtype q_dtype, int q_heads,
                             int nq, const float* d_tau, int max_tokens, int* d_tokens, int* d_count,
                             int* d_stats, cudaStream_t stream) {
  ThreshArgs a{};
  const int D = t->desc.head_dim;
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  const bool sbf = sum_bf16(t);
  a.Q = d_Q;
  a.q_bf16 = q_dtype == ZHA_BF16;
  a.q_heads = q_heads;
  a.nq = nq;
  a.kv_heads = t->desc.kv_heads;
  a.group = q_heads / t->desc.kv_heads;
  a.pyr = t->pyr;
  a.pyr_unit_stride = t->unit_rows * D;
  a.radii = t->radii;
  for (int l = 0; l <= t->L; ++l) {
    a.off[l] = t->off[l];
    a.n[l] = t->n[l];
  }
  a.L = t->L;
  a.b = t->desc.branching;
  a.lb = t->desc.leaf_block;
  a.N = t->N;
  a.K = static_cast<const char*>(d_K);
  a.k_unit_stride = t->desc.capacity_tokens * D * (bf ? 2LL : 4LL);
  a.tau = d_tau;
  a.max_tokens = max_tokens;
  a.tokens = d_tokens;
  a.count = d_count;
  a.stats = d_stats;
  a.total_queries = (long long)t->desc.batch * q_heads * nq;
  const size_t smem = (size_t)2 * kFrontierCap * 4 + kChunk * 4 + kChunk + kThWarps * 4 + 16 + (size_t)D * 8;
  cudaError_t e;
  if (sbf)
    e = bf ? (D == 128 ? run_threshold<uint16_t, uint16_t, 128>(a, smem, stream)
                       : run_threshold<uint16_t, uint16_t, 64>(a, smem, stream))
           : (D == 128 ? run_threshold<float, uint16_t, 128>(a, smem, stream)
                       : run_threshold<float, uint16_t, 64>(a, smem, stream));
  else
    e = bf ? (D == 128 ? run_threshold<uint16_t, float, 128>(a, smem, stream)
                       : run_threshold<uint16_t, float, 64>(a, smem, stream))
           : (D == 128 ? run_threshold<float, float, 128>(a, smem, stream)
                       : run_threshold<float, float, 64>(a, smem, stream));
  ++t->launches;
  return e;
}

}  // namespace zha

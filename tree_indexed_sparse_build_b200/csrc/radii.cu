// Bounding-sphere radii of the tree's nodes ("Louver" explainer, index design: every cluster
// of keys is enclosed in a bounding sphere, a center and a radius, so a query can prune the
// clusters whose sphere misses its halfspace {p : q . p >= tau}).  The center of a node is
// its stored summary (fp32 or bf16); the radius covers every key of its subtree:
//   leaf i:  r = max over its tokens t < N of ||k_t - c_i||
//   node i:  r = max over its existing children j of (||c_j - c_i|| + r_j)
// (a child's sphere lies inside the ball of radius ||c_j - c_i|| + r_j around c_i).
// Distances are formed in fp64 from the stored values and rounded up to fp32 with a
// relative margin of 1e-12, so a stored radius is never below the true one.
//
// One warp per node; each lane holds head_dim / 32 dims.  Leaves [lo, hi] of every unit,
// then each level's ancestors of that range, one launch per level.
#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

namespace {

constexpr int kRadThreads = 256;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float radius_up(double r) { return __double2float_ru(r * (1.0 + 1e-12)); }

template <typename TK, typename TS, int D>
__global__ void __launch_bounds__(kRadThreads) radius_leaf_kernel(const char* K, long long k_unit_stride,
                                                                  const void* pyr, long long pyr_unit_stride,
                                                                  float* radii, long long off0, long long lo,
                                                                  long long count, long long units,
                                                                  long long N, long long lb) {
  constexpr int DPL = D / 32;
  const long long w = ((long long)blockIdx.x * kRadThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_release();
  if (w >= units * count) return;
  const long long unit = w / count, i = lo + (w - unit * count);
  const TS* c = static_cast<const TS*>(pyr) + unit * pyr_unit_stride + (off0 + i) * D;
  const TK* Ku = reinterpret_cast<const TK*>(K + unit * k_unit_stride);
  double cv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) cv[e] = (double)SumT<TS>::load(c[lane * DPL + e]);
  const long long t0 = i * lb, t1 = min(t0 + lb, N);
  double best = 0.0;
  for (long long t = t0; t < t1; ++t) {
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      double k;
      if constexpr (sizeof(TK) == 2)
        k = (double)bf16_bits_to_f32(Ku[t * D + lane * DPL + e]);
      else
        k = (double)Ku[t * D + lane * DPL + e];
      const double x = k - cv[e];
      s = fma(x, x, s);
    }
    s = warp_sum_d(s);
    best = fmax(best, s);
  }
  if (lane == 0) radii[unit * pyr_unit_stride / D + off0 + i] = radius_up(sqrt(best));
}

template <typename TS, int D>
__global__ void __launch_bounds__(kRadThreads) radius_level_kernel(const void* pyr, long long pyr_unit_stride,
                                                                   float* radii, long long off_l,
                                                                   long long off_c, long long lo,
                                                                   long long count, long long units,
                                                                   long long n_child, int b) {
  constexpr int DPL = D / 32;
  const long long w = ((long long)blockIdx.x * kRadThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_release();
  if (w >= units * count) return;
  const long long unit = w / count, i = lo + (w - unit * count);
  const TS* pu = static_cast<const TS*>(pyr) + unit * pyr_unit_stride;
  const float* ru = radii + unit * (pyr_unit_stride / D);
  double cv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) cv[e] = (double)SumT<TS>::load(pu[(off_l + i) * D + lane * DPL + e]);
  const long long j0 = i * b, j1 = min(j0 + (long long)b, n_child);
  double best = 0.0;
  for (long long j = j0; j < j1; ++j) {
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      const double x = (double)SumT<TS>::load(pu[(off_c + j) * D + lane * DPL + e]) - cv[e];
      s = fma(x, x, s);
    }
    s = warp_sum_d(s);
    best = fmax(best, sqrt(s) + (double)ru[off_c + j]);
  }
  if (lane == 0) radii[unit * (pyr_unit_stride / D) + off_l + i] = radius_up(best);
}

unsigned grid_for(long long warps) { return (unsigned)((warps * 32 + kRadThreads - 1) / kRadThreads); }

template <typename TK, typename TS, int D>
cudaError_t radii_levels(zha_tree* t, const char* K, long long lo, long long hi, cudaStream_t s) {
  const long long k_stride = t->desc.capacity_tokens * D * (long long)sizeof(TK);
  const long long stride = t->unit_rows * D;
  const long long units = t->units;
  long long cnt = hi - lo + 1;
  cudaError_t e = launch_pdl(radius_leaf_kernel<TK, TS, D>, dim3(grid_for(units * cnt)), dim3(kRadThreads), 0, s,
                             K, k_stride, (const void*)t->pyr, stride, t->radii, t->off[0], lo, cnt, units, t->N,
                             (long long)t->desc.leaf_block);
  ++t->launches;
  if (e != cudaSuccess) return e;
  const int b = t->desc.branching;
  for (int l = 1; l <= t->L; ++l) {
    lo /= b;
    hi /= b;
    cnt = hi - lo + 1;
    e = launch_pdl(radius_level_kernel<TS, D>, dim3(grid_for(units * cnt)), dim3(kRadThreads), 0, s,
                   (const void*)t->pyr, stride, t->radii, t->off[l], t->off[l - 1], lo, cnt, units, t->n[l - 1], b);
    ++t->launches;
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <typename TK, typename TS>
cudaError_t radii_d(zha_tree* t, const char* K, long long lo, long long hi, cudaStream_t s) {
  return t->desc.head_dim == 128 ? radii_levels<TK, TS, 128>(t, K, lo, hi, s)
                                 : radii_levels<TK, TS, 64>(t, K, lo, hi, s);
}

}  // namespace

cudaError_t launch_radii(zha_tree* t, const void* d_K, long long lo, long long hi, cudaStream_t s) {
  if (!t->radii || t->N == 0 || hi < lo) return cudaSuccess;
  const char* K = static_cast<const char*>(d_K);
  const bool bf = t->desc.kv_dtype == ZHA_BF16;
  if (sum_bf16(t))
    return bf ? radii_d<uint16_t, uint16_t>(t, K, lo, hi, s) : radii_d<float, uint16_t>(t, K, lo, hi, s);
  return bf ? radii_d<uint16_t, float>(t, K, lo, hi, s) : radii_d<float, float>(t, K, lo, hi, s);
}

}  // namespace zha

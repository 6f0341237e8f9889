// Summary pyramid: leaf means over leaf blocks of K, then unweighted means of the
// existing children, level by level up to the root ("Subquadratic Attention with a
// Hierarchical Tree-Structured Indexer", abstract: recursively compressed key summaries
// over the KV cache; the tree deepens as the cache grows).
//
// One launch ("pass") computes a first level from its source rows (K tokens for the
// leaves, or the stored level below) and up to k further levels above it inside the CTA.
// A CTA owns `chunk` consecutive first-level nodes, a multiple of b^k, so the k upper
// levels of its subtree need no other CTA.  Sums are formed in fp64 and kept in shared
// memory in fp64 between the levels of a pass; each level is rounded once when stored
// (fp32 storage), or to fp32 and then bf16 (bf16 storage, where the kept fp64 value is the
// stored one, so a parent always averages its children's stored values; SumT in
// device_common.cuh).  Only nodes inside the touched range [lo, hi] of each level are
// recomputed; the others are read back from the pyramid (append).
//
// Memory: the first pass streams K once with 16-byte coalesced loads (a row of
// head_dim elements is read by LPR consecutive lanes, one node per lane group, 8 rows
// in flight per lane) and writes each summary row once.
#include <algorithm>

#include "device_common.cuh"
#include "zha_internal.h"

namespace zha {

constexpr int kPassThreads = 256;
constexpr int kMaxPassLevels = 8;  // first level + up to 7 above it in one CTA
constexpr int kChunkTarget = 16;   // at least this many first-level nodes per CTA
constexpr int kChunkMaxPow = 32;   // b^k <= 32 bounds the CTA's fp64 shared memory

struct PassArgs {
  const char* src;                    // unit 0, row 0 of the source level
  long long src_unit_stride;          // bytes between units
  long long n_src;                    // rows present at the source level
  long long blk0;                     // source rows per first-level node
  int b;
  int k;                              // levels above the first, inside the CTA
  int chunk;                          // first-level nodes per CTA (multiple of b^k)
  void* pyr;                          // unit 0 of the pyramid (summary storage type)
  long long pyr_unit_stride;          // elements between units
  long long lvl_off[kMaxPassLevels];  // row offset of the pass's level m inside a unit
  long long lvl_n[kMaxPassLevels];    // nodes at level m
  long long lo[kMaxPassLevels];       // touched range at level m (inclusive)
  long long hi[kMaxPassLevels];
  long long chunk0;                   // chunk index of blockIdx.x == 0
};

// VEC consecutive stored elements from registers (16- or 8-byte stores).
template <typename TS, int VEC>
__device__ __forceinline__ void store_piece(TS* dst, const TS* v) {
  constexpr int BYTES = VEC * (int)sizeof(TS);
  if constexpr (BYTES % 16 == 0) {
#pragma unroll
    for (int c = 0; c < BYTES / 16; ++c) reinterpret_cast<uint4*>(dst)[c] = reinterpret_cast<const uint4*>(v)[c];
  } else {
    static_assert(BYTES == 8, "4 bf16 values");
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(v);
  }
}

// TIn: the source rows' type (K's, or the summaries' for the upper passes); TS: summaries.
template <typename TIn, typename TS, int D>
__global__ void __launch_bounds__(kPassThreads) pyramid_pass_kernel(const PassArgs a) {
  constexpr int VEC = Vec16<TIn>::N;  // elements per 16-byte load
  constexpr int LPR = D / VEC;        // lanes covering one row
  constexpr int SPW = 32 / LPR;       // node slots per warp
  constexpr int SLOTS = (kPassThreads / 32) * SPW;
  constexpr long long ROWB = (long long)D * sizeof(TIn);
  static_assert(LPR <= 32 && 32 % LPR == 0, "row must split evenly over a warp");

  extern __shared__ double smem_d[];
  pdl_wait();
  pdl_release();
  double* bufA = smem_d;                        // [chunk][D]
  double* bufB = smem_d + (size_t)a.chunk * D;  // [chunk / b][D]

  const int unit = blockIdx.y;
  const long long chunk = a.chunk0 + blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp * SPW + lane / LPR;
  const int col = (lane % LPR) * VEC;
  const char* src = a.src + (long long)unit * a.src_unit_stride + (long long)col * sizeof(TIn);
  TS* pyr_u = static_cast<TS*>(a.pyr) + (long long)unit * a.pyr_unit_stride;

  // ---- first level of the pass: one node per lane group
  const long long base0 = chunk * a.chunk;
  for (int j = slot; j < a.chunk; j += SLOTS) {
    const long long i = base0 + j;
    if (i >= a.lvl_n[0]) break;  // nodes ascend with j
    TS* dst = pyr_u + (a.lvl_off[0] + i) * D + col;
    double* sm = bufA + (size_t)j * D + col;
    if (i >= a.lo[0] && i <= a.hi[0]) {
      const long long r0 = i * a.blk0;
      const long long r1 = min(r0 + a.blk0, a.n_src);
      const long long nrows = r1 - r0;
      const char* p = src + r0 * ROWB;
      double acc[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
      long long r = 0;
      for (; r + 8 <= nrows; r += 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = ldg16(p + (r + u) * ROWB);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float f[VEC];
          Vec16<TIn>::to_f32(v[u], f);
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += (double)f[e];
        }
      }
      for (; r < nrows; ++r) {
        float f[VEC];
        Vec16<TIn>::to_f32(ldg16(p + r * ROWB), f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += (double)f[e];
      }
      const double cnt = (double)nrows;
      alignas(16) TS out[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const double v = acc[e] / cnt;
        out[e] = SumT<TS>::store(v);
        sm[e] = SumT<TS>::kept(v);
      }
      store_piece<TS, VEC>(dst, out);
    } else {
#pragma unroll
      for (int e = 0; e < VEC; ++e) sm[e] = (double)SumT<TS>::load(dst[e]);
    }
  }
  __syncthreads();

  // ---- upper levels of the pass, fp64 in shared memory (ping-pong A/B)
  double* cur = bufA;
  double* nxt = bufB;
  int child_nodes = a.chunk;  // nodes of level m-1 owned by this CTA
  for (int m = 1; m <= a.k; ++m) {
    const int nn = child_nodes / a.b;
    const long long basem = chunk * nn;   // first node of level m owned by this CTA
    const long long basec = basem * a.b;  // its first child
    for (int idx = threadIdx.x; idx < nn * D; idx += kPassThreads) {
      const int j = idx / D, e = idx - (idx / D) * D;
      const long long i = basem + j;
      if (i >= a.lvl_n[m]) continue;
      double v;
      TS* dst = pyr_u + (a.lvl_off[m] + i) * D + e;
      if (i >= a.lo[m] && i <= a.hi[m]) {
        const long long c0 = i * a.b;
        const long long c1 = min(c0 + (long long)a.b, a.lvl_n[m - 1]);
        double s = 0.0;
        for (long long c = c0; c < c1; ++c) s += cur[(size_t)(c - basec) * D + e];
        const double mean = s / (double)(c1 - c0);
        *dst = SumT<TS>::store(mean);
        v = SumT<TS>::kept(mean);
      } else {
        v = (double)SumT<TS>::load(*dst);
      }
      nxt[(size_t)j * D + e] = v;
    }
    __syncthreads();
    double* tmp = cur;
    cur = nxt;
    nxt = tmp;
    child_nodes = nn;
  }
}

// Small appends in one launch.  One CTA per unit stages, with 1-D bulk copies (TMA) on
// one mbarrier, everything the touched path needs: the tokens of the touched leaves
// [lo, hi] (one contiguous run) and, for every level l >= 1, the stored children of the
// touched nodes (one contiguous run per level).  It then recomputes the leaves in fp64
// and walks up: a touched node averages its existing children, taking touched children
// from the fp64 values just computed and the others from the staged rows.  One memory
// round trip for the whole path.  Used when hi - lo + 1 <= kPathMaxLeaves and the staged
// rows fit in shared memory.
constexpr int kPathMaxLeaves = 8;
constexpr int kPathThreads = 256;
constexpr size_t kPathSmemCap = 160 * 1024;
constexpr long long kPathWaitCycles = kCopyWaitCycles;

struct AppendPathArgs {
  const char* K;               // unit 0, token 0
  long long k_unit_stride;     // bytes between units
  long long N, lb;
  int b, L;
  void* pyr;
  long long pyr_unit_stride;   // elements
  long long off[kMaxLevels];
  long long n[kMaxLevels];
  long long lo, hi;            // touched leaves
  long long sib0[kMaxLevels];  // first staged child row at level l - 1, for l >= 1
  int sib_rows[kMaxLevels];    // staged child rows for level l
  int sib_off[kMaxLevels];     // byte offset of those rows in shared memory
  int tok_rows;                // staged token rows
  int fp64_off;                // byte offset of the two fp64 node buffers
  int bar_off;
  unsigned* err;
  long long first_wait;        // bound of the first wait for the copies
};

template <typename TIn, typename TS, int D>
__global__ void __launch_bounds__(kPathThreads) append_path_kernel(const AppendPathArgs a) {
  extern __shared__ __align__(128) unsigned char psm[];
  const int unit = blockIdx.x;
  const char* Ku = a.K + (long long)unit * a.k_unit_stride;
  TS* pyr_u = static_cast<TS*>(a.pyr) + (long long)unit * a.pyr_unit_stride;
  const TIn* tok = reinterpret_cast<const TIn*>(psm);
  double* cur = reinterpret_cast<double*>(psm + a.fp64_off);
  double* nxt = cur + kPathMaxLeaves * D;
  uint64_t* bar = reinterpret_cast<uint64_t*>(psm + a.bar_off);
  pdl_wait();
  pdl_release();

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    uint32_t bytes = (uint32_t)a.tok_rows * D * sizeof(TIn);
    for (int l = 1; l <= a.L; ++l) bytes += (uint32_t)a.sib_rows[l] * D * (uint32_t)sizeof(TS);
    mbar_arrive_expect_tx(bar, bytes);
    const long long r0 = a.lo * a.lb;
    bulk_copy_g2s(psm, Ku + r0 * D * (long long)sizeof(TIn), (uint32_t)a.tok_rows * D * sizeof(TIn), bar);
    for (int l = 1; l <= a.L; ++l)
      if (a.sib_rows[l] > 0)
        bulk_copy_g2s(psm + a.sib_off[l], pyr_u + (a.off[l - 1] + a.sib0[l]) * D,
                      (uint32_t)a.sib_rows[l] * D * (uint32_t)sizeof(TS), bar);
  }
  __syncthreads();
  const bool ok = mbar_wait_bounded(bar, 0, a.err, kDevErrTimeout, a.first_wait);
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) mbar_wait_bounded(bar, 0, a.err, kDevErrTimeout, kPathWaitCycles);
    return;
  }

  // leaves
  const int nn = (int)(a.hi - a.lo + 1);
  for (int idx = threadIdx.x; idx < nn * D; idx += kPathThreads) {
    const int j = idx / D, e = idx - (idx / D) * D;
    const long long i = a.lo + j;
    const long long r0 = i * a.lb, r1 = min(r0 + a.lb, a.N);
    const long long base = r0 - a.lo * a.lb;
    double s = 0.0;
    for (long long r = 0; r < r1 - r0; ++r) {
      if constexpr (sizeof(TIn) == 2)
        s += (double)bf16_bits_to_f32(tok[(base + r) * D + e]);
      else
        s += (double)tok[(base + r) * D + e];
    }
    const double v = s / (double)(r1 - r0);
    cur[j * D + e] = SumT<TS>::kept(v);
    pyr_u[(a.off[0] + i) * D + e] = SumT<TS>::store(v);
  }
  __syncthreads();

  long long lo = a.lo, hi = a.hi;
  for (int l = 1; l <= a.L; ++l) {
    const long long plo = lo / a.b, phi = hi / a.b;
    const int np = (int)(phi - plo + 1);
    const TS* sib = reinterpret_cast<const TS*>(psm + a.sib_off[l]);
    for (int idx = threadIdx.x; idx < np * D; idx += kPathThreads) {
      const int j = idx / D, e = idx - (idx / D) * D;
      const long long i = plo + j;
      const long long c0 = i * a.b, c1 = min(c0 + (long long)a.b, a.n[l - 1]);
      double s = 0.0;
      for (long long c = c0; c < c1; ++c)
        s += (c >= lo && c <= hi) ? cur[(c - lo) * D + e] : (double)SumT<TS>::load(sib[(c - a.sib0[l]) * D + e]);
      const double v = s / (double)(c1 - c0);
      nxt[j * D + e] = SumT<TS>::kept(v);
      pyr_u[(a.off[l] + i) * D + e] = SumT<TS>::store(v);
    }
    __syncthreads();
    double* tmp = cur;
    cur = nxt;
    nxt = tmp;
    lo = plo;
    hi = phi;
  }
}

int levels_for(long long n0, long long b) {
  if (n0 <= 0) return 0;
  int L = 1;
  long long span = b;
  while (span < n0) {
    span *= b;
    ++L;
  }
  return L;
}

namespace {

template <typename TIn, typename TS, int D>
cudaError_t launch_pass(const PassArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
  auto kern = pyramid_pass_kernel<TIn, TS, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, grid, dim3(kPassThreads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TIn, typename TS, int D>
cudaError_t launch_path(const AppendPathArgs& a, unsigned grid, size_t smem, cudaStream_t s) {
  auto kern = append_path_kernel<TIn, TS, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(grid), dim3(kPathThreads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

long long ipow(long long b, int k) {
  long long r = 1;
  for (int i = 0; i < k; ++i) r *= b;
  return r;
}

}  // namespace

cudaError_t launch_pyramid(zha_tree* t, const void* d_K, long long N, long long lo,
                           long long hi, cudaStream_t stream, int* launches) {
  const int D = t->desc.head_dim;
  const bool sbf = sum_bf16(t);
  const int ssz = sum_bytes(t);
  if (hi - lo + 1 <= kPathMaxLeaves) {
    // a few touched leaves (small appends, tiny trees): one launch walks the path to the root
    AppendPathArgs a{};
    const bool bf = t->desc.kv_dtype == ZHA_BF16;
    const int esz = bf ? 2 : 4;
    a.K = static_cast<const char*>(d_K);
    a.k_unit_stride = t->desc.capacity_tokens * D * (long long)esz;
    a.N = N;
    a.lb = t->desc.leaf_block;
    a.b = t->desc.branching;
    a.L = t->L;
    a.pyr = t->pyr;
    a.pyr_unit_stride = t->unit_rows * D;
    for (int l = 0; l <= t->L; ++l) {
      a.off[l] = t->off[l];
      a.n[l] = t->n[l];
    }
    a.lo = lo;
    a.hi = hi;
    a.err = t->d_err;
    a.first_wait = first_wait_cycles(t);
    a.tok_rows = (int)(std::min((hi + 1) * a.lb, N) - lo * a.lb);
    size_t o = (size_t)a.tok_rows * D * esz;
    long long clo = lo, chi = hi;
    for (int l = 1; l <= t->L; ++l) {
      const long long plo = clo / a.b, phi = chi / a.b;
      const long long r0 = plo * a.b, r1 = std::min((phi + 1) * a.b, t->n[l - 1]);
      o = (o + 127) / 128 * 128;
      a.sib0[l] = r0;
      a.sib_rows[l] = (int)(r1 - r0);
      a.sib_off[l] = (int)o;
      o += (size_t)(r1 - r0) * D * ssz;
      clo = plo;
      chi = phi;
    }
    o = (o + 127) / 128 * 128;
    a.fp64_off = (int)o;
    o += 2 * (size_t)kPathMaxLeaves * D * sizeof(double);
    a.bar_off = (int)o;
    o += 8;
    if (o <= kPathSmemCap) {
      const unsigned grid = (unsigned)t->units;
      cudaError_t e;
      if (sbf)
        e = bf ? (D == 128 ? launch_path<uint16_t, uint16_t, 128>(a, grid, o, stream)
                           : launch_path<uint16_t, uint16_t, 64>(a, grid, o, stream))
               : (D == 128 ? launch_path<float, uint16_t, 128>(a, grid, o, stream)
                           : launch_path<float, uint16_t, 64>(a, grid, o, stream));
      else
        e = bf ? (D == 128 ? launch_path<uint16_t, float, 128>(a, grid, o, stream)
                           : launch_path<uint16_t, float, 64>(a, grid, o, stream))
               : (D == 128 ? launch_path<float, float, 128>(a, grid, o, stream)
                           : launch_path<float, float, 64>(a, grid, o, stream));
      ++t->launches;
      if (launches) *launches = 1;
      return e;
    }
  }
  const long long b = t->desc.branching;
  const int L = t->L;
  int kmax = 0;
  while (ipow(b, kmax + 1) <= kChunkMaxPow && kmax + 1 < kMaxPassLevels) ++kmax;
  int count = 0;
  for (int level = 0; level <= L;) {
    const int k = std::min(kmax, L - level);
    const long long bk = ipow(b, k);
    const long long rep = bk >= kChunkTarget ? 1 : (kChunkTarget + bk - 1) / bk;
    const long long chunk = bk * rep;
    const long long span = ipow(b, level);  // leaves under one node of `level`
    PassArgs a{};
    a.b = (int)b;
    a.k = k;
    a.chunk = (int)chunk;
    a.pyr = t->pyr;
    a.pyr_unit_stride = t->unit_rows * D;
    long long lo_l = lo / span, hi_l = hi / span;
    for (int m = 0; m <= k; ++m) {
      const long long sm = ipow(b, m);
      a.lvl_off[m] = t->off[level + m];
      a.lvl_n[m] = t->n[level + m];
      a.lo[m] = lo_l / sm;
      a.hi[m] = std::min(hi_l / sm, t->n[level + m] - 1);
    }
    const bool from_tokens = level == 0;
    // source rows: K tokens (the cache's type) or the stored level below (the summaries')
    const bool src_bf = from_tokens ? t->desc.kv_dtype == ZHA_BF16 : sbf;
    if (from_tokens) {
      a.src = static_cast<const char*>(d_K);
      a.src_unit_stride = t->desc.capacity_tokens * D * (long long)(src_bf ? 2 : 4);
      a.n_src = N;
      a.blk0 = t->desc.leaf_block;
    } else {
      a.src = static_cast<const char*>(t->pyr) + t->off[level - 1] * D * (long long)ssz;
      a.src_unit_stride = t->unit_rows * D * (long long)ssz;
      a.n_src = t->n[level - 1];
      a.blk0 = b;
    }
    const long long c0 = a.lo[0] / chunk, c1 = a.hi[0] / chunk;
    a.chunk0 = c0;
    dim3 grid((unsigned)(c1 - c0 + 1), (unsigned)t->units);
    const size_t smem = (size_t)(chunk + (k > 0 ? chunk / b : 0)) * D * sizeof(double);
    cudaError_t e;
    if (sbf)
      e = src_bf ? (D == 128 ? launch_pass<uint16_t, uint16_t, 128>(a, grid, smem, stream)
                             : launch_pass<uint16_t, uint16_t, 64>(a, grid, smem, stream))
                 : (D == 128 ? launch_pass<float, uint16_t, 128>(a, grid, smem, stream)
                             : launch_pass<float, uint16_t, 64>(a, grid, smem, stream));
    else
      e = src_bf ? (D == 128 ? launch_pass<uint16_t, float, 128>(a, grid, smem, stream)
                             : launch_pass<uint16_t, float, 64>(a, grid, smem, stream))
                 : (D == 128 ? launch_pass<float, float, 128>(a, grid, smem, stream)
                             : launch_pass<float, float, 64>(a, grid, smem, stream));
    if (e != cudaSuccess) return e;
    ++count;
    ++t->launches;
    level += k + 1;
  }
  if (launches) *launches = count;
  return cudaSuccess;
}

}  // namespace zha

// Host-side state of a tree set and the launch entry points each kernel file provides.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/zha.h"

namespace zha {

constexpr int kMaxLevels = 48;      // levels 0 .. root; 2^47 leaves is far beyond any capacity
constexpr size_t kHeaderBytes = 256;
constexpr int kMaxBeam = 1024;
constexpr int kMaxCandidates = 4096;  // beam * branching bound for the route kernel

// Bits of the device error word.
enum : unsigned { kDevErrTimeout = 1u, kDevErrBadLeaf = 2u };

// Bound, in SM clock cycles, on every wait for a kernel's bulk copies (about a second).  A wait
// that runs out records kDevErrTimeout; the kernel then waits for the copies it issued with
// this same bound before it leaves.  zha_tree_set_wait_limit lowers the first bound (not
// the second) so tests can make a wait run out.
constexpr long long kCopyWaitCycles = 2000000000LL;

// Launch `kern` with programmatic stream serialization (see pdl_wait in
// device_common.cuh): the kernel may begin while its predecessor drains.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace zha

struct zha_tree {
  zha_tree_desc desc;
  char* ws;                    // caller's workspace
  size_t ws_bytes;
  unsigned* d_err;             // device error word (workspace header)
  void* pyr;                   // summaries: [units][unit_rows][head_dim], fp32 or bf16 bits
  long long units;
  long long unit_rows;         // rows per unit, all capacity-sized levels
  int Lcap;                    // levels for a full cache
  long long ncap[zha::kMaxLevels];  // capacity nodes per level
  long long off[zha::kMaxLevels];   // row offset of each level inside a unit
  long long N;                 // tokens currently summarised
  int L;                       // current levels (root at level L); 0 when empty
  long long n[zha::kMaxLevels];     // current nodes per level
  long long launches;          // kernels launched through this handle
  float* radii;                // caller's bounding-sphere radii [units][unit_rows], or null
  int sms;                     // SMs of the device the tree was created on
  int device;
  long long wait_limit;        // > 0: bound on a kernel's first wait for its copies (testing)
};

namespace zha {

// The bound of a kernel's first wait for its copies on this tree.
inline long long first_wait_cycles(const zha_tree* t) {
  return t->wait_limit > 0 ? t->wait_limit : kCopyWaitCycles;
}

// Bytes of one stored summary element (desc.summary_dtype).
inline int sum_bytes(const zha_tree* t) { return t->desc.summary_dtype == ZHA_BF16 ? 2 : 4; }
inline bool sum_bf16(const zha_tree* t) { return t->desc.summary_dtype == ZHA_BF16; }

// Levels above the leaves for n0 leaves: smallest L >= 1 with b^L >= n0 (0 if n0 == 0).
int levels_for(long long n0, long long b);

// Summary passes (tree_build.cu): recompute leaves [lo, hi] and all their ancestors
// up to level L, given tokens [0, N) of K.  Returns a cudaError_t.
cudaError_t launch_pyramid(zha_tree* t, const void* d_K, long long N, long long lo,
                           long long hi, cudaStream_t stream, int* launches);

// Route (route.cu).
cudaError_t launch_route(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads,
                         int nq, int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                         cudaStream_t stream);

// Fused route + attention (route.cu): one launch routes each query and attends over its
// leaves.  fused == false when a query's widest level does not fit the staged kernel.
// launch_decode with append_leaf >= 0: the launch also extends the tree by the tokens that
// the caller appended to leaf append_leaf (the tree's host shape already updated;
// requires append_ok).
struct DecodePlan {
  bool fused;
  bool warp;              // many queries: the warp-per-query kernel (route_warp.cu)
  bool group;             // at most two queries per SM: the CTA-per-query kernel (route_group.cuh)
  int group_warps;        // its warps per CTA (8 or 16)
  size_t rows_bytes;      // candidate-row / K-V stage region per query
  int stage_tokens;       // tokens per stage buffer
  int nbuf;               // stage buffers (2 or 3)
  int attn_warps;         // warps per query the attention wants (wide launches)
  size_t smem_per_query;
  bool append_ok;         // a one-leaf append can ride along (wide launches)
  size_t path_off, path_bytes;  // that append's region inside the row region
};
// allow_warp = false: the staged kernel's plan only (the causal and buffered calls run the
// staged kernel whatever the launch shape).  Otherwise many queries take the warp-per-query
// kernel and few the CTA-per-query kernel, where their shared memory fits.
DecodePlan plan_decode(const zha_tree* t, int q_heads, int nq, int beam, bool allow_warp = true);
cudaError_t launch_decode(zha_tree* t, const DecodePlan& p, const void* d_Q, zha_dtype q_dtype,
                          int q_heads, int nq, int beam, const void* d_K, const void* d_V,
                          float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace,
                          void* d_O, zha_dtype o_dtype, cudaStream_t stream,
                          long long append_leaf = -1);

// Causal routing (route.cu): query qg of every head routes over the tree of tokens
// 0 .. positions[qg % nq] (0 .. prefix_pos for every query when d_positions is null), and
// attends over its leaves' tokens in that prefix when d_O is given -- and over the
// buf_tokens tokens after the prefix (an append buffer; prefix_pos + 1 a multiple of the
// leaf block).  *unsupported: the shape does not fit the staged kernel (nothing launched).
cudaError_t launch_causal(zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq, int beam,
                          const long long* d_positions, const void* d_K, const void* d_V, float scale,
                          int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                          zha_dtype o_dtype, cudaStream_t stream, bool* unsupported,
                          long long prefix_pos = -1, int buf_tokens = 0);

// Bounding-sphere radii (radii.cu): recompute leaves [lo, hi] of every unit and all their
// ancestors (no-op without radii attached).
cudaError_t launch_radii(zha_tree* t, const void* d_K, long long lo, long long hi, cudaStream_t s);

// Threshold descent (threshold.cu): every token t < N with q . k_t >= tau per query.
cudaError_t launch_threshold(zha_tree* t, const void* d_K, const void* d_Q, zha_dtype q_dtype, int q_heads,
                             int nq, const float* d_tau, int max_tokens, int* d_tokens, int* d_count,
                             int* d_stats, cudaStream_t stream);

// Attention (attend.cu).
struct AttnPlan {
  int leaves_per_split;
  int splits;
  bool cluster;        // splits of a query merge inside one thread-block cluster
  int stage_tokens;
  int stages;          // smem buffers (1 or 2)
  size_t smem_bytes;
  size_t scratch_bytes;
};
constexpr int kMaxClusterSplits = 8;  // splits of one query merged inside a cluster
AttnPlan plan_attention(const zha_tree* t, int q_heads, int nq, int beam, int max_splits = 1 << 30);
cudaError_t launch_attention(zha_tree* t, const AttnPlan& plan, const void* d_Q,
                             zha_dtype q_dtype, int q_heads, int nq, const void* d_K,
                             const void* d_V, const int* d_leaf_idx, int beam, float scale,
                             void* d_O, zha_dtype o_dtype, void* d_scratch, cudaStream_t stream);

}  // namespace zha

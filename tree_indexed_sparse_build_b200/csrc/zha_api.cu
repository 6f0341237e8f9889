// C ABI of libzha (include/zha.h): argument checks, tree bookkeeping, kernel dispatch.
// Every device buffer belongs to the caller; nothing here allocates device memory.
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "zha_internal.h"

using namespace zha;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool desc_ok(const zha_tree_desc* d) {
  if (!d) return false;
  if (d->batch < 1 || d->kv_heads < 1 || (long long)d->batch * d->kv_heads > 65535) return false;
  if (d->branching < 2 || d->leaf_block < 1 || d->capacity_tokens < 1) return false;
  if (d->kv_dtype != ZHA_F32 && d->kv_dtype != ZHA_BF16) return false;
  if (d->summary_dtype != ZHA_F32 && d->summary_dtype != ZHA_BF16) return false;
  return true;
}

bool dim_supported(int d) { return d == 64 || d == 128; }

// Capacity geometry: ncap[l], off[l], Lcap, unit_rows.  False on overflow.
bool layout(const zha_tree_desc* d, long long* ncap, long long* off, int* Lcap, long long* rows) {
  const long long n0 = (d->capacity_tokens + d->leaf_block - 1) / d->leaf_block;
  const int L = levels_for(n0, d->branching);
  if (L + 1 > kMaxLevels) return false;
  long long n = n0, total = 0;
  for (int l = 0; l <= L; ++l) {
    ncap[l] = n;
    off[l] = total;
    total += n;
    n = (n + d->branching - 1) / d->branching;
  }
  *Lcap = L;
  *rows = total;
  return true;
}

void set_shape(zha_tree* t, long long N) {
  t->N = N;
  const long long n0 = N <= 0 ? 0 : (N + t->desc.leaf_block - 1) / t->desc.leaf_block;
  t->L = levels_for(n0, t->desc.branching);
  long long n = n0;
  for (int l = 0; l < kMaxLevels; ++l) {
    t->n[l] = l <= t->L ? n : 0;
    n = (n + t->desc.branching - 1) / t->desc.branching;
  }
}

zha_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA; }

bool dtype_ok(zha_dtype d) { return d == ZHA_F32 || d == ZHA_BF16; }

}  // namespace

extern "C" {

size_t zha_tree_workspace_bytes(const zha_tree_desc* desc) {
  if (!desc_ok(desc) || !dim_supported(desc->head_dim)) return 0;
  long long ncap[kMaxLevels], off[kMaxLevels], rows;
  int L;
  if (!layout(desc, ncap, off, &L, &rows)) return 0;
  const size_t esz = desc->summary_dtype == ZHA_BF16 ? 2 : 4;
  return kHeaderBytes + (size_t)desc->batch * desc->kv_heads * (size_t)rows * desc->head_dim * esz;
}

zha_status zha_tree_init(const zha_tree_desc* desc, void* d_workspace, size_t workspace_bytes,
                         zha_tree** out) {
  if (!out) return ZHA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!desc_ok(desc)) return ZHA_ERR_INVALID_ARG;
  if (!dim_supported(desc->head_dim)) return ZHA_ERR_UNSUPPORTED;
  if (!d_workspace || !aligned(d_workspace, 256)) return ZHA_ERR_INVALID_ARG;
  const size_t need = zha_tree_workspace_bytes(desc);
  if (need == 0) return ZHA_ERR_UNSUPPORTED;
  if (workspace_bytes < need) return ZHA_ERR_INVALID_ARG;
  zha_tree* t = static_cast<zha_tree*>(std::calloc(1, sizeof(zha_tree)));
  if (!t) return ZHA_ERR_INVALID_ARG;
  t->desc = *desc;
  t->ws = static_cast<char*>(d_workspace);
  t->ws_bytes = workspace_bytes;
  t->d_err = reinterpret_cast<unsigned*>(t->ws);
  t->pyr = t->ws + kHeaderBytes;
  t->units = (long long)desc->batch * desc->kv_heads;
  layout(desc, t->ncap, t->off, &t->Lcap, &t->unit_rows);
  set_shape(t, 0);
  if (cudaGetDevice(&t->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&t->sms, cudaDevAttrMultiProcessorCount, t->device) != cudaSuccess ||
      cudaMemset(t->d_err, 0, sizeof(unsigned)) != cudaSuccess) {
    std::free(t);
    return ZHA_ERR_CUDA;
  }
  *out = t;
  return ZHA_OK;
}

zha_status zha_tree_destroy(zha_tree* tree) {
  if (!tree) return ZHA_ERR_INVALID_ARG;
  std::free(tree);
  return ZHA_OK;
}

zha_status zha_tree_build(zha_tree* t, const void* d_K, long long seq_len, void* stream) {
  if (!t || seq_len < 0) return ZHA_ERR_INVALID_ARG;
  if (seq_len > t->desc.capacity_tokens) return ZHA_ERR_CAPACITY;
  if (seq_len > 0 && (!d_K || !aligned(d_K, 16))) return ZHA_ERR_INVALID_ARG;
  set_shape(t, seq_len);
  if (seq_len == 0) return ZHA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_pyramid(t, d_K, seq_len, 0, t->n[0] - 1, st, nullptr);
  if (e == cudaSuccess) e = launch_radii(t, d_K, 0, t->n[0] - 1, st);
  return cuda_status(e);
}

zha_status zha_tree_append(zha_tree* t, const void* d_K, long long new_seq_len, void* stream) {
  if (!t || new_seq_len < t->N) return ZHA_ERR_INVALID_ARG;
  if (new_seq_len > t->desc.capacity_tokens) return ZHA_ERR_CAPACITY;
  if (new_seq_len == t->N) return ZHA_OK;
  if (!d_K || !aligned(d_K, 16)) return ZHA_ERR_INVALID_ARG;
  if (t->N == 0) return zha_tree_build(t, d_K, new_seq_len, stream);
  const long long lo = t->N / t->desc.leaf_block;
  const long long hi = (new_seq_len - 1) / t->desc.leaf_block;
  set_shape(t, new_seq_len);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_pyramid(t, d_K, new_seq_len, lo, hi, st, nullptr);
  if (e == cudaSuccess) e = launch_radii(t, d_K, lo, hi, st);
  return cuda_status(e);
}

zha_status zha_route(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                     int beam, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* stream) {
  if (!t || !dtype_ok(q_dtype) || q_heads < 1 || nq < 0) return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if ((long long)beam * t->desc.branching > kMaxCandidates) return ZHA_ERR_UNSUPPORTED;
  if (t->N == 0) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_Q || !d_leaf_idx || !aligned(d_Q, 16) || !aligned(d_leaf_idx, 4)) return ZHA_ERR_INVALID_ARG;
  if ((d_leaf_score && !aligned(d_leaf_score, 4)) || (d_trace && !aligned(d_trace, 4)))
    return ZHA_ERR_INVALID_ARG;
  // The handle is logically const for routing; only its launch counter moves.
  return cuda_status(launch_route(const_cast<zha_tree*>(t), d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score,
                                  d_trace, static_cast<cudaStream_t>(stream)));
}

size_t zha_attn_scratch_bytes(const zha_tree* t, int q_heads, int nq, int beam) {
  if (!t || q_heads < 1 || nq < 1 || beam < 1 || beam > kMaxBeam) return 0;
  return plan_attention(t, q_heads, nq, beam).scratch_bytes;
}

zha_status zha_sparse_attn_decode(const zha_tree* t, const void* d_Q, zha_dtype q_dtype,
                                  int q_heads, int nq, const void* d_K, const void* d_V,
                                  const int* d_leaf_idx, int beam, float scale, void* d_O,
                                  zha_dtype o_dtype, void* d_scratch, size_t scratch_bytes,
                                  void* stream) {
  if (!t || !dtype_ok(q_dtype) || !dtype_ok(o_dtype) || q_heads < 1 || nq < 0)
    return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if (t->N == 0) return ZHA_ERR_INVALID_ARG;
  if (!(scale == scale)) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_Q || !d_K || !d_V || !d_leaf_idx || !d_O) return ZHA_ERR_INVALID_ARG;
  if (!aligned(d_Q, 16) || !aligned(d_K, 16) || !aligned(d_V, 16) || !aligned(d_O, 16) ||
      !aligned(d_leaf_idx, 4))
    return ZHA_ERR_INVALID_ARG;
  const AttnPlan plan = plan_attention(t, q_heads, nq, beam);
  if (plan.smem_bytes > 227 * 1024) return ZHA_ERR_UNSUPPORTED;
  if (plan.scratch_bytes > 0) {
    if (!d_scratch || !aligned(d_scratch, 16) || scratch_bytes < plan.scratch_bytes)
      return ZHA_ERR_INVALID_ARG;
  }
  return cuda_status(launch_attention(const_cast<zha_tree*>(t), plan, d_Q, q_dtype, q_heads, nq, d_K, d_V, d_leaf_idx,
                                      beam, scale, d_O, o_dtype, d_scratch,
                                      static_cast<cudaStream_t>(stream)));
}

zha_status zha_decode(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                      int beam, const void* d_K, const void* d_V, float scale, int* d_leaf_idx,
                      float* d_leaf_score, int* d_trace, void* d_O, zha_dtype o_dtype,
                      void* stream) {
  if (!t || !dtype_ok(q_dtype) || !dtype_ok(o_dtype) || q_heads < 1 || nq < 0)
    return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if ((long long)beam * t->desc.branching > kMaxCandidates) return ZHA_ERR_UNSUPPORTED;
  if (t->N == 0) return ZHA_ERR_INVALID_ARG;
  if (!(scale == scale)) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_Q || !d_K || !d_V || !d_leaf_idx || !d_O) return ZHA_ERR_INVALID_ARG;
  if (!aligned(d_Q, 16) || !aligned(d_K, 16) || !aligned(d_V, 16) || !aligned(d_O, 16) ||
      !aligned(d_leaf_idx, 4) || (d_leaf_score && !aligned(d_leaf_score, 4)) ||
      (d_trace && !aligned(d_trace, 4)))
    return ZHA_ERR_INVALID_ARG;
  zha_tree* tm = const_cast<zha_tree*>(t);  // only the launch counter moves
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DecodePlan dp = plan_decode(t, q_heads, nq, beam);
  if (dp.fused)
    return cuda_status(launch_decode(tm, dp, d_Q, q_dtype, q_heads, nq, beam, d_K, d_V, scale,
                                     d_leaf_idx, d_leaf_score, d_trace, d_O, o_dtype, s));
  // Levels too wide for the staged kernel: route, then attention with splits merged
  // inside clusters (no scratch).
  const AttnPlan ap = plan_attention(t, q_heads, nq, beam, kMaxClusterSplits);
  if (ap.smem_bytes > 227 * 1024 || ap.scratch_bytes > 0) return ZHA_ERR_UNSUPPORTED;
  cudaError_t e = launch_route(tm, d_Q, q_dtype, q_heads, nq, beam, d_leaf_idx, d_leaf_score, d_trace, s);
  if (e != cudaSuccess) return ZHA_ERR_CUDA;
  return cuda_status(launch_attention(tm, ap, d_Q, q_dtype, q_heads, nq, d_K, d_V, d_leaf_idx, beam,
                                      scale, d_O, o_dtype, nullptr, s));
}

zha_status zha_decode_step(zha_tree* t, const void* d_K, const void* d_V, long long new_seq_len,
                           const void* d_Q, zha_dtype q_dtype, int q_heads, int nq, int beam,
                           float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                           zha_dtype o_dtype, void* stream) {
  // the checks of both calls, before anything is launched or the tree changes
  if (!t || new_seq_len < t->N || !dtype_ok(q_dtype) || !dtype_ok(o_dtype) || q_heads < 1 || nq < 0)
    return ZHA_ERR_INVALID_ARG;
  if (new_seq_len > t->desc.capacity_tokens) return ZHA_ERR_CAPACITY;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if ((long long)beam * t->desc.branching > kMaxCandidates) return ZHA_ERR_UNSUPPORTED;
  if (new_seq_len == 0 || !(scale == scale)) return ZHA_ERR_INVALID_ARG;
  if (!d_Q || !d_K || !d_V || !d_leaf_idx || !d_O) return ZHA_ERR_INVALID_ARG;
  if (!aligned(d_Q, 16) || !aligned(d_K, 16) || !aligned(d_V, 16) || !aligned(d_O, 16) ||
      !aligned(d_leaf_idx, 4) || (d_leaf_score && !aligned(d_leaf_score, 4)) ||
      (d_trace && !aligned(d_trace, 4)))
    return ZHA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long lb = t->desc.leaf_block;
  // (a tree with radii attached takes the two launches: the fused append does not update them)
  const bool one_leaf = t->N > 0 && new_seq_len > t->N && t->N / lb == (new_seq_len - 1) / lb && !t->radii;
  if (one_leaf && nq > 0) {
    zha_tree saved = *t;
    set_shape(t, new_seq_len);
    const DecodePlan dp = plan_decode(t, q_heads, nq, beam);
    if (dp.append_ok)
      return cuda_status(launch_decode(t, dp, d_Q, q_dtype, q_heads, nq, beam, d_K, d_V, scale, d_leaf_idx,
                                       d_leaf_score, d_trace, d_O, o_dtype, s, (new_seq_len - 1) / lb));
    *t = saved;  // not fusable: append, then decode
  }
  const zha_status st = zha_tree_append(t, d_K, new_seq_len, stream);
  if (st != ZHA_OK) return st;
  return zha_decode(t, d_Q, q_dtype, q_heads, nq, beam, d_K, d_V, scale, d_leaf_idx, d_leaf_score,
                    d_trace, d_O, o_dtype, stream);
}

// d_positions null: every query at position prefix_pos, with buf_tokens buffered tokens
// after it attended as well (zha_decode_buffered).
static zha_status causal_call(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                              const long long* d_positions, int beam, const void* d_K, const void* d_V,
                              float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                              zha_dtype o_dtype, void* stream, long long prefix_pos = -1,
                              int buf_tokens = 0) {
  if (!t || !dtype_ok(q_dtype) || !dtype_ok(o_dtype) || q_heads < 1 || nq < 0) return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if ((long long)beam * t->desc.branching > kMaxCandidates) return ZHA_ERR_UNSUPPORTED;
  if (t->N == 0) return ZHA_ERR_INVALID_ARG;
  if (d_O && !(scale == scale)) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_Q || !d_K || (!d_positions && prefix_pos < 0) || !d_leaf_idx || (d_O && !d_V))
    return ZHA_ERR_INVALID_ARG;
  if (!aligned(d_Q, 16) || !aligned(d_K, 16) || !aligned(d_positions, 8) || !aligned(d_leaf_idx, 4) ||
      (d_O && (!aligned(d_O, 16) || !aligned(d_V, 16))) || (d_leaf_score && !aligned(d_leaf_score, 4)) ||
      (d_trace && !aligned(d_trace, 4)))
    return ZHA_ERR_INVALID_ARG;
  bool unsupported = false;
  const cudaError_t e = launch_causal(const_cast<zha_tree*>(t), d_Q, q_dtype, q_heads, nq, beam, d_positions,
                                      d_K, d_V, scale, d_leaf_idx, d_leaf_score, d_trace, d_O, o_dtype,
                                      static_cast<cudaStream_t>(stream), &unsupported, prefix_pos, buf_tokens);
  if (unsupported) return ZHA_ERR_UNSUPPORTED;
  return cuda_status(e);
}

zha_status zha_route_causal(const zha_tree* t, const void* d_K, const void* d_Q, zha_dtype q_dtype,
                            int q_heads, int nq, const long long* d_positions, int beam, int* d_leaf_idx,
                            float* d_leaf_score, int* d_trace, void* stream) {
  return causal_call(t, d_Q, q_dtype, q_heads, nq, d_positions, beam, d_K, nullptr, 1.0f, d_leaf_idx,
                     d_leaf_score, d_trace, nullptr, ZHA_F32, stream);
}

zha_status zha_decode_causal(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                             const long long* d_positions, int beam, const void* d_K, const void* d_V,
                             float scale, int* d_leaf_idx, float* d_leaf_score, int* d_trace, void* d_O,
                             zha_dtype o_dtype, void* stream) {
  if (!d_O) return ZHA_ERR_INVALID_ARG;
  return causal_call(t, d_Q, q_dtype, q_heads, nq, d_positions, beam, d_K, d_V, scale, d_leaf_idx,
                     d_leaf_score, d_trace, d_O, o_dtype, stream);
}

zha_status zha_decode_buffered(const zha_tree* t, const void* d_Q, zha_dtype q_dtype, int q_heads, int nq,
                               int beam, const void* d_K, const void* d_V, long long n_routed,
                               long long n_tokens, float scale, int* d_leaf_idx, float* d_leaf_score,
                               int* d_trace, void* d_O, zha_dtype o_dtype, void* stream) {
  if (!t || !d_O) return ZHA_ERR_INVALID_ARG;
  const long long lb = t->desc.leaf_block;
  if (n_routed < 1 || n_routed % lb != 0 || n_routed > t->N) return ZHA_ERR_INVALID_ARG;
  if (n_tokens < n_routed) return ZHA_ERR_INVALID_ARG;
  if (n_tokens > t->desc.capacity_tokens) return ZHA_ERR_CAPACITY;
  if (n_tokens - n_routed > (1LL << 30)) return ZHA_ERR_UNSUPPORTED;
  return causal_call(t, d_Q, q_dtype, q_heads, nq, nullptr, beam, d_K, d_V, scale, d_leaf_idx, d_leaf_score,
                     d_trace, d_O, o_dtype, stream, n_routed - 1, (int)(n_tokens - n_routed));
}

size_t zha_tree_radii_bytes(const zha_tree* t) {
  return t ? (size_t)t->units * (size_t)t->unit_rows * sizeof(float) : 0;
}

zha_status zha_tree_attach_radii(zha_tree* t, float* d_radii, size_t bytes, const void* d_K, void* stream) {
  if (!t) return ZHA_ERR_INVALID_ARG;
  if (!d_radii) {
    t->radii = nullptr;
    return ZHA_OK;
  }
  if (!aligned(d_radii, 16) || bytes < zha_tree_radii_bytes(t)) return ZHA_ERR_INVALID_ARG;
  if (t->N > 0 && (!d_K || !aligned(d_K, 16))) return ZHA_ERR_INVALID_ARG;
  t->radii = d_radii;
  if (t->N == 0) return ZHA_OK;
  return cuda_status(launch_radii(t, d_K, 0, t->n[0] - 1, static_cast<cudaStream_t>(stream)));
}

zha_status zha_threshold_route(const zha_tree* t, const void* d_K, const void* d_Q, zha_dtype q_dtype,
                               int q_heads, int nq, const float* d_tau, int max_tokens, int* d_tokens,
                               int* d_count, int* d_stats, void* stream) {
  if (!t || !dtype_ok(q_dtype) || q_heads < 1 || nq < 0 || max_tokens < 1) return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (t->N == 0 || !t->radii) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_K || !d_Q || !d_tau || !d_tokens || !d_count) return ZHA_ERR_INVALID_ARG;
  if (!aligned(d_K, 16) || !aligned(d_Q, 16) || !aligned(d_tau, 4) || !aligned(d_tokens, 4) ||
      !aligned(d_count, 4) || (d_stats && !aligned(d_stats, 4)))
    return ZHA_ERR_INVALID_ARG;
  return cuda_status(launch_threshold(const_cast<zha_tree*>(t), d_K, d_Q, q_dtype, q_heads, nq, d_tau, max_tokens,
                                      d_tokens, d_count, d_stats, static_cast<cudaStream_t>(stream)));
}

zha_status zha_tree_check(zha_tree* t, void* stream) {
  if (!t) return ZHA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  if (cudaMemcpyAsync(&h, t->d_err, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ZHA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ZHA_ERR_CUDA;
  if (h != 0) {
    if (cudaMemsetAsync(t->d_err, 0, sizeof(unsigned), s) != cudaSuccess) return ZHA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ZHA_ERR_CUDA;
  }
  if (h & kDevErrTimeout) return ZHA_ERR_TIMEOUT;
  if (h & kDevErrBadLeaf) return ZHA_ERR_DEVICE;
  return ZHA_OK;
}

long long zha_tree_seq_len(const zha_tree* t) { return t ? t->N : -1; }
int zha_tree_levels(const zha_tree* t) { return t ? t->L : -1; }
long long zha_tree_level_nodes(const zha_tree* t, int level) {
  if (!t || level < 0 || level > t->L) return 0;
  return t->n[level];
}
long long zha_tree_level_offset(const zha_tree* t, int level) {
  if (!t || level < 0 || level > t->Lcap) return -1;
  return t->off[level];
}
long long zha_tree_unit_rows(const zha_tree* t) { return t ? t->unit_rows : 0; }
const void* zha_tree_summaries(const zha_tree* t) { return t ? t->pyr : nullptr; }
long long zha_tree_launch_count(const zha_tree* t) { return t ? t->launches : -1; }
zha_status zha_tree_get_desc(const zha_tree* t, zha_tree_desc* out) {
  if (!t || !out) return ZHA_ERR_INVALID_ARG;
  *out = t->desc;
  return ZHA_OK;
}
int zha_tree_device(const zha_tree* t) { return t ? t->device : -1; }
zha_status zha_tree_set_wait_limit(zha_tree* t, long long cycles) {
  if (!t || cycles < 0) return ZHA_ERR_INVALID_ARG;
  t->wait_limit = cycles;
  return ZHA_OK;
}

const char* zha_status_string(zha_status s) {
  switch (s) {
    case ZHA_OK: return "ok";
    case ZHA_ERR_INVALID_ARG: return "invalid argument";
    case ZHA_ERR_CAPACITY: return "sequence length beyond tree capacity";
    case ZHA_ERR_UNSUPPORTED: return "unsupported shape";
    case ZHA_ERR_CUDA: return "CUDA error";
    case ZHA_ERR_TIMEOUT: return "bounded device wait expired";
    case ZHA_ERR_DEVICE: return "invalid data met on the device";
  }
  return "unknown status";
}

}  // extern "C"

// Sparse decode attention for callers that cannot allocate device memory.
//
// zha_sparse_attn_decode takes its split-KV partials in a scratch buffer the caller
// allocates.  Some callers have no way to do that: an operator hook that is handed only
// its input and output pointers (no workspace, no allocator), or a code path where
// cudaMalloc is not allowed because it synchronizes the device or because all device
// memory belongs to another allocator.  zha_sparse_attn_decode_noalloc runs the same
// attention kernels with the partials placed in a fixed array that lives in this
// library's own device memory.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes bytes.  Every GPU
// that loads this library holds it until the process exits.  Host code cannot pass the
// variable itself to a kernel (on the host its name is only a stand-in for the symbol),
// so the first call on each device, with that device current, looks the device address
// up with cudaGetSymbolAddress and caches it.  Nothing in it has to start at zero: every
// split writes its partial in full before the combine step reads it.  All calls share
// the one array, so two calls whose kernels overlap on the GPU race on it.
#include <mutex>

#include "zha_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 128 * 1024;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" zha_status zha_sparse_attn_decode_noalloc(const zha_tree* t, const void* d_Q,
                                                     zha_dtype q_dtype, int q_heads, int nq,
                                                     const void* d_K, const void* d_V,
                                                     const int* d_leaf_idx, int beam, float scale,
                                                     void* d_O, zha_dtype o_dtype, void* stream) {
  const bool dt_ok = (q_dtype == ZHA_F32 || q_dtype == ZHA_BF16) &&
                     (o_dtype == ZHA_F32 || o_dtype == ZHA_BF16);
  if (!t || !dt_ok || q_heads < 1 || nq < 0) return ZHA_ERR_INVALID_ARG;
  if (q_heads % t->desc.kv_heads != 0) return ZHA_ERR_INVALID_ARG;
  if (beam < 1 || beam > zha::kMaxBeam) return ZHA_ERR_INVALID_ARG;
  if (t->N == 0) return ZHA_ERR_INVALID_ARG;
  if (!(scale == scale)) return ZHA_ERR_INVALID_ARG;
  if (nq == 0) return ZHA_OK;
  if (!d_Q || !d_K || !d_V || !d_leaf_idx || !d_O) return ZHA_ERR_INVALID_ARG;
  if (!aligned16(d_Q) || !aligned16(d_K) || !aligned16(d_V) || !aligned16(d_O) ||
      (reinterpret_cast<uintptr_t>(d_leaf_idx) & 3u) != 0)
    return ZHA_ERR_INVALID_ARG;
  // The array's address is looked up (and cached) for the current device, and the kernels
  // launch there: both must be the tree's device.
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZHA_ERR_CUDA;
  if (dev != t->device) return ZHA_ERR_INVALID_ARG;
  const zha::AttnPlan plan = zha::plan_attention(t, q_heads, nq, beam);
  if (plan.smem_bytes > 227 * 1024) return ZHA_ERR_UNSUPPORTED;
  if (plan.scratch_bytes > kNoAllocScratchBytes) return ZHA_ERR_CAPACITY;
  void* scratch = nullptr;
  if (plan.scratch_bytes > 0 && scratch_address(&scratch) != cudaSuccess) return ZHA_ERR_CUDA;
  const cudaError_t e = zha::launch_attention(const_cast<zha_tree*>(t), plan, d_Q, q_dtype, q_heads,
                                              nq, d_K, d_V, d_leaf_idx, beam, scale, d_O, o_dtype,
                                              scratch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA;
}

extern "C" size_t zha_noalloc_scratch_capacity(void) { return kNoAllocScratchBytes; }

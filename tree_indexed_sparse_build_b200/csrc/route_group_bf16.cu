// Instantiations of route_group_kernel for bf16 K/V rows (see route_group.cuh).
#include "route_group.cuh"

namespace zha {

cudaError_t route_group_launch_bf16(int D, bool s16, int nw, bool append, const RouteArgs& a, size_t smem,
                                    cudaStream_t s) {
  return run_group_kv<uint16_t>(D, s16, nw, append, a, smem, s);
}

}  // namespace zha

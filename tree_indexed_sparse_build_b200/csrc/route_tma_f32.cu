// Instantiations of route_tma_kernel for fp32 K/V rows and fp32 summaries (see route_kernel.cuh).
#include "route_kernel.cuh"

namespace zha {

cudaError_t route_tma_launch_f32(int D, bool grouped, bool narrow, const RouteArgs& a, unsigned blocks,
                                 int threads, size_t smem, cudaStream_t s, int path) {
  return run_route_tma_d_impl<float, float>(D, grouped, narrow, a, blocks, threads, smem, s, path);
}

}  // namespace zha

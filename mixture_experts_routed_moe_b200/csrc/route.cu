// Router top-k ("Experts backends", introduction: each token goes to k experts
// that a router picks; the experts' results are later summed with the routing
// weights).
//
// One warp per token over logits in global memory; the per-token selection
// (fp32 softmax denominator, k shuffle arg-max rounds with ties to the lower
// index, renormalisation over the chosen k) is route_token in route_core.cuh.
#include "moe_common.cuh"
#include "moe_internal.h"
#include "route_core.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

template <int kPerLane>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) route_kernel(const float* __restrict__ logits, int T, int E,
                                                                    int k, int* __restrict__ topk_idx,
                                                                    float* __restrict__ topk_w) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarpsPerBlock + warp;
  if (t >= T) return;
  route_token<kPerLane>(logits + static_cast<size_t>(t) * E, E, k, lane, topk_idx + static_cast<size_t>(t) * k,
                        topk_w + static_cast<size_t>(t) * k);
}

template <int kPerLane>
cudaError_t launch_route_t(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st) {
  const int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  return launch_pdl(route_kernel<kPerLane>, dim3(blocks), dim3(kWarpsPerBlock * 32), 0, st, logits, T, E, k, idx,
                    w);
}

}  // namespace

cudaError_t launch_route(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st) {
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) return launch_route_t<1>(logits, T, E, k, idx, w, st);
  if (per_lane <= 2) return launch_route_t<2>(logits, T, E, k, idx, w, st);
  if (per_lane <= 4) return launch_route_t<4>(logits, T, E, k, idx, w, st);
  if (per_lane <= 8) return launch_route_t<8>(logits, T, E, k, idx, w, st);
  if (per_lane <= 16) return launch_route_t<16>(logits, T, E, k, idx, w, st);
  return launch_route_t<32>(logits, T, E, k, idx, w, st);
}

}  // namespace moe

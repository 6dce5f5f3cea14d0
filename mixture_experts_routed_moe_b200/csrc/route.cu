// Router top-k ("Experts backends", introduction: a router selects k experts
// for each token; the expert outputs are later aggregated with the routing
// weights).
//
// One warp per token. Each lane holds up to kPerLane logits (expert
// lane + 32*i). The warp computes the fp32 softmax denominator over all E
// experts, then selects k times the largest remaining logit (equal logits:
// lower index first) with a shuffle reduction over (value, index), and finally
// renormalises the chosen probabilities over the k. Selection compares the
// logits themselves, which orders experts exactly as the softmax does.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ bool beats(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int kPerLane>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) route_kernel(const float* __restrict__ logits, int T, int E,
                                                                    int k, int* __restrict__ topk_idx,
                                                                    float* __restrict__ topk_w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarpsPerBlock + warp;
  if (t >= T) return;
  const float* row = logits + static_cast<size_t>(t) * E;

  float v[kPerLane];
  float vmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
    vmax = fmaxf(vmax, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));

  // softmax denominator over all experts (fp32)
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i)
    if (lane + 32 * i < E) z += expf(v[i] - vmax);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);

  uint32_t taken = 0;  // bit i: expert lane + 32*i already selected
  float psum = 0.f, pcomp = 0.f;  // compensated (Kahan) sum of the chosen probabilities
  int* idx_out = topk_idx + static_cast<size_t>(t) * k;
  float* w_out = topk_w + static_cast<size_t>(t) * k;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && beats(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (beats(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    // the owner lane marks the winner as taken
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    const float p = expf(bv - vmax) / z;  // softmax probability of the winner
    const float yk = p - pcomp;
    const float tk = psum + yk;
    pcomp = (tk - psum) - yk;
    psum = tk;
    if (lane == 0) {
      idx_out[j] = bi;
      w_out[j] = p;
    }
  }
  __syncwarp();
  // renormalise over the chosen k (each lane rescales its own slots)
  for (int j = lane; j < k; j += 32) w_out[j] = w_out[j] / psum;
}

template <int kPerLane>
cudaError_t launch_route_t(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st) {
  const int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  route_kernel<kPerLane><<<blocks, kWarpsPerBlock * 32, 0, st>>>(logits, T, E, k, idx, w);
  return cudaGetLastError();
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

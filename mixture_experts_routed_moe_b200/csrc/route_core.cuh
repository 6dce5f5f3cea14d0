// Top-k routing of one token by one warp ("Experts backends", introduction:
// each token goes to k experts that a router picks, and the experts' results
// are later summed with the routing weights). Shared by the routing kernel (logits
// in global memory) and the fused router GEMM (logits in shared memory), so
// both give the same bits for the same logits.
//
// Each lane holds up to kPerLane logits (expert lane + 32*i). The warp
// computes the fp32 softmax denominator over all E experts, then selects k
// times the largest remaining logit (equal logits: lower index first) with a
// shuffle reduction over (value, index), and finally renormalises the chosen
// probabilities over the k. Selection compares the logits themselves, which
// orders experts exactly as the softmax does.
#pragma once

#include "moe_common.cuh"

namespace moe {

__device__ __forceinline__ bool route_beats(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// row: the token's E logits (global or shared memory); idx_out / w_out: its k slots.
template <int kPerLane>
__device__ __forceinline__ void route_token(const float* row, int E, int k, int lane, int* idx_out, float* w_out) {
  float v[kPerLane];
  float vmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? row[e] : -INFINITY;
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
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && route_beats(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (route_beats(ov, oi, bv, bi)) {
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

}  // namespace moe

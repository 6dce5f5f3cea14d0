// Top-k routing of one token by one warp ("Experts backends", introduction:
// each token goes to k experts that a router picks, and the experts' results
// are later summed with the routing weights). Shared by the routing kernel (logits
// in global memory) and the fused router GEMM (logits in shared memory), so
// both give the same bits for the same logits.
//
// Each lane holds up to kPerLane logits (expert lane + 32*i). The warp selects
// k times the largest remaining logit (equal logits: lower index first):
// every lane offers its best untaken (logit, expert), one warp max-reduction
// over order-preserving integer keys of the logits finds the value and one
// min-reduction over the experts offering it breaks ties. Selection compares
// the logits themselves, which orders experts exactly as the softmax does.
// The weights are the softmax probabilities renormalised over the k chosen
// experts: w_j = exp(l_j - l_max) / sum_j' exp(l_j' - l_max), where the first
// selected logit is l_max and the softmax denominator over all E experts
// cancels. The sum is compensated (Kahan).
#pragma once

#include "moe_common.cuh"

namespace moe {

// Order-preserving map of a (non-NaN) float to an unsigned key: larger floats
// give larger keys, -0 and +0 the same one, and the inverse map is exact.
__device__ __forceinline__ uint32_t route_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float route_key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// row: the token's E logits (global or shared memory); idx_out / w_out: its k slots.
template <int kPerLane>
__device__ __forceinline__ void route_token(const float* row, int E, int k, int lane, int* idx_out, float* w_out) {
  // keys of this lane's logits (expert lane + 32*i); a taken or absent expert
  // has key 0, below every logit's key
  uint32_t key[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? route_key(row[e]) : 0u;
  }
  float vmax = 0.f, psum = 0.f, pcomp = 0.f;
  // slot j < 32 is kept by lane j until the end (the k selected experts and
  // their softmax numerators), so the slots are written once, coalesced
  int my_idx = 0;
  float my_p = 0.f;
  for (int j = 0; j < k; ++j) {
    // this lane's best untaken expert (i ascending keeps the lower index on ties)
    uint32_t best = 0;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      if (key[i] > best) {
        best = key[i];
        bi = i;
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, best);
    // lanes holding the maximum offer their expert; the lowest index wins
    const uint32_t cand = (best == kmax && kmax != 0u) ? static_cast<uint32_t>(lane + 32 * bi) : 0x7fffffffu;
    const int win = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
    if ((win & 31) == lane) {
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (i == (win >> 5)) key[i] = 0u;
    }
    const float bv = route_key_value(kmax);
    if (j == 0) vmax = bv;
    const float p = expf(bv - vmax);  // exp(l_j - l_max): the softmax numerator
    const float yk = p - pcomp;
    const float tk = psum + yk;
    pcomp = (tk - psum) - yk;
    psum = tk;
    if (j < 32) {
      if (lane == j) {
        my_idx = win;
        my_p = p;
      }
    } else if (lane == 0) {  // slots beyond 32 go out now and are rescaled below
      idx_out[j] = win;
      w_out[j] = p;
    }
  }
  // renormalise over the chosen k
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = my_p / psum;
  }
  if (k > 32) {
    __syncwarp();
    for (int j = 32 + lane; j < k; j += 32) w_out[j] = w_out[j] / psum;
  }
}

}  // namespace moe

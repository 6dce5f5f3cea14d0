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
// cancels. The k numerators are computed after the selection, one per lane,
// and summed in a fixed butterfly order.
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
  // selection: slot j < 32 is kept by lane j (its expert and key); later
  // slots (k > 32) go to global memory at once
  int my_idx = 0;
  uint32_t my_key = 0;
  uint32_t key0 = 0;
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
    if (j == 0) key0 = kmax;
    if (j < 32) {
      if (lane == j) {
        my_idx = win;
        my_key = kmax;
      }
    } else if (lane == 0) {
      idx_out[j] = win;
      w_out[j] = route_key_value(kmax);  // the logit for now; the weight below
    }
  }
  // weights: the softmax numerators exp(l_j - l_max) of the chosen experts,
  // one per lane, their sum over the k slots (a fixed butterfly order, and
  // for k > 32 the later slots added in slot order, compensated), and p_j / sum
  const float vmax = route_key_value(key0);
  const float p = lane < k ? expf(route_key_value(my_key) - vmax) : 0.f;
  float psum = p;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
  if (k > 32) {
    // the later slots' numerators, added in slot order with compensation (Kahan)
    __syncwarp();
    float rest = 0.f, comp = 0.f;
    for (int j = 32; j < k; ++j) {
      const float yk = expf(w_out[j] - vmax) - comp;
      const float tk = rest + yk;
      comp = (tk - rest) - yk;
      rest = tk;
    }
    psum += rest;
    __syncwarp();
    if (lane == 0)
      for (int j = 32; j < k; ++j) w_out[j] = expf(w_out[j] - vmax) / psum;
  }
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = p / psum;
  }
}

}  // namespace moe

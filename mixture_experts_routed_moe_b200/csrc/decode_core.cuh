// Weight-streaming building blocks of the small-token expert forward on the
// CUDA cores, used by the fused single-launch forward (fused_decode.cu) and
// the FP4 decode kernels (decode_fp4.cu). With only a few tokens per expert
// the layer is bound by reading each touched expert's weights once from HBM:
// a warp owns a few consecutive weight rows of one expert, streams them with
// 16-byte no-L1 loads and dots them against up to four of that expert's
// activation rows.
#pragma once

#include "moe_common.cuh"

namespace moe {
namespace dec {

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x);
  f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y);
  f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z);
  f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w);
  f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16-byte activation load: through the read-only path for inputs of the
// launch, or from L2 (ld.global.cg) for rows written earlier in the same launch.
template <bool kCoherent>
__device__ __forceinline__ uint4 load_act(const uint4* p) {
  if constexpr (kCoherent)
    return __ldcg(p);
  else
    return __ldg(p);
}

// acc[r][q] += <weight row r, activation row q> over this lane's 16-byte
// chunks (NR rows, NQ activation rows). All NR weight loads of a chunk step
// are issued together; each weight chunk is converted to fp32 once and each
// activation chunk once, then shared by every (row, token) pair.
template <int NR, int NQ, bool kCoherent = false>
__device__ __forceinline__ void dot_rows(const __nv_bfloat16* const (&w)[NR], const __nv_bfloat16* const (&a)[4],
                                         int nch, int lane, float (&acc)[NR][4]) {
  for (int ch = lane; ch < nch; ch += 32) {
    uint4 wv[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) wv[r] = ld_stream_u4(w[r] + ch * 8);
    float xf[NQ][8];
#pragma unroll
    for (int q = 0; q < NQ; ++q) unpack8(load_act<kCoherent>(reinterpret_cast<const uint4*>(a[q]) + ch), xf[q]);
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float wf[8];
      unpack8(wv[r], wf);
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[r][q] = fmaf(wf[i], xf[q][i], acc[r][q]);
    }
  }
}

// gate/up: weight rows 0..3 are gate rows n0.., rows 4..7 the up rows I+n0..;
// h[row0 + q, n0 + r] = act(gate_r . x_q) * (up_r . x_q) in bf16, for NQ rows.
template <int NQ>
__device__ __forceinline__ void gate_up_group(const __nv_bfloat16* const (&w)[8], const __nv_bfloat16* const (&a)[4],
                                              int nch, int lane, __nv_bfloat16* h, size_t row0, int I, int n0,
                                              int act) {
  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
  dot_rows<8, NQ>(w, a, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float g = warp_sum(acc[r][q]), u = warp_sum(acc[4 + r][q]);
      if (lane == r) h[(row0 + q) * I + n0 + r] = __float2bfloat16_rn(gated_act(act, g, u));
    }
}

// down: 8 consecutive rows c0..c0+7 of H; y[row0 + q, c0 + r] = Wd_r . h_q in bf16.
template <int NQ, bool kCoherent = false>
__device__ __forceinline__ void down_group(const __nv_bfloat16* const (&w)[8], const __nv_bfloat16* const (&a)[4],
                                           int nch, int lane, __nv_bfloat16* y, size_t row0, int H, int c0) {
  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
  dot_rows<8, NQ, kCoherent>(w, a, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float v = warp_sum(acc[r][q]);
      if (lane == r) y[(row0 + q) * H + c0 + r] = __float2bfloat16_rn(v);
    }
}

}  // namespace dec
}  // namespace moe

// Weighted combine back to token order ("Experts backends", introduction: a
// token's result is the sum of its k experts' results, each scaled by the
// routing weight of that expert).
//
//   out[t, :] = bf16( sum_{j = 0..k-1} topk_w[t, j] * y[slot_row[t*k+j], :] )
//
// fp32 fused multiply-adds in ascending j, no atomics, so the result does not
// depend on scheduling. One block per token; each thread produces 8 output
// columns per step from 16-byte loads of the k expert-output rows.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 128;

__global__ void __launch_bounds__(kBlock) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                         const int* __restrict__ slot_row,
                                                         const float* __restrict__ topk_w,
                                                         __nv_bfloat16* __restrict__ out, int H, int k) {
  const int t = blockIdx.x;
  const int* rows = slot_row + static_cast<size_t>(t) * k;
  const float* w = topk_w + static_cast<size_t>(t) * k;
  uint4* o = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H);
  for (int c = threadIdx.x; c < H / 8; c += kBlock) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int r = __ldg(rows + j);
      if (r < 0) continue;  // assignment rejected by the permute stage (bad index)
      const float wj = __ldg(w + j);
      const uint4 v = ld_stream_u4(y + static_cast<size_t>(r) * H + c * 8);
      acc[0] = fmaf(wj, bf16_lo(v.x), acc[0]);
      acc[1] = fmaf(wj, bf16_hi(v.x), acc[1]);
      acc[2] = fmaf(wj, bf16_lo(v.y), acc[2]);
      acc[3] = fmaf(wj, bf16_hi(v.y), acc[3]);
      acc[4] = fmaf(wj, bf16_lo(v.z), acc[4]);
      acc[5] = fmaf(wj, bf16_hi(v.z), acc[5]);
      acc[6] = fmaf(wj, bf16_lo(v.w), acc[6]);
      acc[7] = fmaf(wj, bf16_hi(v.w), acc[7]);
    }
    o[c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                      pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace

cudaError_t launch_combine(const moe_shape* s, const Plan& p, const float* topk_w, void* out, uint8_t* ws,
                           cudaStream_t st) {
  combine_kernel<<<s->T, kBlock, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(ws + p.y),
                                          reinterpret_cast<const int*>(ws + p.slot_row), topk_w,
                                          static_cast<__nv_bfloat16*>(out), s->H, s->k);
  return cudaGetLastError();
}

}  // namespace moe

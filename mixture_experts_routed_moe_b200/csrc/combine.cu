// Weighted combine back to token order ("Experts backends", introduction: a
// token's result is the sum of its k experts' results, each scaled by the
// routing weight of that expert).
//
//   out[t, :] = bf16( sum_{j = 0..k-1} topk_w[t, j] * y[slot_row[t*k+j], :] )
//
// fp32 fused multiply-adds in ascending j, no atomics, so the result does not
// depend on scheduling. One block per token (its k rows and weights staged in
// shared memory); each thread produces 8 output columns per step from 16-byte
// loads of the k expert-output rows, four rows' loads in flight at a time.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 128;
constexpr int kBatch = 4;  // expert-output rows whose loads are in flight together

__global__ void __launch_bounds__(kBlock) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                         const int* __restrict__ slot_row,
                                                         const float* __restrict__ topk_w,
                                                         __nv_bfloat16* __restrict__ out, int H, int k) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  extern __shared__ int s_slot[];  // [k] rows, then [k] weights
  float* s_w = reinterpret_cast<float*>(s_slot + k);
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += kBlock) {
    s_slot[j] = __ldg(slot_row + static_cast<size_t>(t) * k + j);
    s_w[j] = __ldg(topk_w + static_cast<size_t>(t) * k + j);
  }
  __syncthreads();
  uint4* o = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H);
  for (int c = threadIdx.x; c < H / 8; c += kBlock) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += kBatch) {
      // issue the batch's loads first, then accumulate in ascending j
      uint4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int j = j0 + b;
        const int r = j < k ? s_slot[j] : -1;
        v[b] = r >= 0 ? ld_stream_u4(y + static_cast<size_t>(r) * H + c * 8) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int j = j0 + b;
        if (j >= k || s_slot[j] < 0) continue;  // past k, or rejected by the permute stage (bad index)
        const float wj = s_w[j];
        acc[0] = fmaf(wj, bf16_lo(v[b].x), acc[0]);
        acc[1] = fmaf(wj, bf16_hi(v[b].x), acc[1]);
        acc[2] = fmaf(wj, bf16_lo(v[b].y), acc[2]);
        acc[3] = fmaf(wj, bf16_hi(v[b].y), acc[3]);
        acc[4] = fmaf(wj, bf16_lo(v[b].z), acc[4]);
        acc[5] = fmaf(wj, bf16_hi(v[b].z), acc[5]);
        acc[6] = fmaf(wj, bf16_lo(v[b].w), acc[6]);
        acc[7] = fmaf(wj, bf16_hi(v[b].w), acc[7]);
      }
    }
    o[c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                      pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace

cudaError_t launch_combine(const moe_shape* s, const Plan& p, const float* topk_w, void* out, uint8_t* ws,
                           cudaStream_t st) {
  const size_t smem = static_cast<size_t>(s->k) * (sizeof(int) + sizeof(float));  // k <= 1024: at most 8 KB
  return launch_pdl(combine_kernel, dim3(s->T), dim3(kBlock), smem, st,
                    reinterpret_cast<const __nv_bfloat16*>(ws + p.y), reinterpret_cast<const int*>(ws + p.slot_row),
                    topk_w, static_cast<__nv_bfloat16*>(out), s->H, s->k);
}

}  // namespace moe

// Small-token path: the expert matmuls as weight streaming ("Experts
// backends": the batched_mm backend is the fastest for small inputs and the
// decode-stage switch moves generation onto it; here the same per-token form
// is done without duplicating any parameters).
//
// With only a few tokens per expert, the layer is bound by reading each
// touched expert's weights once from HBM. Every warp owns a few consecutive
// weight rows of one touched expert, streams them with 16-byte no-L1 loads and
// dots them against all of that expert's tokens (kept in L1/L2). No tile
// padding, no tensor cores: the FMAs are far below the CUDA-core peak at these
// token counts.
//
//   gate/up:  h[row, n] = silu(<x_t, Wg_e[n]>) * <x_t, Wu_e[n]>  (bf16)
//   down:     y[row, c] = <h[row], Wd_e[c]>                      (bf16)
//
// Rows are the unpadded expert-major permuted rows (tile size 1).
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 256;
constexpr int kWarpsPerBlock = kBlock / 32;

// Reduce 32 per-lane partial sums across the warp with 31 shuffles; afterwards
// lane l holds the full sum of value index l.
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// gate/up: a task is (touched expert u, 4 consecutive rows n0..n0+3 of I, a
// group of up to 4 of the expert's tokens). Value index (0..31) =
// half*16 + row*4 + token, half 0 = gate, 1 = up.
__global__ void __launch_bounds__(kBlock) decode_gate_up_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wgu, const int* __restrict__ cnt,
    const int* __restrict__ row_off, const int* __restrict__ row_src, const int* __restrict__ touched,
    const int* __restrict__ hdr, __nv_bfloat16* __restrict__ h, int H, int I, int k) {
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = I / 4;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = H / 8;  // 16-byte chunks per row
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int n0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 4;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const __nv_bfloat16* wg = wgu + (static_cast<size_t>(e) * 2 * I + n0) * H;
    const __nv_bfloat16* wu = wg + static_cast<size_t>(I) * H;
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* xt[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = r_e + g0 + min(q, ntok - 1);
        xt[q] = x + static_cast<size_t>(row_src[rr] / k) * H;
      }
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      for (int ch = lane; ch < nch; ch += 32) {
        uint4 a[4], b[4], xv[4];
#pragma unroll
        for (int rw = 0; rw < 4; ++rw) {
          a[rw] = ld_stream_u4(wg + static_cast<size_t>(rw) * H + ch * 8);
          b[rw] = ld_stream_u4(wu + static_cast<size_t>(rw) * H + ch * 8);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = __ldg(reinterpret_cast<const uint4*>(xt[q]) + ch);
#pragma unroll
        for (int rw = 0; rw < 4; ++rw)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[rw * 4 + q] = dot8_bf16(a[rw], xv[q], acc[rw * 4 + q]);
            acc[16 + rw * 4 + q] = dot8_bf16(b[rw], xv[q], acc[16 + rw * 4 + q]);
          }
      }
      const float sum = warp_transpose_reduce(acc, lane);
      const float up = __shfl_down_sync(0xffffffffu, sum, 16);
      if (lane < 16) {
        const int rw = lane >> 2, q = lane & 3;
        if (q < ntok) h[static_cast<size_t>(r_e + g0 + q) * I + n0 + rw] = __float2bfloat16_rn(swiglu(sum, up));
      }
    }
  }
}

// down: a task is (touched expert u, 8 consecutive rows c0..c0+7 of H, a group
// of up to 4 tokens). Value index = row*4 + token.
__global__ void __launch_bounds__(kBlock) decode_down_kernel(
    const __nv_bfloat16* __restrict__ h, const __nv_bfloat16* __restrict__ wd, const int* __restrict__ cnt,
    const int* __restrict__ row_off, const int* __restrict__ touched, const int* __restrict__ hdr,
    __nv_bfloat16* __restrict__ y, int H, int I) {
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = H / 8;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = I / 8;
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int c0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 8;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const __nv_bfloat16* w = wd + (static_cast<size_t>(e) * H + c0) * I;
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* ht[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) ht[q] = h + static_cast<size_t>(r_e + g0 + min(q, ntok - 1)) * I;
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      for (int ch = lane; ch < nch; ch += 32) {
        uint4 a[8], hv[4];
#pragma unroll
        for (int rw = 0; rw < 8; ++rw) a[rw] = ld_stream_u4(w + static_cast<size_t>(rw) * I + ch * 8);
#pragma unroll
        for (int q = 0; q < 4; ++q) hv[q] = *(reinterpret_cast<const uint4*>(ht[q]) + ch);
#pragma unroll
        for (int rw = 0; rw < 8; ++rw)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[rw * 4 + q] = dot8_bf16(a[rw], hv[q], acc[rw * 4 + q]);
      }
      const float sum = warp_transpose_reduce(acc, lane);
      const int rw = lane >> 2, q = lane & 3;
      if (q < ntok) y[static_cast<size_t>(r_e + g0 + q) * H + c0 + rw] = __float2bfloat16_rn(sum);
    }
  }
}

}  // namespace

// which = 0: gate/up (x -> h); which = 1: down (h -> y).
cudaError_t launch_decode(const moe_shape* s, const Plan& p, const void* x, const void* w_gate_up,
                          const void* w_down, uint8_t* ws, int which, int num_sms, cudaStream_t st) {
  const int* cnt = reinterpret_cast<const int*>(ws + p.cnt);
  const int* row_off = reinterpret_cast<const int*>(ws + p.mt_base);  // tile size 1: offsets are rows
  const int* row_src = reinterpret_cast<const int*>(ws + p.row_src);
  const int* touched = reinterpret_cast<const int*>(ws + p.touched);
  const int* hdr = reinterpret_cast<const int*>(ws + p.hdr);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + p.h);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  // enough resident warps to keep ~100 KB of weight loads in flight per SM
  const int grid = num_sms * 4;
  if (which == 0) {
    decode_gate_up_kernel<<<grid, kBlock, 0, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                   static_cast<const __nv_bfloat16*>(w_gate_up), cnt, row_off,
                                                   row_src, touched, hdr, h, s->H, s->I, s->k);
  } else {
    decode_down_kernel<<<grid, kBlock, 0, st>>>(h, static_cast<const __nv_bfloat16*>(w_down), cnt, row_off, touched,
                                                hdr, y, s->H, s->I);
  }
  return cudaGetLastError();
}

}  // namespace moe

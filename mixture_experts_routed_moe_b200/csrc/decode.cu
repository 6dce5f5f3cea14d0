// Small-token path: the expert matmuls as weight streaming ("Experts
// backends": the batched_mm backend is the fastest for small inputs and the
// decode-stage switch moves generation onto it; here the same per-token form
// is done without duplicating any parameters).
//
// With only a few tokens per expert, the layer is bound by reading each
// touched expert's weights once from HBM. Every warp owns a few consecutive
// weight rows of one touched expert, streams them with 16-byte no-L1 loads and
// dots them against all of that expert's tokens (kept in L1/L2), converting
// each weight chunk to fp32 once for all tokens. No tile padding, no tensor
// cores: the work is bound by HBM. The grid is exactly one wave of resident
// blocks.
//
//   gate/up:  h[row, n] = act(<x_t, Wg_e[n]>) * <x_t, Wu_e[n]>   (bf16)
//   down:     y[row, c] = <h[row], Wd_e[c]>                      (bf16)
//
// Rows are the unpadded expert-major permuted rows (tile size 1).
#include "decode_core.cuh"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 256;
constexpr int kWarpsPerBlock = kBlock / 32;

using dec::down_group;
using dec::gate_up_group;

__global__ void __launch_bounds__(kBlock) decode_gate_up_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wgu, const int* __restrict__ cnt,
    const int* __restrict__ row_off, const int* __restrict__ row_src, const int* __restrict__ touched,
    const int* __restrict__ hdr, __nv_bfloat16* __restrict__ h, int H, int I, int k, int act) {
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
    const __nv_bfloat16* w[8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      w[r] = wg + static_cast<size_t>(r) * H;
      w[4 + r] = wg + (static_cast<size_t>(I) + r) * H;
    }
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = x + static_cast<size_t>(row_src[r_e + g0 + min(q, ntok - 1)] / k) * H;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: gate_up_group<1>(w, a, nch, lane, h, row0, I, n0, act); break;
        case 2: gate_up_group<2>(w, a, nch, lane, h, row0, I, n0, act); break;
        case 3: gate_up_group<3>(w, a, nch, lane, h, row0, I, n0, act); break;
        default: gate_up_group<4>(w, a, nch, lane, h, row0, I, n0, act); break;
      }
    }
  }
}

// down: a task is (touched expert u, 8 consecutive rows c0..c0+7 of H).
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
    const __nv_bfloat16* w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = wd + (static_cast<size_t>(e) * H + c0 + r) * I;
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = h + static_cast<size_t>(r_e + g0 + min(q, ntok - 1)) * I;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: down_group<1>(w, a, nch, lane, y, row0, H, c0); break;
        case 2: down_group<2>(w, a, nch, lane, y, row0, H, c0); break;
        case 3: down_group<3>(w, a, nch, lane, y, row0, H, c0); break;
        default: down_group<4>(w, a, nch, lane, y, row0, H, c0); break;
      }
    }
  }
}

}  // namespace

bool decode_supported(const moe_shape*) { return true; }

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
  // exactly one wave of resident blocks: every warp starts at once and the
  // grid-stride task loop spreads the rows evenly over all of them
  static int per_sm[2] = {0, 0};  // resident blocks per SM (same on every B200)
  if (per_sm[which] == 0) {
    int n = 0;
    cudaError_t err = which == 0
                          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_gate_up_kernel, kBlock, 0)
                          : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_down_kernel, kBlock, 0);
    if (err != cudaSuccess) return err;
    per_sm[which] = n < 1 ? 1 : n;
  }
  const int grid = num_sms * per_sm[which];
  if (which == 0) {
    decode_gate_up_kernel<<<grid, kBlock, 0, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                   static_cast<const __nv_bfloat16*>(w_gate_up), cnt, row_off,
                                                   row_src, touched, hdr, h, s->H, s->I, s->k, s->act);
  } else {
    decode_down_kernel<<<grid, kBlock, 0, st>>>(h, static_cast<const __nv_bfloat16*>(w_down), cnt, row_off, touched,
                                                hdr, y, s->H, s->I);
  }
  return cudaGetLastError();
}

}  // namespace moe

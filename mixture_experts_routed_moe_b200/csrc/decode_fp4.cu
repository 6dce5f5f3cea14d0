// Small-token path for FP4 experts ("Experts backends", section "FP8 and FP4
// quantized experts": FP4-packed expert weights with power-of-two UE8M0
// scales). Weights are e2m1 codes, two per byte (even element in the low
// nibble), with one UE8M0 byte per row and block of 32 consecutive elements
// along the reduction dimension; activations stay bf16. As on the bf16
// small-token path, the layer is bound by reading each touched expert's
// weights once from HBM, now half a byte per weight.
//
// A 16-byte weight chunk holds 32 codes, exactly one scale block: each lane
// converts its chunk's codes once (e2m1 pairs -> f16 pairs -> fp32, exact),
// sums their products with every token's activations, and scales each
// per-chunk sum once by 2^(b-127).
//
//   gate/up:  h[row, n] = act(G) * U, G = sum_blk 2^(bg[blk]-127) * <x_t, codes of Wg[n] in blk>   (bf16)
//   down:     y[row, c] = sum_blk 2^(bd[blk]-127) * <h[row], codes of Wd[c] in blk>           (bf16)
#include <cuda_fp4.h>

#include "decode_core.cuh"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 256;
constexpr int kWarpsPerBlock = kBlock / 32;
// tokens dotted per pass over the weight rows (each adds 8 x 2 fp32 sums and
// 8 activation floats per lane; two keep the kernel at two blocks per SM
// without spills)
constexpr int kTokensPerPass = 2;

// The 8 e2m1 codes of one 32-bit word (lowest nibble first) as fp32.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t v, float (&f)[8]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const __half2 h2 = __half2(__nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>((v >> (8 * b)) & 0xFFu),
                                                          __NV_E2M1));
    const float2 f2 = __half22float2(h2);
    f[2 * b] = f2.x;
    f[2 * b + 1] = f2.y;
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  const uint32_t lo = (i & 1) ? v.y : v.x, hi = (i & 1) ? v.w : v.z;
  return (i & 2) ? hi : lo;
}

// The 8 weight rows of a task: rows 0..3 start at w0, rows 4..7 at w1, rows
// of one group `stride` bytes apart (packed codes); their scale rows likewise
// from s0, s1 with `sstride`. Two base addresses instead of 16 pointers keep
// the kernels at two blocks per SM without spills.
struct Rows8 {
  const uint8_t* w0;
  const uint8_t* w1;
  const uint8_t* s0;
  const uint8_t* s1;
  size_t stride, sstride;
};

// acc[r][q] += sum over this lane's chunks of 2^(b_r-127) * <codes of row r in
// the chunk, activation row q>: 8 weight rows, NQ activation rows (bf16).
template <int NQ>
__device__ __forceinline__ void dot_rows_fp4(const Rows8& rw, const __nv_bfloat16* const (&a)[kTokensPerPass],
                                             int nch, int lane, float (&acc)[8][NQ]) {
  for (int ch = lane; ch < nch; ch += 32) {
    uint4 wv[8];
    float sc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const size_t off = static_cast<size_t>(r & 3) * rw.stride + static_cast<size_t>(ch) * 16;
      wv[r] = ld_stream_u4((r < 4 ? rw.w0 : rw.w1) + off);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
      sc[r] = ue8m0_value(__ldg((r < 4 ? rw.s0 : rw.s1) + static_cast<size_t>(r & 3) * rw.sstride + ch));
    float part[8][NQ];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int q = 0; q < NQ; ++q) part[r][q] = 0.f;
#pragma unroll 1
    for (int sub = 0; sub < 4; ++sub) {  // 8 elements per step: one weight word, one activation uint4
      float xf[NQ][8];
#pragma unroll
      for (int q = 0; q < NQ; ++q) dec::unpack8(__ldg(reinterpret_cast<const uint4*>(a[q]) + ch * 4 + sub), xf[q]);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float wf[8];
        e2m1x8_to_f32(word_of(wv[r], sub), wf);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int i = 0; i < 8; ++i) part[r][q] = fmaf(wf[i], xf[q][i], part[r][q]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int q = 0; q < NQ; ++q) acc[r][q] = fmaf(sc[r], part[r][q], acc[r][q]);
  }
}

template <int NQ>
__device__ __forceinline__ void gate_up_group_fp4(const Rows8& rw, const __nv_bfloat16* const (&a)[kTokensPerPass],
                                                  int nch, int lane, __nv_bfloat16* h, size_t row0, int I, int n0,
                                                  int act) {
  float acc[8][NQ];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < NQ; ++q) acc[r][q] = 0.f;
  dot_rows_fp4<NQ>(rw, a, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float g = dec::warp_sum(acc[r][q]), u = dec::warp_sum(acc[4 + r][q]);
      if (lane == r) h[(row0 + q) * I + n0 + r] = __float2bfloat16_rn(gated_act(act, g, u));
    }
}

template <int NQ>
__device__ __forceinline__ void down_group_fp4(const Rows8& rw, const __nv_bfloat16* const (&a)[kTokensPerPass],
                                               int nch, int lane, __nv_bfloat16* y, size_t row0, int H, int c0) {
  float acc[8][NQ];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < NQ; ++q) acc[r][q] = 0.f;
  dot_rows_fp4<NQ>(rw, a, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float v = dec::warp_sum(acc[r][q]);
      if (lane == r) y[(row0 + q) * H + c0 + r] = __float2bfloat16_rn(v);
    }
}

// gate/up: a task is (touched expert u, 4 consecutive rows n0..n0+3 of I);
// weight rows 0..3 are gate rows n0.., rows 4..7 the up rows I+n0...
__global__ void __launch_bounds__(kBlock, 2) decode_fp4_gate_up_kernel(
    const __nv_bfloat16* __restrict__ x, const uint8_t* __restrict__ wgu, const uint8_t* __restrict__ sgu,
    const int* __restrict__ cnt, const int* __restrict__ row_off, const int* __restrict__ row_src,
    const int* __restrict__ touched, const int* __restrict__ hdr, __nv_bfloat16* __restrict__ h, int H, int I, int k,
    int act) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = I / 4;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = H / 32;  // 16-byte chunks (32 codes, one scale block) per row
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int n0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 4;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const size_t g_row = static_cast<size_t>(e) * 2 * I + n0;  // gate rows; the up rows follow I later
    const Rows8 rw{wgu + g_row * (H / 2), wgu + (g_row + I) * (H / 2), sgu + g_row * (H / 32),
                   sgu + (g_row + I) * (H / 32), static_cast<size_t>(H / 2), static_cast<size_t>(H / 32)};
    for (int g0 = 0; g0 < c_e; g0 += kTokensPerPass) {
      const int ntok = min(kTokensPerPass, c_e - g0);
      const __nv_bfloat16* a[kTokensPerPass];
#pragma unroll
      for (int q = 0; q < kTokensPerPass; ++q)
        a[q] = x + static_cast<size_t>(row_src[r_e + g0 + min(q, ntok - 1)] / k) * H;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      if (ntok == 1)
        gate_up_group_fp4<1>(rw, a, nch, lane, h, row0, I, n0, act);
      else
        gate_up_group_fp4<2>(rw, a, nch, lane, h, row0, I, n0, act);
    }
  }
}

// down: a task is (touched expert u, 8 consecutive rows c0..c0+7 of H).
__global__ void __launch_bounds__(kBlock, 2) decode_fp4_down_kernel(
    const __nv_bfloat16* __restrict__ h, const uint8_t* __restrict__ wd, const uint8_t* __restrict__ sd,
    const int* __restrict__ cnt, const int* __restrict__ row_off, const int* __restrict__ touched,
    const int* __restrict__ hdr, __nv_bfloat16* __restrict__ y, int H, int I) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = H / 8;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = I / 32;
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int c0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 8;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const size_t d_row = static_cast<size_t>(e) * H + c0;
    const Rows8 rw{wd + d_row * (I / 2), wd + (d_row + 4) * (I / 2), sd + d_row * (I / 32), sd + (d_row + 4) * (I / 32),
                   static_cast<size_t>(I / 2), static_cast<size_t>(I / 32)};
    for (int g0 = 0; g0 < c_e; g0 += kTokensPerPass) {
      const int ntok = min(kTokensPerPass, c_e - g0);
      const __nv_bfloat16* a[kTokensPerPass];
#pragma unroll
      for (int q = 0; q < kTokensPerPass; ++q) a[q] = h + static_cast<size_t>(r_e + g0 + min(q, ntok - 1)) * I;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      if (ntok == 1)
        down_group_fp4<1>(rw, a, nch, lane, y, row0, H, c0);
      else
        down_group_fp4<2>(rw, a, nch, lane, y, row0, H, c0);
    }
  }
}

}  // namespace

// which = 0: gate/up (x -> h); which = 1: down (h -> y).
cudaError_t launch_decode_fp4(const moe_shape* s, const Plan& p, const void* x, const void* w_gate_up,
                              const void* w_down, const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws,
                              int which, int num_sms, cudaStream_t st) {
  const int* cnt = reinterpret_cast<const int*>(ws + p.cnt);
  const int* row_off = reinterpret_cast<const int*>(ws + p.mt_base);  // tile size 1: offsets are rows
  const int* row_src = reinterpret_cast<const int*>(ws + p.row_src);
  const int* touched = reinterpret_cast<const int*>(ws + p.touched);
  const int* hdr = reinterpret_cast<const int*>(ws + p.hdr);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + p.h);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  static int per_sm[2] = {0, 0};  // resident blocks per SM: the grid is exactly one wave
  if (per_sm[which] == 0) {
    int n = 0;
    cudaError_t err = which == 0
                          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_fp4_gate_up_kernel, kBlock, 0)
                          : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_fp4_down_kernel, kBlock, 0);
    if (err != cudaSuccess) return err;
    per_sm[which] = n < 1 ? 1 : n;
  }
  const int grid = num_sms * per_sm[which];
  if (which == 0) {
    return launch_pdl(decode_fp4_gate_up_kernel, dim3(grid), dim3(kBlock), 0, st, static_cast<const __nv_bfloat16*>(x),
                      static_cast<const uint8_t*>(w_gate_up), sw_gate_up, cnt, row_off, row_src, touched, hdr, h, s->H,
                      s->I, s->k, s->act);
  }
  return launch_pdl(decode_fp4_down_kernel, dim3(grid), dim3(kBlock), 0, st, h, static_cast<const uint8_t*>(w_down),
                    sw_down, cnt, row_off, touched, hdr, y, s->H, s->I);
}

}  // namespace moe

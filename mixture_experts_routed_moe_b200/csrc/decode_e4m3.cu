// Small-token path for FP8 experts ("Experts backends", section "FP8 and FP4
// quantized experts": e4m3 weights with one power-of-two UE8M0 scale per
// 128x128 block; activations quantised per row in 1x128 groups with fp32
// scales). As on the bf16 small-token path, the layer is bound by reading each
// touched expert's weights once from HBM, so the e4m3 codes are streamed with
// 16-byte no-L1 loads and dotted on the CUDA cores against that expert's few
// rows; no tile padding, no tensor cores.
//
//   x:       codes xq[t, :] and fp32 group scales xs[t, kb] of each token t,
//            quantised once by the permute stage; row `row` (expert-major, tile
//            size 1) belongs to token t = row_src[row] / k
//   gate/up: hf[row, n] = act(G) * U, with
//            G = sum_kb 2^(bg[kb]-127) * xs[t, kb] * <xq[t, block kb], Wg[n, block kb]>
//            and U likewise from the up rows                          (fp32)
//   quant:   hq[row, :], hs[row, :] = 1x128 quantisation of hf, the rule
//            the permute stage applies to x                            (e4m3)
//   down:    y[row, c] = sum_kb 2^(bd[kb]-127) * hs[row, kb] * <hq[row, block kb], Wd[c, block kb]>
//                                                                      (bf16)
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 256;
constexpr int kWarpsPerBlock = kBlock / 32;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// acc[r][q] += 2^(b_r - 127) * s_q * <weight row r, activation row q> over
// this lane's 16-byte chunks. A chunk holds 16 codes and lies in 128-column
// block ch / 8, so one weight scale (shared by the kG rows of a scale group,
// srow[r / kG][kb]) and one activation scale (as[q][kb]) apply to the whole
// chunk: its 16 products are summed first, then scaled once. Every weight and
// activation word is converted to fp32 once per chunk.
template <int NR, int kG, int NQ>
__device__ __forceinline__ void dot_rows_e4m3(const uint8_t* const (&w)[NR], const uint8_t* const (&srow)[NR / kG],
                                              const uint8_t* const (&a)[4], const float* const (&as)[4], int nch,
                                              int lane, float (&acc)[NR][4]) {
  for (int ch = lane; ch < nch; ch += 32) {
    uint4 wv[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) wv[r] = ld_stream_u4(w[r] + static_cast<size_t>(ch) * 16);
    const int kb = ch >> 3;
    float wsc[NR / kG];
#pragma unroll
    for (int g = 0; g < NR / kG; ++g) wsc[g] = ue8m0_value(__ldg(srow[g] + kb));
    uint4 xv[NQ];
    float xsc[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      xv[q] = __ldg(reinterpret_cast<const uint4*>(a[q]) + ch);
      xsc[q] = __ldg(as[q] + kb);
    }
    float part[NR][NQ];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int q = 0; q < NQ; ++q) part[r][q] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float xf[NQ][4];
#pragma unroll
      for (int q = 0; q < NQ; ++q) e4m3x4_to_f32(word_of(xv[q], j), xf[q]);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        float wf[4];
        e4m3x4_to_f32(word_of(wv[r], j), wf);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int i = 0; i < 4; ++i) part[r][q] = fmaf(wf[i], xf[q][i], part[r][q]);
      }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int q = 0; q < NQ; ++q) acc[r][q] = fmaf(part[r][q], wsc[r / kG] * xsc[q], acc[r][q]);
  }
}

// gate/up: a task is (touched expert u, 4 consecutive rows n0..n0+3 of I);
// weight rows 0..3 are gate rows n0.. (scale group 0), rows 4..7 the up rows
// I+n0.. (scale group 1). n0 is a multiple of 4, so each group lies in one
// 128-row scale block.
template <int NQ>
__device__ __forceinline__ void gate_up_group(const uint8_t* const (&w)[8], const uint8_t* const (&srow)[2],
                                              const uint8_t* const (&a)[4], const float* const (&as)[4], int nch,
                                              int lane, float* hf, size_t row0, int I, int n0, int act) {
  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
  dot_rows_e4m3<8, 4, NQ>(w, srow, a, as, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float g = warp_sum(acc[r][q]), u = warp_sum(acc[4 + r][q]);
      if (lane == r) hf[(row0 + q) * I + n0 + r] = gated_act(act, g, u);
    }
}

__global__ void __launch_bounds__(kBlock, 2) decode_e4m3_gate_up_kernel(
    const uint8_t* __restrict__ xq, const float* __restrict__ xs, const uint8_t* __restrict__ wgu,
    const uint8_t* __restrict__ sgu, const int* __restrict__ cnt, const int* __restrict__ row_off,
    const int* __restrict__ row_src, const int* __restrict__ touched, const int* __restrict__ hdr,
    float* __restrict__ hf, int H, int I, int k, int act) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = I / 4;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = H / 16;  // 16-byte chunks per weight row
  const int KB = H / 128;  // scale columns per weight block row
  const int SB = 2 * I / 128;  // scale block rows per expert
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int n0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 4;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const uint8_t* w[8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      w[r] = wgu + (static_cast<size_t>(e) * 2 * I + n0 + r) * H;
      w[4 + r] = wgu + (static_cast<size_t>(e) * 2 * I + I + n0 + r) * H;
    }
    const uint8_t* srow[2] = {sgu + (static_cast<size_t>(e) * SB + n0 / 128) * KB,
                              sgu + (static_cast<size_t>(e) * SB + (I + n0) / 128) * KB};
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const uint8_t* a[4];
      const float* as[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const size_t t = static_cast<size_t>(row_src[r_e + g0 + min(q, ntok - 1)] / k);
        a[q] = xq + t * H;
        as[q] = xs + t * KB;
      }
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: gate_up_group<1>(w, srow, a, as, nch, lane, hf, row0, I, n0, act); break;
        case 2: gate_up_group<2>(w, srow, a, as, nch, lane, hf, row0, I, n0, act); break;
        case 3: gate_up_group<3>(w, srow, a, as, nch, lane, hf, row0, I, n0, act); break;
        default: gate_up_group<4>(w, srow, a, as, nch, lane, hf, row0, I, n0, act); break;
      }
    }
  }
}

// One warp per (row, 128-column group) of hf: s = amax/448 in fp32 (1 for an
// all-zero group), codes e4m3(h/s) with IEEE division, round to nearest even,
// saturating. Each lane owns 4 consecutive columns.
__global__ void __launch_bounds__(kBlock) decode_e4m3_quant_h_kernel(const float* __restrict__ hf,
                                                                      uint8_t* __restrict__ hq,
                                                                      float* __restrict__ hs, long long rows, int I) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long gwarp = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  const long long nwarps = static_cast<long long>(gridDim.x) * kWarpsPerBlock;
  const int G = I / 128;
  const long long total = rows * G;
  for (long long t = gwarp; t < total; t += nwarps) {
    const long long row = t / G;
    const int g = static_cast<int>(t - row * G);
    const size_t at = static_cast<size_t>(row) * I + g * 128 + lane * 4;
    const float4 v = *reinterpret_cast<const float4*>(hf + at);
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const GroupDivisor dv = make_group_divisor(sc);
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(group_div(dv, v.x), group_div(dv, v.y)),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(group_div(dv, v.z), group_div(dv, v.w)),
                                                 __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(hq + at) = lo | (hi << 16);
    if (lane == 0) hs[static_cast<size_t>(row) * G + g] = sc;
  }
}

// down: a task is (touched expert u, 8 consecutive rows c0..c0+7 of H), one
// scale group (c0 is a multiple of 8, so the rows share a 128-row block).
template <int NQ>
__device__ __forceinline__ void down_group(const uint8_t* const (&w)[8], const uint8_t* const (&srow)[1],
                                           const uint8_t* const (&a)[4], const float* const (&as)[4], int nch,
                                           int lane, __nv_bfloat16* y, size_t row0, int H, int c0) {
  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
  dot_rows_e4m3<8, 8, NQ>(w, srow, a, as, nch, lane, acc);
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float v = warp_sum(acc[r][q]);
      if (lane == r) y[(row0 + q) * H + c0 + r] = __float2bfloat16_rn(v);
    }
}

__global__ void __launch_bounds__(kBlock, 2) decode_e4m3_down_kernel(
    const uint8_t* __restrict__ hq, const float* __restrict__ hs, const uint8_t* __restrict__ wd,
    const uint8_t* __restrict__ sd, const int* __restrict__ cnt, const int* __restrict__ row_off,
    const int* __restrict__ touched, const int* __restrict__ hdr, __nv_bfloat16* __restrict__ y, int H, int I) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerBlock;
  const int n_touched = hdr[kHdrTouched];
  const int row_groups = H / 8;
  const long long total = static_cast<long long>(n_touched) * row_groups;
  const int nch = I / 16;
  const int KB = I / 128;
  const int SB = H / 128;
  for (long long task = gwarp; task < total; task += nwarps) {
    const int u = static_cast<int>(task / row_groups);
    const int c0 = static_cast<int>(task - static_cast<long long>(u) * row_groups) * 8;
    const int e = touched[u];
    const int c_e = cnt[e];
    const int r_e = row_off[e];
    const uint8_t* w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = wd + (static_cast<size_t>(e) * H + c0 + r) * I;
    const uint8_t* srow[1] = {sd + (static_cast<size_t>(e) * SB + c0 / 128) * KB};
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const uint8_t* a[4];
      const float* as[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const size_t row = static_cast<size_t>(r_e + g0 + min(q, ntok - 1));
        a[q] = hq + row * I;
        as[q] = hs + row * KB;
      }
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: down_group<1>(w, srow, a, as, nch, lane, y, row0, H, c0); break;
        case 2: down_group<2>(w, srow, a, as, nch, lane, y, row0, H, c0); break;
        case 3: down_group<3>(w, srow, a, as, nch, lane, y, row0, H, c0); break;
        default: down_group<4>(w, srow, a, as, nch, lane, y, row0, H, c0); break;
      }
    }
  }
}

template <typename K>
cudaError_t one_wave(K kernel, int* cached, int num_sms, int* grid) {
  if (*cached == 0) {
    int n = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kBlock, 0);
    if (err != cudaSuccess) return err;
    *cached = n < 1 ? 1 : n;
  }
  *grid = num_sms * *cached;
  return cudaSuccess;
}

}  // namespace

// which = 0: gate/up (xq -> hf) then the h quantisation (hf -> hq, hs);
// which = 1: down (hq -> y).
cudaError_t launch_decode_e4m3(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                               const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws, int which,
                               int num_sms, cudaStream_t st) {
  const int* cnt = reinterpret_cast<const int*>(ws + p.cnt);
  const int* row_off = reinterpret_cast<const int*>(ws + p.mt_base);  // tile size 1: offsets are rows
  const int* row_src = reinterpret_cast<const int*>(ws + p.row_src);
  const int* touched = reinterpret_cast<const int*>(ws + p.touched);
  const int* hdr = reinterpret_cast<const int*>(ws + p.hdr);
  const uint8_t* xq = ws + p.xa;
  const float* xs = reinterpret_cast<const float*>(ws + p.xs);
  float* hf = reinterpret_cast<float*>(ws + p.hf);
  uint8_t* hq = ws + p.h;
  float* hs = reinterpret_cast<float*>(ws + p.hs);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  static int per_sm[3] = {0, 0, 0};  // resident blocks per SM (same on every B200)
  int grid = 0;
  cudaError_t err;
  if (which == 0) {
    err = one_wave(decode_e4m3_gate_up_kernel, &per_sm[0], num_sms, &grid);
    if (err != cudaSuccess) return err;
    err = launch_pdl(decode_e4m3_gate_up_kernel, dim3(grid), dim3(kBlock), 0, st, xq, xs,
                     static_cast<const uint8_t*>(w_gate_up), sw_gate_up, cnt, row_off, row_src, touched, hdr, hf, s->H,
                     s->I, s->k, s->act);
    if (err != cudaSuccess) return err;
    err = one_wave(decode_e4m3_quant_h_kernel, &per_sm[1], num_sms, &grid);
    if (err != cudaSuccess) return err;
    const long long groups = p.m_rows * (s->I / 128);
    const long long need = (groups + kWarpsPerBlock - 1) / kWarpsPerBlock;
    grid = static_cast<int>(need < grid ? (need < 1 ? 1 : need) : grid);
    return launch_pdl(decode_e4m3_quant_h_kernel, dim3(grid), dim3(kBlock), 0, st, hf, hq, hs, p.m_rows, s->I);
  } else {
    err = one_wave(decode_e4m3_down_kernel, &per_sm[2], num_sms, &grid);
    if (err != cudaSuccess) return err;
    return launch_pdl(decode_e4m3_down_kernel, dim3(grid), dim3(kBlock), 0, st, hq, hs,
                      static_cast<const uint8_t*>(w_down), sw_down, cnt, row_off, touched, hdr, y, s->H, s->I);
  }
}

}  // namespace moe

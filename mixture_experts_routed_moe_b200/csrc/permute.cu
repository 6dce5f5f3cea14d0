// Expert-major permutation of the T*k assignments ("Experts backends",
// backend table rows grouped_mm / deepgemm: tokens are sorted by their
// selected expert so that one grouped GEMM covers every expert; the deepgemm
// row aligns each expert's block to the GEMM tile).
//
// Layout produced (deterministic, independent of thread timing): expert e owns
// rows [mt_base[e]*bm, mt_base[e+1]*bm), with mt_base the exclusive prefix sum
// of ceil(cnt[e]/bm); inside an expert the assignments appear in ascending
// token order; pad rows hold row_src = -1.
//
// The rank of assignment (t, j) inside its expert is the number of tokens
// t' < t that chose the same expert. It is computed without any ordering
// races: each warp of a 256-token block sets, per expert, a 32-bit mask of its
// lanes (tokens) that chose the expert; a token's rank inside the block is the
// population count of the masks of earlier warps plus the bits of earlier
// lanes in its own warp, and blocks are offset by an exclusive scan of the
// per-block counts.
#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = kPermuteTokens / 32;  // 8 warps, one token per thread
// the single-block permute stages rows itself up to this many elements (a few
// loads per warp); larger volumes go to stage_rows_kernel
constexpr long long kSmallStageElems = 32768;

// Phase 1 of the block-level count: per-warp expert masks in shared memory.
// Records kDevErrIndex for an index outside [0,E) or a repeated expert.
__device__ __forceinline__ void build_masks(uint32_t* s_mask, const int* __restrict__ idx, int t, bool active, int k,
                                            int E, int warp, int lane, int* dev_status) {
  if (!active) return;
  for (int j = 0; j < k; ++j) {
    const int e = idx[static_cast<size_t>(t) * k + j];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
      const uint32_t old = atomicOr(&s_mask[warp * E + e], 1u << lane);
      if (old & (1u << lane)) atomicOr(dev_status, kDevErrIndex);
    } else {
      atomicOr(dev_status, kDevErrIndex);
    }
  }
}

__device__ __forceinline__ int rank_in_block(const uint32_t* s_mask, int e, int E, int warp, int lane) {
  int r = 0;
  for (int w = 0; w < warp; ++w) r += __popc(s_mask[w * E + e]);
  return r + __popc(s_mask[warp * E + e] & ((1u << lane) - 1u));
}

__global__ void __launch_bounds__(kPermuteTokens) permute_count_kernel(const int* __restrict__ idx, int T, int k,
                                                                       int E, int* __restrict__ block_counts,
                                                                       int* __restrict__ local_rank,
                                                                       int* dev_status) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  extern __shared__ uint32_t s_mask[];  // [kWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * E; i += kPermuteTokens) s_mask[i] = 0;
  __syncthreads();
  const int t = blockIdx.x * kPermuteTokens + threadIdx.x;
  const bool active = t < T;
  build_masks(s_mask, idx, t, active, k, E, warp, lane, dev_status);
  __syncthreads();
  if (active) {
    for (int j = 0; j < k; ++j) {
      const size_t a = static_cast<size_t>(t) * k + j;
      const int e = idx[a];
      local_rank[a] = (static_cast<unsigned>(e) < static_cast<unsigned>(E)) ? rank_in_block(s_mask, e, E, warp, lane)
                                                                             : 0;
    }
  }
  for (int e = threadIdx.x; e < E; e += kPermuteTokens) {
    int c = 0;
    for (int w = 0; w < kWarps; ++w) c += __popc(s_mask[w * E + e]);
    block_counts[static_cast<size_t>(blockIdx.x) * E + e] = c;
  }
}

// Inclusive scan of one value per thread over a block of up to 1024 threads.
__device__ __forceinline__ int block_inclusive_scan(int v, int* s_warp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int w = (lane < nw) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const int r = v + (warp > 0 ? s_warp[warp - 1] : 0);
  __syncthreads();
  return r;
}

// Per-expert totals (thread e), expert offsets, pad rows and the list of
// experts that received tokens. `counts` holds per-block counts on entry and
// per-block exclusive bases on exit. Runs as one block of 1024 threads.
__device__ __forceinline__ void scan_experts(int* __restrict__ counts, int nblk, int E, int bm, int* __restrict__ cnt,
                                             int* __restrict__ mt_base, int* __restrict__ pt_base,
                                             int* __restrict__ touched, int* __restrict__ hdr,
                                             int* __restrict__ row_src, int* s_warp) {
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    // exclusive prefix over the blocks, eight independent loads in flight at a
    // time (one dependent load per block made this a chain of global latencies)
    for (int b0 = 0; b0 < nblk; b0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = b0 + j < nblk ? counts[static_cast<size_t>(b0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (b0 + j < nblk) counts[static_cast<size_t>(b0 + j) * E + e] = c;
        c += v[j];
      }
    }
    cnt[e] = c;
  }
  const int tiles = (e < E) ? (c + bm - 1) / bm : 0;
  const int used = (e < E && c > 0) ? 1 : 0;
  const int pairs = (tiles + 1) / 2;  // 256-row tile pairs of the 2-CTA GEMM
  const int tiles_incl = block_inclusive_scan(tiles, s_warp);
  const int used_incl = block_inclusive_scan(used, s_warp);
  const int pairs_incl = block_inclusive_scan(pairs, s_warp);
  if (e < E) {
    const int base = tiles_incl - tiles;
    mt_base[e] = base;
    pt_base[e] = pairs_incl - pairs;
    if (used) touched[used_incl - 1] = e;
    for (int r = base * bm + c; r < (base + tiles) * bm; ++r) row_src[r] = -1;
    if (e == E - 1) {
      mt_base[E] = tiles_incl;
      pt_base[E] = pairs_incl;
      hdr[kHdrMTiles] = tiles_incl;
      hdr[kHdrTouched] = used_incl;
      hdr[kHdrRows] = tiles_incl * bm;
      hdr[kHdrPairs] = pairs_incl;
    }
  }
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(int* counts, int nblk, int E, int bm, int* cnt,
                                                            int* mt_base, int* pt_base, int* touched, int* hdr,
                                                            int* row_src) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  __shared__ int s_warp[32];
  scan_experts(counts, nblk, E, bm, cnt, mt_base, pt_base, touched, hdr, row_src, s_warp);
}

// Copy one assignment's bf16 hidden-state row into its permuted row (one warp).
__device__ __forceinline__ void copy_row_bf16(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ xa,
                                              int t, int row, int H, int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  uint4* dst = reinterpret_cast<uint4*>(xa + static_cast<size_t>(row) * H);
  for (int c = lane; c < H / 8; c += 32) dst[c] = __ldg(src + c);
}

// Quantise one 128-column group of a bf16 row with one half-warp (lane l16
// holds columns 8*l16 .. 8*l16+7, in v): scale s = amax/448 in fp32 (1 for
// an all-zero group) and codes e4m3(x/s) of the IEEE quotient, round to nearest
// even, saturating -- the FP8 experts' dynamic per-row activation scales.
__device__ __forceinline__ uint2 quant_group_codes(const uint4& v, unsigned hmask, float* sc_out) {
  const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(hmask, amax, o));
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const GroupDivisor dv = make_group_divisor(sc);
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(group_div(dv, f[4 * i]), group_div(dv, f[4 * i + 1])),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(group_div(dv, f[4 * i + 2]), group_div(dv, f[4 * i + 3])), __NV_SATFINITE, __NV_E4M3);
    w[i] = lo | (hi << 16);
  }
  *sc_out = sc;
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void quant_group_e4m3(const uint4& v, unsigned hmask, int l16, uint2* dst, float* scale) {
  float sc;
  *dst = quant_group_codes(v, hmask, &sc);
  if (l16 == 0) *scale = sc;
}

// Quantise one token's row into permuted row `row` (one warp; each half-warp
// owns one group at a time).
__device__ __forceinline__ void quant_row_e4m3(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ xq,
                                               float* __restrict__ xs, int t, int row, int H, int lane) {
  const int half = lane >> 4, l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (16 * half);
  const int G = H / 128;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  for (int g = half; g < G; g += 2)
    quant_group_e4m3(__ldg(src + g * 16 + l16), hmask, l16,
                     reinterpret_cast<uint2*>(xq + static_cast<size_t>(row) * H + g * 128) + l16,
                     xs + static_cast<size_t>(row) * G + g);
}

// Copies (bf16, into xa) or quantises (e4m3, into xq/xs) activation rows, one
// half-warp per (source, 128-column group) task spread over many blocks, so
// the row traffic is not left to the single block of the small permute.
// With slot_row the sources are assignments a (token a / k, destination row
// slot_row[a], skipped when negative); without it they are tokens, each
// written once to row t (the e4m3 DECODE path reads x per token).
__global__ void __launch_bounds__(256) stage_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const int* __restrict__ slot_row, long long n_src, int k,
                                                         int H, __nv_bfloat16* __restrict__ xa,
                                                         uint8_t* __restrict__ xq, float* __restrict__ xs) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int G = H / 128;
  const long long total = n_src * G;
  const int l16 = threadIdx.x & 15;
  const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x / 16);
  for (long long task = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 16; task < total;
       task += stride) {
    const long long a = task / G;
    const int g = static_cast<int>(task - a * G);
    long long row = a, t = a;
    if (slot_row != nullptr) {
      row = slot_row[a];
      t = a / k;
      if (row < 0) continue;  // the whole half-warp skips together
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + g * 128) + l16);
    if (xa != nullptr)
      reinterpret_cast<uint4*>(xa + static_cast<size_t>(row) * H + g * 128)[l16] = v;
    else
      quant_group_e4m3(v, hmask, l16, reinterpret_cast<uint2*>(xq + static_cast<size_t>(row) * H + g * 128) + l16,
                       xs + static_cast<size_t>(row) * G + g);
  }
}

// One warp per token: writes row_src / slot_row of the token's k assignments
// and, when xa is given, copies the token's hidden state into each of their
// permuted rows (or, when xq is given, quantises it once and writes the codes
// and group scales to each row). The token row is read once per 32
// assignments, not once per assignment.
__global__ void __launch_bounds__(256) permute_scatter_kernel(const int* __restrict__ idx, int T, int k, int E, int bm,
                                                              const int* __restrict__ block_base,
                                                              const int* __restrict__ local_rank,
                                                              const int* __restrict__ mt_base,
                                                              int* __restrict__ row_src, int* __restrict__ slot_row,
                                                              const __nv_bfloat16* __restrict__ x,
                                                              __nv_bfloat16* __restrict__ xa, uint8_t* __restrict__ xq,
                                                              float* __restrict__ xs, int H) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long t = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const int b = static_cast<int>(t / kPermuteTokens);
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  const int G = H / 128;
  const int half = lane >> 4, l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (16 * half);
  for (int j0 = 0; j0 < k; j0 += 32) {
    const int nj = min(32, k - j0);
    int row = -1;
    if (lane < nj) {
      const long long a = t * k + j0 + lane;
      const int e = idx[a];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        row = mt_base[e] * bm + block_base[static_cast<size_t>(b) * E + e] + local_rank[a];
        row_src[row] = static_cast<int>(a);
      }
      slot_row[a] = row;
    }
    if (xa != nullptr) {
      // uniform trip count (H/8 need not be a multiple of 32): every lane
      // reaches the full-warp row broadcasts
      const int nc = H / 8;
      uint4 vn = lane < nc ? __ldg(src + lane) : make_uint4(0u, 0u, 0u, 0u);
      for (int c0 = 0; c0 < nc; c0 += 32) {
        const int c = c0 + lane;
        const uint4 v = vn;  // the next chunk's load is in flight while this one is stored
        if (c + 32 < nc) vn = __ldg(src + c + 32);
        for (int j = 0; j < nj; ++j) {
          const int r = __shfl_sync(0xffffffffu, row, j);
          if (r >= 0 && c < nc) reinterpret_cast<uint4*>(xa + static_cast<size_t>(r) * H)[c] = v;
        }
      }
    }
    if (xq != nullptr) {
      // both half-warps run the same number of iterations (G rounded up to
      // even), so the full-warp row broadcasts below stay converged
      uint4 vn = half < G ? __ldg(src + half * 16 + l16) : make_uint4(0u, 0u, 0u, 0u);
      for (int g0 = 0; g0 < G; g0 += 2) {
        const int g = g0 + half;
        const uint4 v = vn;  // the next group's load is in flight while this one is quantised
        if (g + 2 < G) vn = __ldg(src + (g + 2) * 16 + l16);
        uint2 codes = make_uint2(0u, 0u);
        float sc = 1.f;
        if (g < G) codes = quant_group_codes(v, hmask, &sc);
        for (int j = 0; j < nj; ++j) {
          const int r = __shfl_sync(0xffffffffu, row, j);
          if (r >= 0 && g < G) {
            reinterpret_cast<uint2*>(xq + static_cast<size_t>(r) * H + g * 128)[l16] = codes;
            if (l16 == 0) xs[static_cast<size_t>(r) * G + g] = sc;
          }
        }
      }
    }
  }
}

// Everything in one block of 1024 threads, for T <= kPermuteTokens.
__global__ void __launch_bounds__(1024) permute_small_kernel(const int* __restrict__ idx, int T, int k, int E, int bm,
                                                             int* __restrict__ cnt, int* __restrict__ mt_base,
                                                             int* __restrict__ pt_base,
                                                             int* __restrict__ touched, int* __restrict__ hdr,
                                                             int* __restrict__ row_src, int* __restrict__ slot_row,
                                                             int* __restrict__ local_rank, int* dev_status,
                                                             const __nv_bfloat16* __restrict__ x,
                                                             __nv_bfloat16* __restrict__ xa, uint8_t* __restrict__ xq,
                                                             float* __restrict__ xs, int H) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  extern __shared__ uint32_t s_mask[];  // [kWarps][E]
  __shared__ int s_warp[32];
  __shared__ int s_base[1024];  // per-expert block base is always 0 here; holds mt_base*bm
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) s_mask[i] = 0;
  __syncthreads();
  const int t = threadIdx.x;
  const bool active = t < T;  // T <= 256: warps 0..7 hold the tokens
  build_masks(s_mask, idx, t, active, k, E, warp, lane, dev_status);
  __syncthreads();
  if (active) {
    for (int j = 0; j < k; ++j) {
      const int a = t * k + j;
      const int e = idx[a];
      local_rank[a] = (static_cast<unsigned>(e) < static_cast<unsigned>(E)) ? rank_in_block(s_mask, e, E, warp, lane)
                                                                             : 0;
    }
  }
  // per-expert totals from the masks
  int c = 0;
  if (threadIdx.x < E)
    for (int w = 0; w < kWarps; ++w) c += __popc(s_mask[w * E + threadIdx.x]);
  const int e = threadIdx.x;
  const int tiles = (e < E) ? (c + bm - 1) / bm : 0;
  const int used = (e < E && c > 0) ? 1 : 0;
  const int pairs = (tiles + 1) / 2;
  const int tiles_incl = block_inclusive_scan(tiles, s_warp);
  const int used_incl = block_inclusive_scan(used, s_warp);
  const int pairs_incl = block_inclusive_scan(pairs, s_warp);
  if (e < E) {
    const int base = tiles_incl - tiles;
    cnt[e] = c;
    mt_base[e] = base;
    pt_base[e] = pairs_incl - pairs;
    s_base[e] = base * bm;
    if (used) touched[used_incl - 1] = e;
    for (int r = base * bm + c; r < (base + tiles) * bm; ++r) row_src[r] = -1;
    if (e == E - 1) {
      mt_base[E] = tiles_incl;
      pt_base[E] = pairs_incl;
      hdr[kHdrMTiles] = tiles_incl;
      hdr[kHdrTouched] = used_incl;
      hdr[kHdrRows] = tiles_incl * bm;
      hdr[kHdrPairs] = pairs_incl;
    }
  }
  __syncthreads();
  // scatter: one warp per assignment
  for (int a = warp; a < T * k; a += 32) {
    const int e2 = idx[a];
    if (static_cast<unsigned>(e2) >= static_cast<unsigned>(E)) {
      if (lane == 0) slot_row[a] = -1;
      continue;
    }
    const int row = s_base[e2] + local_rank[a];
    if (lane == 0) {
      row_src[row] = a;
      slot_row[a] = row;
    }
    if (xa != nullptr) copy_row_bf16(x, xa, a / k, row, H, lane);
    if (xq != nullptr) quant_row_e4m3(x, xq, xs, a / k, row, H, lane);
  }
}

}  // namespace

cudaError_t launch_permute(const moe_shape* s, const Plan& p, const int* topk_idx, const void* x, uint8_t* ws,
                           cudaStream_t st) {
  const int T = s->T, k = s->k, E = s->E, H = s->H;
  int* status = reinterpret_cast<int*>(ws + p.status);
  int* hdr = reinterpret_cast<int*>(ws + p.hdr);
  int* counts = reinterpret_cast<int*>(ws + p.block_counts);
  int* cnt = reinterpret_cast<int*>(ws + p.cnt);
  int* mt_base = reinterpret_cast<int*>(ws + p.mt_base);
  int* pt_base = reinterpret_cast<int*>(ws + p.pt_base);
  int* touched = reinterpret_cast<int*>(ws + p.touched);
  int* lrank = reinterpret_cast<int*>(ws + p.local_rank);
  int* row_src = reinterpret_cast<int*>(ws + p.row_src);
  int* slot_row = reinterpret_cast<int*>(ws + p.slot_row);
  const bool fp8 = s->wdtype == MOE_DT_E4M3;
  const bool prefill = p.path == MOE_PATH_PREFILL;
  // PREFILL: x copied (bf16) or quantised (e4m3) into the permuted rows;
  // e4m3 DECODE: x quantised once per token; bf16 DECODE: x copied into the
  // expert-major rows for the tensor-core kernels, else read in place
  const bool copy_x = (prefill || p.tc_stream) && !fp8;
  __nv_bfloat16* xa = copy_x ? reinterpret_cast<__nv_bfloat16*>(ws + p.xa) : nullptr;
  uint8_t* xq = fp8 ? ws + p.xa : nullptr;
  float* xs = fp8 ? reinterpret_cast<float*>(ws + p.xs) : nullptr;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const size_t mask_bytes = sizeof(uint32_t) * kWarps * E;
  const long long A = static_cast<long long>(T) * k;
  const int G = H / 128;
  // rows are staged by the permute kernels themselves only where that is
  // short: the single-block permute for at most kSmallStageElems elements
  const bool stage_in_small = (prefill || copy_x) && A * H <= kSmallStageElems;
  auto stage = [&](const int* slots, long long n_src) -> cudaError_t {
    const long long tasks = n_src * G;
    const long long want = (tasks + 15) / 16;  // blocks of 16 half-warps
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    const unsigned grid = static_cast<unsigned>(std::max<long long>(1, std::min(want, cap)));
    return launch_pdl(stage_rows_kernel, dim3(grid), dim3(256), 0, st, xb, slots, n_src, k, H, xa, xq, xs);
  };

  cudaError_t err = cudaMemsetAsync(status, 0, kStatusWordsZeroed * sizeof(int), st);
  if (err != cudaSuccess) return err;
  if (T <= kSmallPermuteT) {
    err = launch_pdl(permute_small_kernel, dim3(1), dim3(1024), mask_bytes, st, topk_idx, T, k, E, p.bm, cnt, mt_base,
                     pt_base, touched, hdr, row_src, slot_row, lrank, status, xb, stage_in_small ? xa : nullptr,
                     stage_in_small ? xq : nullptr, stage_in_small ? xs : nullptr, H);
    if (err != cudaSuccess) return err;
    if (stage_in_small || (!prefill && !fp8 && !copy_x)) return cudaSuccess;
    return (prefill || copy_x) ? stage(slot_row, A) : stage(nullptr, T);
  }
  err = launch_pdl(permute_count_kernel, dim3(p.nblk), dim3(kPermuteTokens), mask_bytes, st, topk_idx, T, k, E, counts,
                   lrank, status);
  if (err != cudaSuccess) return err;
  err = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, st, counts, p.nblk, E, p.bm, cnt, mt_base, pt_base,
                   touched, hdr, row_src);
  if (err != cudaSuccess) return err;
  err = launch_pdl(permute_scatter_kernel, dim3(static_cast<unsigned>((T + 7) / 8)), dim3(256), 0, st, topk_idx, T, k,
                   E, p.bm, counts, lrank, mt_base, row_src, slot_row, xb, xa, prefill ? xq : nullptr,
                   prefill ? xs : nullptr, H);
  if (err != cudaSuccess) return err;
  return (!prefill && fp8) ? stage(nullptr, T) : cudaSuccess;
}

}  // namespace moe

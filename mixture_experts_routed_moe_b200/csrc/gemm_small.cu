// Small-token expert GEMMs on the tensor cores, operands swapped ("Experts
// backends": small inputs favour the per-token batched form, and the
// decode-stage switch moves generation onto it; here the few tokens of an
// expert become the MMA's N instead of being padded to a 128-row tile).
//
//   gate/up:  h[r, n] = act(<x_r, Wg_e[n]>) * <x_r, Wu_e[n]>   (bf16)
//   down:     y[r, c] = <h_r, Wd_e[c]>                         (bf16)
//
// for the expert-major rows r of expert e (tile size 1, no padding). A unit of
// work is (touched expert, block of 128 weight rows): the weight rows are the
// MMA's M = 128 and the A operand, the expert's token rows (up to 128 per
// pass, padded to a multiple of 16) its N and the B operand, K the hidden (or
// intermediate) dimension, streamed by TMA in 64-wide steps. The gate/up unit
// issues two MMAs per step, the 128 gate rows into accumulator columns
// [0, N) and the matching 128 up rows into [N, 2N), so one thread (one TMEM
// lane = one weight row) holds both halves of its h column. Each weight byte
// is read once per pass; the expert's token rows come from L2.
//
// Warp roles (192 threads, one CTA per SM, persistent over the units): warp 0
// TMA producer, warp 1 TMEM allocator and MMA issuer, warps 2..5 epilogue
// (warp w reads TMEM lanes 32*(w%4)..+31). Two accumulator buffers let the
// epilogue of one unit overlap the next unit's MMAs. Every wait is bounded.
#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBK = 64;        // bf16 K elements per stage: one 128-byte swizzle row
constexpr int kM = 128;        // weight rows per MMA
constexpr int kMaxN = 128;     // token rows per pass
constexpr int kNBox = 16;      // token rows per TMA box
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kATile = kM * kBK * 2;         // 16 KB
constexpr int kBBox = kNBox * kBK * 2;       // 2 KB
constexpr int kBTile = kMaxN * kBK * 2;      // 16 KB

template <bool kGateUp>
struct SmallCfg {
  static constexpr int kNumA = kGateUp ? 2 : 1;
  static constexpr int kStage = kNumA * kATile + kBTile;  // 48 or 32 KB
  static constexpr int kStages = kGateUp ? 4 : 6;
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStage + (2 * kStages + 5) * 8 + 16;
};

struct SmallParams {
  const int* cnt;
  const int* row_off;  // [E+1] first row of each expert (tile size 1)
  const int* touched;  // touched experts, in expert order
  const int* hdr;
  int n_rb;              // blocks of 128 weight rows per expert: I/128 (gate/up) or H/128 (down)
  int num_kb;            // K / 64
  int w_rows_per_expert; // 2I (gate/up) or H (down)
  int w_second_offset;   // gate/up: rows from a gate row to its up row (I)
  __nv_bfloat16* out;    // h [A, I] or y [A, H]
  int out_ld;
  int* dev_status;
  unsigned long long timeout_ns;
};

// The job sequence every role walks in the same order: unit u (touched
// expert u / n_rb, row block u % n_rb), then its passes of up to kMaxN tokens.
struct Job {
  int e, rb, row0, n_valid, n;  // expert, row block, first token row, tokens in the pass, MMA N
};

__device__ __forceinline__ bool next_job(const SmallParams& p, int n_units, int& unit, int& pass, Job& j) {
  while (unit < n_units) {
    const int u = unit / p.n_rb;
    const int e = p.touched[u];
    const int c = p.cnt[e];
    const int first = pass * kMaxN;
    if (first < c) {
      j.e = e;
      j.rb = unit - u * p.n_rb;
      j.row0 = p.row_off[e] + first;
      j.n_valid = min(kMaxN, c - first);
      j.n = (j.n_valid + kNBox - 1) / kNBox * kNBox;
      ++pass;
      return true;
    }
    unit += gridDim.x;
    pass = 0;
  }
  return false;
}

template <bool kGateUp, int kAct>
__global__ void __launch_bounds__(kThreads, 1)
    small_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const SmallParams p) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  using C = SmallCfg<kGateUp>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* empty = full + C::kStages;
  uint64_t* afull = empty + C::kStages;  // [2]
  uint64_t* aempty = afull + 2;          // [2]
  uint64_t* drain = aempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int n_units = p.hdr[kHdrTouched] * p.n_rb;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_w = l2_policy_evict_first();  // every weight byte is read once
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      int unit = blockIdx.x, pass = 0;
      Job j;
      while (ok && next_job(p, n_units, unit, pass, j)) {
        const int wrow = j.e * p.w_rows_per_expert + j.rb * kM;
        const int nbox = j.n / kNBox;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::kStage;
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(C::kNumA * kATile + nbox * kBBox));
          tma_load_2d_hint(st, &tmW, &full[stage], kb * kBK, wrow, pol_w);
          if (kGateUp) tma_load_2d_hint(st + kATile, &tmW, &full[stage], kb * kBK, wrow + p.w_second_offset, pol_w);
          uint8_t* sb = st + C::kNumA * kATile;
          for (int b = 0; b < nbox; ++b) tma_load_2d(sb + b * kBBox, &tmX, &full[stage], kb * kBK, j.row0 + b * kNBox);
          if (++stage == C::kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        for (int i = 0; i < C::kStages; ++i) {
          if (--stage < 0) {
            stage = C::kStages - 1;
            ph ^= 1;
          }
          int never = 0;
          mbar_wait_bounded(&full[stage], ph, &never, p.dev_status, 1000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      int unit = blockIdx.x, pass = 0;
      Job j;
      while (ok && next_job(p, n_units, unit, pass, j)) {
        if (!mbar_wait_bounded(&aempty[acc], aph ^ 1, s_abort, p.dev_status, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * 256);
        const uint32_t idesc = idesc_bf16_f32(kM, j.n);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], ph, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStage);
          const uint32_t b0 = a0 + C::kNumA * kATile;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
            umma_bf16(d, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc, accum);
            if (kGateUp)
              umma_bf16(d + static_cast<uint32_t>(j.n), sdesc_kmajor_sw128(a0 + kATile + k * 32),
                        sdesc_kmajor_sw128(b0 + k * 32), idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&afull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      // every MMA issued above has finished once this commit arrives
      umma_commit(drain);
      int never = 0;
      mbar_wait_bounded(drain, 0, &never, p.dev_status, p.timeout_ns);
    }
  } else {
    // ---------------- epilogue: one weight row per thread, one token per column ----------------
    const int quad = warp & 3;
    const int i = quad * 32 + lane;  // weight row in the block = output column in the block
    int acc = 0;
    uint32_t aph = 0;
    int unit = blockIdx.x, pass = 0;
    Job j;
    while (next_job(p, n_units, unit, pass, j)) {
      const bool got = mbar_wait_bounded(&afull[acc], aph, s_abort, p.dev_status, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got) || *s_abort != 0) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * 256);
      __nv_bfloat16* o = p.out + static_cast<size_t>(j.row0) * p.out_ld + j.rb * kM + i;
      for (int t0 = 0; t0 < j.n_valid; t0 += 16) {
        uint32_t v[16];
        tmem_ld16(tb + static_cast<uint32_t>(t0), v);
        if (kGateUp) {
          uint32_t u[16];
          tmem_ld16(tb + static_cast<uint32_t>(j.n + t0), u);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (t0 + c < j.n_valid)
              o[static_cast<size_t>(t0 + c) * p.out_ld] =
                  __float2bfloat16_rn(gated_act_t<kAct>(__uint_as_float(v[c]), __uint_as_float(u[c])));
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (t0 + c < j.n_valid) o[static_cast<size_t>(t0 + c) * p.out_ld] = __float2bfloat16_rn(__uint_as_float(v[c]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <bool kGateUp, int kAct>
cudaError_t launch_small_t(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallParams& sp, int grid,
                           cudaStream_t st) {
  using C = SmallCfg<kGateUp>;
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(small_gemm_bf16_kernel<kGateUp, kAct>), &done);
  if (err != cudaSuccess) return err;
  return launch_pdl(small_gemm_bf16_kernel<kGateUp, kAct>, dim3(grid), dim3(kThreads), C::kSmem, st, tmW, tmX, sp);
}

}  // namespace

bool small_gemm_supported(const moe_shape* s) {
  return s->wdtype == MOE_DT_BF16 && s->H % kM == 0 && s->I % kM == 0;
}

// which = 0: gate/up (x rows -> h); which = 1: down (h -> y). The expert-major
// token rows of x (tile size 1) are in the workspace's xa.
cudaError_t launch_small_gemm(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                              uint8_t* ws, int which, int num_sms, cudaStream_t st) {
  const int H = s->H, I = s->I, E = s->E;
  const uint64_t A = static_cast<uint64_t>(p.m_rows);
  SmallParams sp{};
  sp.cnt = reinterpret_cast<const int*>(ws + p.cnt);
  sp.row_off = reinterpret_cast<const int*>(ws + p.mt_base);  // tile size 1: offsets are rows
  sp.touched = reinterpret_cast<const int*>(ws + p.touched);
  sp.hdr = reinterpret_cast<const int*>(ws + p.hdr);
  sp.dev_status = reinterpret_cast<int*>(ws + p.status);
  sp.timeout_ns = wait_limit_ns();
  CUtensorMap tmW, tmX;
  // enough units for every SM when all experts are touched; idle CTAs exit at once
  if (which == 0) {
    if (!encode_tensor_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_gate_up, H,
                              static_cast<uint64_t>(E) * 2 * I, kBK, kM) ||
        !encode_tensor_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.xa, H, A, kBK, kNBox))
      return cudaErrorInvalidValue;
    sp.n_rb = I / kM;
    sp.num_kb = H / kBK;
    sp.w_rows_per_expert = 2 * I;
    sp.w_second_offset = I;
    sp.out = reinterpret_cast<__nv_bfloat16*>(ws + p.h);
    sp.out_ld = I;
    const int grid = std::max(1, std::min(num_sms, E * sp.n_rb));
    switch (s->act) {
      case MOE_ACT_GELU: return launch_small_t<true, MOE_ACT_GELU>(tmW, tmX, sp, grid, st);
      case MOE_ACT_RELU: return launch_small_t<true, MOE_ACT_RELU>(tmW, tmX, sp, grid, st);
      default: return launch_small_t<true, MOE_ACT_SILU>(tmW, tmX, sp, grid, st);
    }
  }
  if (!encode_tensor_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_down, I, static_cast<uint64_t>(E) * H, kBK,
                            kM) ||
      !encode_tensor_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, A, kBK, kNBox))
    return cudaErrorInvalidValue;
  sp.n_rb = H / kM;
  sp.num_kb = I / kBK;
  sp.w_rows_per_expert = H;
  sp.w_second_offset = 0;
  sp.out = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  sp.out_ld = H;
  const int grid = std::max(1, std::min(num_sms, E * sp.n_rb));
  return launch_small_t<false, 0>(tmW, tmX, sp, grid, st);
}

}  // namespace moe

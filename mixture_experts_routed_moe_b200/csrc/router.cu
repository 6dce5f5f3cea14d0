// Router GEMM fused with the top-k routing: logits = x W_r^T, then the routing
// of every token on those logits ("Experts backends", introduction: a router
// picks k experts per token; backend table, row "sonicmoe", fuses the router
// dispatch with the expert GEMMs).
//
//   logits[t, e] = sum_h x[t, h] * W_r[e, h]      bf16 inputs, fp32 accumulate
//   (topk_idx, topk_w)[t] = route_token(logits[t])  (route_core.cuh)
//
// One CTA per 128 tokens, one tile: the token rows are the MMA's M = 128, the
// E router rows (padded to N = a multiple of 16, at most 256) its N, and H its
// K, streamed by TMA through a 4-stage shared-memory ring into
// tcgen05.mma.kind::f16 with the fp32 accumulator in TMEM. When the last MMA
// has landed the ring is free: the epilogue warps move the accumulator rows
// from TMEM into shared memory (and, if asked, to the caller's fp32 logits),
// then all six warps route the tile's tokens from shared memory, one warp per
// token. Rows beyond E in the padded tile are zero (TMA fills out-of-range rows
// with zeros) and are never read by the routing.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// MMA issuer, warps 2..5 epilogue (warp w reads TMEM lanes 32*(w%4)..+31);
// then all sixteen warps route the tile's 128 tokens, eight each (the routing
// of a token is a chain of warp reductions, so more warps in flight is what
// shortens the tile's tail).
#include "moe_common.cuh"
#include "moe_internal.h"
#include "route_core.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;       // K elements per stage (128 bytes of bf16: one swizzle row)
constexpr int kMaxStages = 8;
constexpr size_t kRingBytes = 192 * 1024;  // shared memory for the TMA ring
constexpr int kThreads = 512;
constexpr int kRows = 128;    // tokens per CTA (MMA M)
constexpr int kA = kRows * kBK * 2;  // 16 KB

struct RouterParams {
  int T, H, E, k;
  int n_pad;        // E rounded up to a multiple of 16 (MMA N)
  uint32_t n_alloc; // TMEM columns allocated (power of two >= 32)
  float* logits;    // [T, E] fp32, or null
  int* idx;         // [T, k]
  float* w;         // [T, k]
  unsigned long long timeout_ns;
};

// As many stages as fit the ring (the kernel is bound by the bytes one CTA
// keeps in flight): 6 for E <= 128, 8 for E <= 64, 4 for E = 256.
__host__ __device__ constexpr int router_stages(int n_pad) {
  return static_cast<int>(kRingBytes / static_cast<size_t>(kA + n_pad * kBK * 2)) < kMaxStages
             ? static_cast<int>(kRingBytes / static_cast<size_t>(kA + n_pad * kBK * 2))
             : kMaxStages;
}

__host__ __device__ constexpr size_t router_smem_bytes(int n_pad) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(router_stages(n_pad)) * (kA + n_pad * kBK * 2) +
         (2 * kMaxStages + 1) * 8 + 16;
}

template <int kPerLane>
__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const RouterParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int kB = p.n_pad * kBK * 2;
  const int kStages = router_stages(p.n_pad);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kB);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  // no workspace, so no device status word: the bounded waits record into
  // this shared word and a wait that gives up marks the tile's tokens instead
  int* s_status = reinterpret_cast<int*>(s_tmem + 2);
  // after the last MMA the ring holds the tile's logits, row stride n_pad + 1
  // floats (an odd stride keeps the epilogue's row-per-thread stores free of
  // bank conflicts)
  float* s_logits = reinterpret_cast<float*>(smem);
  const int ld = p.n_pad + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int num_kb = p.H / kBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    *s_abort = 0;
    *s_status = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, p.n_alloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t ph = 0;
      int kb = 0;
      for (; kb < num_kb; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, s_status, p.timeout_ns)) break;
        mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(kA + kB));
        tma_load_2d(sA + stage * kA, &tmX, &full[stage], kb * kBK, row0);
        tma_load_2d(sB + stage * kB, &tmW, &full[stage], kb * kBK, 0);
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
      if (kb < num_kb) {
        // let the copies already issued land before the shared memory is reused
        for (int i = 0; i < kStages; ++i) {
          if (--stage < 0) {
            stage = kStages - 1;
            ph ^= 1;
          }
          int never = 0;
          mbar_wait_bounded(&full[stage], ph, &never, s_status, 1000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16_f32(kRows, p.n_pad);
      int stage = 0;
      uint32_t ph = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait_bounded(&full[stage], ph, s_abort, s_status, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * kA);
        const uint32_t b0 = smem_u32(sB + stage * kB);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16(tmem_base, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc,
                    (kb | k) != 0 ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
      // every MMA issued above has finished once this commit arrives
      umma_commit(tfull);
    }
  } else {
    // ---------------- epilogue: TMEM -> shared (and global) logits ----------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool got = mbar_wait_bounded(tfull, 0, s_abort, s_status, p.timeout_ns) && *s_abort == 0;
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      const int t = row0 + r;
      float* grow = (p.logits != nullptr && t < p.T) ? p.logits + static_cast<size_t>(t) * p.E : nullptr;
      for (int c = 0; c < p.n_pad; c += 16) {
        uint32_t v[16];
        tmem_ld16(tb + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float f = __uint_as_float(v[i]);
          s_logits[r * ld + c + i] = f;
          if (grow != nullptr && c + i < p.E) grow[c + i] = f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---------------- routing: one warp per token of the tile, every warp ----------------
  const int rows = min(kRows, p.T - row0);
  if (*s_abort != 0) {
    // a bounded wait gave up (never in normal operation): mark the tokens
    for (int i = threadIdx.x; i < rows * p.k; i += kThreads) p.idx[static_cast<size_t>(row0) * p.k + i] = -1;
  } else {
    for (int tl = warp; tl < rows; tl += kThreads / 32) {
      const size_t t = static_cast<size_t>(row0 + tl);
      route_token<kPerLane>(s_logits + tl * ld, p.E, p.k, lane, p.idx + t * p.k, p.w + t * p.k);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.n_alloc);
  }
}

template <int kPerLane>
cudaError_t launch_router_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const RouterParams& p, int grid,
                            cudaStream_t st) {
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(router_kernel<kPerLane>), &done);
  if (err != cudaSuccess) return err;
  router_kernel<kPerLane><<<grid, kThreads, router_smem_bytes(p.n_pad), st>>>(tmX, tmW, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const void* x, const void* w_router, int T, int H, int E, int k, float* logits, int* idx,
                          float* w, cudaStream_t st) {
  RouterParams p{};
  p.T = T;
  p.H = H;
  p.E = E;
  p.k = k;
  p.n_pad = (E + 15) / 16 * 16;
  uint32_t n_alloc = 32;
  while (n_alloc < static_cast<uint32_t>(p.n_pad)) n_alloc <<= 1;
  p.n_alloc = n_alloc;
  p.logits = logits;
  p.idx = idx;
  p.w = w;
  p.timeout_ns = wait_limit_ns();
  CUtensorMap tmX, tmW;
  if (!encode_tensor_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, H, T, kBK, kRows) ||
      !encode_tensor_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_router, H, E, kBK, p.n_pad))
    return cudaErrorInvalidValue;
  const int grid = (T + kRows - 1) / kRows;
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) return launch_router_t<1>(tmX, tmW, p, grid, st);
  if (per_lane <= 2) return launch_router_t<2>(tmX, tmW, p, grid, st);
  if (per_lane <= 4) return launch_router_t<4>(tmX, tmW, p, grid, st);
  return launch_router_t<8>(tmX, tmW, p, grid, st);
}

}  // namespace moe

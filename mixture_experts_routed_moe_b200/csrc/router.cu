// Router GEMM fused with the top-k routing: logits = x W_r^T, then the routing
// of every token on those logits ("Experts backends", introduction: a router
// picks k experts per token; backend table, row "sonicmoe", fuses the router
// dispatch with the expert GEMMs).
//
//   logits[t, e] = sum_h x[t, h] * W_r[e, h]      bf16 inputs, fp32 accumulate
//   (topk_idx, topk_w)[t] = route_token(logits[t])  (route_core.cuh)
//
// A cluster of C CTAs (C = 1, 2, 4 or 8, chosen so that the grid covers the
// SMs) owns one tile of 128 tokens; CTA r of the cluster takes the r-th of C
// consecutive ranges of the K dimension. The token rows are the MMA's M = 128,
// the E router rows (padded to N = a multiple of 16, at most 256) its N, and
// the K range is streamed by TMA through a shared-memory ring into
// tcgen05.mma.kind::f16 with the fp32 partial in TMEM. When the last MMA has
// landed the ring is free: the epilogue warps move the partial rows from TMEM
// into shared memory. After a cluster barrier CTA r routes the r-th 128/C of
// the tile's tokens: each token's logit row is the sum of the C partial rows,
// read through distributed shared memory in rank order (one fixed order, so
// the result is deterministic), written to the caller's logits if asked and
// routed from shared memory by one warp per token. Rows beyond E in the padded
// tile are zero (TMA fills out-of-range rows with zeros) and never read.
//
// Warp roles (1024 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// MMA issuer, warps 2..5 epilogue (warp w reads TMEM lanes 32*(w%4)..+31);
// then all 32 warps route the CTA's share of the tokens, one warp per token.
#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "route_core.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;       // K elements per stage (128 bytes of bf16: one swizzle row)
constexpr int kMaxStages = 8;
constexpr size_t kRingBytes = 192 * 1024;  // shared memory for the TMA ring
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 128;    // tokens per tile (MMA M)
constexpr int kA = kRows * kBK * 2;  // 16 KB
constexpr int kMaxCluster = 8;

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
// keeps in flight): 8 for E <= 64, 6 for E <= 128, 4 for E = 256.
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
  // after the last MMA the ring holds this CTA's partial logits, row stride
  // n_pad + 4 floats (16-byte rows, and eight consecutive rows start in eight
  // different 16-byte bank groups, so the epilogue's row-per-thread 16-byte
  // stores are free of bank conflicts), then one summed row per warp
  float* s_part = reinterpret_cast<float*>(smem);
  const int ld = p.n_pad + 4;
  float* s_row = s_part + kRows * ld;  // [kWarps][n_pad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int csize = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int row0 = (blockIdx.x / csize) * kRows;
  const int num_kb = p.H / kBK;
  // this CTA's K range (every CTA gets at least one K block: the host keeps C <= H/64)
  const int kb0 = rank * num_kb / csize, kb1 = (rank + 1) * num_kb / csize;
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
      int kb = kb0;
      for (; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, s_status, p.timeout_ns)) break;
        mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(kA + kB));
        tma_load_2d(sA + stage * kA, &tmX, &full[stage], kb * kBK, row0);
        tma_load_2d(sB + stage * kB, &tmW, &full[stage], kb * kBK, 0);
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
      if (kb < kb1) {
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
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&full[stage], ph, s_abort, s_status, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * kA);
        const uint32_t b0 = smem_u32(sB + stage * kB);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16(tmem_base, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc,
                    (kb > kb0 || k != 0) ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
      // every MMA issued above has finished once this commit arrives
      umma_commit(tfull);
    }
  } else if (warp < 6) {
    // ---------------- epilogue: TMEM -> this CTA's partial rows in shared memory ----------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool got = mbar_wait_bounded(tfull, 0, s_abort, s_status, p.timeout_ns) && *s_abort == 0;
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      for (int c = 0; c < p.n_pad; c += 16) {
        uint32_t v[16];
        tmem_ld16(tb + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(s_part + r * ld + c + i) =
              make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                          __uint_as_float(v[i + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // every CTA of the cluster has its partial rows in shared memory
  cluster_sync();

  // ---------------- routing of this CTA's share of the tile, one warp per token ----------------
  const int rows = min(kRows, p.T - row0);
  const int per = kRows / csize;
  const int first = rank * per, last = min(rows, first + per);
  bool aborted = false;
  for (int q = 0; q < csize; ++q)
    aborted |= ld_cluster_s32(cluster_map(smem_u32(const_cast<int*>(s_abort)), static_cast<uint32_t>(q))) != 0;
  if (aborted) {
    // a bounded wait gave up somewhere in the cluster (never in normal operation): mark the tokens
    for (int i = first * p.k + threadIdx.x; i < last * p.k; i += kThreads)
      p.idx[static_cast<size_t>(row0) * p.k + i] = -1;
  } else {
    float* srow = s_row + warp * p.n_pad;
    for (int tl = first + warp; tl < last; tl += kWarps) {
      const size_t t = static_cast<size_t>(row0 + tl);
      const uint32_t base = smem_u32(s_part + tl * ld);
      // four consecutive experts per lane, the C partials added in rank order
      for (int e = 4 * lane; e < p.n_pad; e += 128) {
        float4 v = ld_cluster_f32x4(cluster_map(base + 4u * e, 0u));
        for (int q = 1; q < csize; ++q) {
          const float4 u = ld_cluster_f32x4(cluster_map(base + 4u * e, static_cast<uint32_t>(q)));
          v.x += u.x;
          v.y += u.y;
          v.z += u.z;
          v.w += u.w;
        }
        *reinterpret_cast<float4*>(srow + e) = v;
        if (p.logits != nullptr) {
          const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (e + i < p.E) p.logits[t * p.E + e + i] = f[i];
        }
      }
      __syncwarp();
      route_token<kPerLane>(srow, p.E, p.k, lane, p.idx + t * p.k, p.w + t * p.k);
      __syncwarp();
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.n_alloc);
  }
}

// Cluster size: the largest of 8, 4, 2 whose clusters (one per 128-token tile)
// the device holds at once and that leaves every CTA at least one K block
// (and at least 16 of the tile's tokens to route); else 1.
int router_cluster_size(const void* kernel, int tiles, int num_kb, size_t smem) {
  for (int c = kMaxCluster; c > 1; c >>= 1) {
    if (c > num_kb || kRows / c < 16) continue;
    const int n = max_active_clusters(kernel, c, kThreads, smem);
    if (n > 0 && tiles <= n) return c;
  }
  return 1;
}

template <int kPerLane>
cudaError_t launch_router_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const RouterParams& p, int tiles,
                            cudaStream_t st) {
  const void* fn = reinterpret_cast<const void*>(router_kernel<kPerLane>);
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(fn, &done);  // before the occupancy query below
  if (err != cudaSuccess) return err;
  const size_t smem = router_smem_bytes(p.n_pad);
  const int csize = router_cluster_size(fn, tiles, p.H / kBK, smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * csize), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = router_smem_bytes(p.n_pad);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_kernel<kPerLane>, tmX, tmW, p);
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
  const int tiles = (T + kRows - 1) / kRows;
  const int per_lane = (E + 31) / 32;
  // the partial rows and the per-warp summed rows reuse the ring
  if (static_cast<size_t>(kRows) * (p.n_pad + 4) * 4 + static_cast<size_t>(kWarps) * p.n_pad * 4 >
      static_cast<size_t>(router_stages(p.n_pad)) * (kA + p.n_pad * kBK * 2))
    return cudaErrorInvalidValue;
  if (per_lane <= 1) return launch_router_t<1>(tmX, tmW, p, tiles, st);
  if (per_lane <= 2) return launch_router_t<2>(tmX, tmW, p, tiles, st);
  if (per_lane <= 4) return launch_router_t<4>(tmX, tmW, p, tiles, st);
  return launch_router_t<8>(tmX, tmW, p, tiles, st);
}

}  // namespace moe

// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA. One persistent kernel serves both projections of the expert MLP
// ("Experts backends", backend table: the expert is up projection, SwiGLU,
// down projection; grouped_mm / deepgemm run all experts in one grouped GEMM
// over expert-sorted tokens):
//
//   gate/up:  h[rows of e, n..n+127] = act(X_e Wg_e^T) * (X_e Wu_e^T)   (SwiGLU/GeGLU/ReGLU in the epilogue)
//   down:     y[rows of e, n..n+N-1] = h_e Wd_e^T
//
// Tile = (expert e, 128-row block of e's permuted rows, N-column block). The
// tile list is only known on the device (expert counts come from routing), so
// each CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ... and maps a tile
// number to (e, m, n) with the per-expert tile prefix sum. Within an expert the
// N blocks are the outer loop and the row blocks the inner one, so CTAs that
// run at the same time share weight tiles through L2. The gate/up projection
// of many small experts runs in clusters of two CTAs that walk the tiles
// together, one N block each, so they also share the activation rows.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0      TMA producer: A tile [128 x 64] and B tile [N x 64] per stage
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 MMAs of K=16 per stage
//   warps 2..9  epilogue: TMEM -> registers -> act(gate)*up / bf16 -> a
//               64-byte-swizzled staging tile in shared memory -> TMA tile
//               store; two warps per TMEM lane quadrant, half the columns each
//               (with four, the epilogue took as long as a tile's MMAs)
// Shared memory holds a 4-stage ring; TMEM holds two accumulators of N fp32
// columns so the epilogue of one tile overlaps the MMAs of the next.
// For gate/up, B stacks the 128 gate rows n..n+127 (expert rows n) over the 128
// up rows (expert rows I+n), and one MMA with N=256 produces both halves.
#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;  // bf16 elements per 128-byte row of a stage
constexpr int kStages = 4;
constexpr int kThreads = 320;  // producer, MMA issuer, 8 epilogue warps
constexpr int kEpiWarps = 8;

struct GemmParams {
  const int* mt_base;  // [E+1] per-expert 128-row tile prefix
  const int* cnt;      // [E]
  int E;
  int stage_bufs;  // staging tiles per epilogue warp (2 when shared memory allows, else 1)
  int num_kb;             // K / 64
  int n_tiles;            // N blocks per expert
  int b_rows_per_expert;  // rows of one expert's B matrix
  int b_tile_stride;      // B rows between consecutive N blocks
  int b_second_offset;    // B rows from the first to the second 128-row half (N = 256)
  __nv_bfloat16* out;
  int out_ld;         // elements per output row
  int out_tile_cols;  // output columns per tile
  int act;  // gate activation (moe_activation)
  int* dev_status;
  unsigned long long timeout_ns;
  int stall_loads;  // failure-detection test: the producer issues nothing
  int cs;           // CTAs per cluster sharing one row block (1: no clusters)
};

// The tiles of CTA `rank` in a cluster of cs CTAs: the cluster walks groups
// (expert, row block, cs consecutive column blocks) and its CTA `rank` takes
// column block group * cs + rank, so the cs CTAs stream the same activation
// rows at the same time and all but the first find them in L2. False when
// that column block does not exist (the last group of an expert may be short).
__device__ __forceinline__ bool cluster_tile(int g, int rank, int cs, const int* s_mt, const int* s_cnt, int E,
                                             int NT, TileCoord* c) {
  *c = tile_coord(g, s_mt, s_cnt, E, (NT + cs - 1) / cs);
  c->n = c->n * cs + rank;
  return c->n < NT;
}

constexpr int kStageBox = 32 * 64;  // one staging tile: 32 rows x 32 bf16 columns (64-byte rows)

template <int kN>
struct Layout {
  static constexpr int kA = kTileM * kBK * 2;  // 16 KB
  static constexpr int kB = kN * kBK * 2;      // 32 KB for N = 256
  static constexpr int kStage = kA + kB;
  static constexpr int kBarriers = 2 * kStages + 5;
  static constexpr size_t bytes(int E, int bufs) {
    return 1024 /*alignment slack*/ + static_cast<size_t>(kStages) * kStage +
           static_cast<size_t>(kEpiWarps) * bufs * kStageBox + kBarriers * 8 + 16 +
           static_cast<size_t>(2 * E + 1) * 4;
  }
};

// Converts 32 fp32 columns of one row per lane to bf16 and stores the warp's
// 32 x 32 tile at (x, y) of `map` through the staging buffer `stg` (the TMA
// store that last read it must be done, which the caller waits for).
__device__ __forceinline__ void store_box_bf16(const CUtensorMap* map, uint8_t* stg, const uint32_t (&pk)[16],
                                               bool store, int x, int y, int lane) {
  const uint32_t sb = smem_u32(stg);
#pragma unroll
  for (int i = 0; i < 4; ++i) st_shared_v4(sb + sw64_offset(lane, i), pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  fence_proxy_async_shared();
  __syncwarp();
  if (lane == 0 && store) {
    tma_store_2d(map, stg, x, y);
    bulk_commit_group();
  }
}

// Staging-buffer rotation of one epilogue warp: wait until the next buffer is
// free (no TMA store still reads it) and return it.
__device__ __forceinline__ uint8_t* next_stage(uint8_t* stage0, int bufs, int& buf, int lane) {
  if (lane == 0) {
    if (bufs == 2)
      bulk_wait_group_read<1>();
    else
      bulk_wait_group_read<0>();
  }
  __syncwarp();
  uint8_t* stg = stage0 + buf * kStageBox;
  buf = (buf + 1) % bufs;
  return stg;
}

// act(gate) * up for this thread's row: TMEM columns [64*half, 64*half+64) of
// the gate block and the same of the up block, stored as 64 bf16 h values at
// columns x0 .. x0+63 of rows y0 .. y0+31 (the warp's rows).
template <int kAct>
__device__ __forceinline__ void epilogue_gated(uint32_t tb, int half, const CUtensorMap* map, uint8_t* stage0,
                                               int bufs, int& buf, bool store, int x0, int y0, int lane) {
#pragma unroll 1
  for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
    uint32_t g[32], u[32];
    tmem_ld32(tb + cc * 32, g);
    tmem_ld32(tb + 128 + cc * 32, u);
    tmem_ld_wait();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(gated_act_t<kAct>(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                          gated_act_t<kAct>(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
    uint8_t* stg = next_stage(stage0, bufs, buf, lane);
    store_box_bf16(map, stg, pk, store, x0 + (cc - 2 * half) * 32, y0, lane);
  }
}

template <int kN, bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  using L = Layout<kN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * L::kA;
  uint8_t* sO = sB + kStages * L::kB;  // [8 warps][stage_bufs][kStageBox]
  uint64_t* full = reinterpret_cast<uint64_t*>(sO + kEpiWarps * p.stage_bufs * kStageBox);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [2]
  uint64_t* tempty = tfull + 2;       // [2]
  uint64_t* drain = tempty + 2;       // [1]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_mt = reinterpret_cast<int*>(s_tmem + 4);
  int* s_cnt = s_mt + p.E + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i <= p.E; i += kThreads) s_mt[i] = p.mt_base[i];
  for (int i = threadIdx.x; i < p.E; i += kThreads) s_cnt[i] = p.cnt[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 2 * kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int NT = p.n_tiles;
  const int total = s_mt[p.E] * ((NT + p.cs - 1) / p.cs);  // tile groups
  const int rank = static_cast<int>(blockIdx.x) % p.cs;      // CTA rank in its cluster
  const int first = static_cast<int>(blockIdx.x) / p.cs, step = static_cast<int>(gridDim.x) / p.cs;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_a = l2_policy_evict_last();
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int g = first; ok && !p.stall_loads && g < total; g += step) {
        TileCoord c;
        if (!cluster_tile(g, rank, p.cs, s_mt, s_cnt, p.E, NT, &c)) continue;
        const int brow = c.e * p.b_rows_per_expert + c.n * p.b_tile_stride;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kStage);
          // A rows are re-read by every N block of the expert: ask L2 to keep them
          tma_load_2d_hint(sA + stage * L::kA, &tmA, &full[stage], kb * kBK, c.row0, pol_a);
          tma_load_2d(sB + stage * L::kB, &tmB, &full[stage], kb * kBK, brow);
          if (kN == 256)
            tma_load_2d(sB + stage * L::kB + 128 * kBK * 2, &tmB, &full[stage], kb * kBK, brow + p.b_second_offset);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        for (int i = 0; i < kStages; ++i) {
          if (--stage < 0) {
            stage = kStages - 1;
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
      constexpr uint32_t idesc = idesc_bf16_f32(kTileM, kN);
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int g = first; ok && g < total; g += step) {
        TileCoord c;
        if (!cluster_tile(g, rank, p.cs, s_mt, s_cnt, p.E, NT, &c)) continue;
        if (!mbar_wait_bounded(&tempty[acc], aph ^ 1, s_abort, p.dev_status, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * kN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], ph, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kA);
          const uint32_t b0 = smem_u32(sB + stage * L::kB);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc,
                      (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      // every MMA issued above has finished once this commit arrives
      umma_commit(drain);
      int never = 0;
      mbar_wait_bounded(drain, 0, &never, p.dev_status, p.timeout_ns);
    }
  } else {
    // ---------------- epilogue ----------------
    // two warps per TMEM lane quadrant (a warp may only read lanes
    // 32*(warp%4) .. +31), each converting half of the tile's columns
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    uint8_t* stage0 = sO + (warp - 2) * p.stage_bufs * kStageBox;
    int buf = 0;
    int acc = 0;
    uint32_t aph = 0;
    for (int g = first; g < total; g += step) {
      TileCoord c;
      if (!cluster_tile(g, rank, p.cs, s_mt, s_cnt, p.E, NT, &c)) continue;
      const bool got = mbar_wait_bounded(&tfull[acc], aph, s_abort, p.dev_status, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * kN);
      // the warp's 32 rows are stored whole: rows past the expert's count are
      // pad rows of its own last block, which no later stage reads
      const int y0 = c.row0 + quad * 32;
      const int x0 = c.n * p.out_tile_cols + half * (kSwiGLU ? 64 : kN / 2);
      if constexpr (kSwiGLU) {
        // gate columns 0..127, up columns 128..255 of the accumulator
        switch (p.act) {
          case MOE_ACT_GELU: epilogue_gated<MOE_ACT_GELU>(tb, half, &tmO, stage0, p.stage_bufs, buf, true, x0, y0, lane); break;
          case MOE_ACT_RELU: epilogue_gated<MOE_ACT_RELU>(tb, half, &tmO, stage0, p.stage_bufs, buf, true, x0, y0, lane); break;
          default: epilogue_gated<MOE_ACT_SILU>(tb, half, &tmO, stage0, p.stage_bufs, buf, true, x0, y0, lane); break;
        }
      } else {
        constexpr int kChunks = kN / 32 / 2;  // 32-column chunks per half
#pragma unroll 1
        for (int cc = half * kChunks; cc < (half + 1) * kChunks; ++cc) {
          uint32_t v[32];
          tmem_ld32(tb + cc * 32, v);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          uint8_t* stg = next_stage(stage0, p.stage_bufs, buf, lane);
          store_box_bf16(&tmO, stg, pk, true, x0 + (cc - half * kChunks) * 32, y0, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
    if (lane == 0) bulk_wait_group<0>();  // every store of this warp has landed
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kN);
  }
}

template <int kN, bool kSwiGLU>
cudaError_t launch_one(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmO, GemmParams gp,
                       int grid, cudaStream_t st) {
  gp.stage_bufs = Layout<kN>::bytes(gp.E, 2) <= kSmemLimit ? 2 : 1;
  const size_t smem = Layout<kN>::bytes(gp.E, gp.stage_bufs);
  if (smem > kSmemLimit) return cudaErrorInvalidValue;
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(grouped_gemm_bf16_kernel<kN, kSwiGLU>), &done);
  if (err != cudaSuccess) return err;
  if (gp.cs == 1) {
    grouped_gemm_bf16_kernel<kN, kSwiGLU><<<grid, kThreads, smem, st>>>(tmA, tmB, tmO, gp);
    return cudaGetLastError();
  }
  // every cluster of the persistent grid must be resident at once: with an
  // odd SM count in a GPC, fewer than num_sms / cs clusters fit
  const int maxc = max_active_clusters(reinterpret_cast<const void*>(grouped_gemm_bf16_kernel<kN, kSwiGLU>), gp.cs,
                                       kThreads, smem);
  if (maxc > 0) grid = std::min(grid, gp.cs * maxc);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);  // a multiple of gp.cs
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(gp.cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_bf16_kernel<kN, kSwiGLU>, tmA, tmB, tmO, gp);
}

}  // namespace

// Clusters of two CTAs for the gate/up projection when many small experts are
// in flight at once (an expert's tiles, column blocks x its average row blocks,
// fewer than the SMs): there each expert's activation rows are otherwise read
// from DRAM once per column block, because the CTAs sharing them drift apart.
// Measured on the prefill-shaped layer (E=128, 6 column blocks, ~4 row blocks
// per expert): 564 -> 526 us; on the skewed layer (112 column blocks per
// expert) clusters were 3% slower, and clusters of 3 or more slower still.
int gate_up_cluster_size(const moe_shape* s, int n_tiles, int num_sms) {
  const long long rows = static_cast<long long>(s->T) * s->k;
  const long long mt_per_expert = std::max<long long>(1, (rows + static_cast<long long>(s->E) * kTileM - 1) /
                                                             (static_cast<long long>(s->E) * kTileM));
  return (n_tiles % 2 == 0 && n_tiles * mt_per_expert < num_sms) ? 2 : 1;
}

// which = 0: gate/up + SwiGLU (xa -> h); which = 1: down (h -> y).
cudaError_t launch_gemm_bf16(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                             uint8_t* ws, int which, int num_sms, cudaStream_t st) {
  const int H = s->H, I = s->I, E = s->E;
  GemmParams gp{};
  gp.mt_base = reinterpret_cast<const int*>(ws + p.mt_base);
  gp.cnt = reinterpret_cast<const int*>(ws + p.cnt);
  gp.E = E;
  gp.dev_status = reinterpret_cast<int*>(ws + p.status);
  gp.timeout_ns = wait_limit_ns();
  gp.stall_loads = which == 0 && stall_gate_up_loads() ? 1 : 0;
  gp.cs = 1;
  gp.act = s->act;
  // every tile count is bounded by the row capacity
  const int max_mtiles = static_cast<int>(p.m_rows / kTileM);
  CUtensorMap tmA, tmB, tmO;
  if (which == 0) {
    if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.xa, H, p.m_rows, kBK, kTileM) ||
        !encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_gate_up, H,
                              static_cast<uint64_t>(E) * 2 * I, kBK, 128) ||
        !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, p.m_rows, 32, 32,
                              CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
    gp.num_kb = H / kBK;
    gp.n_tiles = I / 128;
    gp.b_rows_per_expert = 2 * I;
    gp.b_tile_stride = 128;
    gp.b_second_offset = I;
    gp.out = reinterpret_cast<__nv_bfloat16*>(ws + p.h);
    gp.out_ld = I;
    gp.out_tile_cols = 128;
    gp.cs = gate_up_cluster_size(s, gp.n_tiles, num_sms);
    const int groups = max_mtiles * ((gp.n_tiles + gp.cs - 1) / gp.cs);
    const int grid = gp.cs * std::max(1, std::min(num_sms / gp.cs, groups));
    return launch_one<256, true>(tmA, tmB, tmO, gp, grid, st);
  }
  if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, p.m_rows, kBK, kTileM) ||
      !encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_down, I, static_cast<uint64_t>(E) * H, kBK,
                            128) ||
      !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.y, H, p.m_rows, 32, 32,
                            CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  gp.num_kb = I / kBK;
  gp.b_rows_per_expert = H;
  gp.b_second_offset = 128;
  gp.out = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  gp.out_ld = H;
  // (H % 256 == 0 runs on the CTA-pair kernel, gemm_bf16_pair.cu)
  gp.n_tiles = H / 128;
  gp.b_tile_stride = 128;
  gp.out_tile_cols = 128;
  const int grid = std::max(1, std::min(num_sms, max_mtiles * gp.n_tiles));
  return launch_one<128, false>(tmA, tmB, tmO, gp, grid, st);
}

}  // namespace moe

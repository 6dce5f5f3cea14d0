// Down projection on CTA pairs: tcgen05.mma.cta_group::2 with 256-row tiles
// ("Experts backends", backend table: the expert ends with its down
// projection; grouped_mm / deepgemm run all experts in one grouped GEMM over
// expert-sorted tokens):
//
//   y[rows of e, n..n+255] = h_e Wd_e^T        on 256 rows x 256 y columns
//
// A cluster of two CTAs (one per SM of a pair) computes one 256 x 256 tile:
// each CTA stages its own 128 rows of A and one half of B (y columns
// n..n+127 in the leader, n+128..n+255 in the peer), so a CTA moves 32 KB per 64-wide
// K step instead of 48 KB and the 6-stage ring hides 5 K steps of latency.
// Both CTAs' TMA copies complete on the leader's barrier; only the leader
// issues the MMAs, and its commits arrive on the stage and accumulator
// barriers of both CTAs. Each CTA's TMEM holds its 128 rows of the
// accumulator (two 256-column buffers), which its own epilogue drains; the
// peer's epilogue releases a buffer by arriving on the leader's barrier.
// The epilogue converts 32 columns at a time to bf16, writes them into a
// 64-byte-swizzled staging tile in shared memory (two per warp, so one fills
// while the other is read) and stores it with a TMA tile store; the release of
// the accumulator therefore never waits for global stores to drain.
//
// Tiles pair up consecutive 128-row blocks of one expert (an expert with an
// odd count pairs its last block with rows the peer computes and discards).
// No TMA multicast is used. (The gate/up projection measured faster on the
// single-CTA kernel and stays there.)
#include "moe_common.cuh"
#include "moe_internal.h"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;
constexpr int kStages = 6;
constexpr int kThreads = 192;
constexpr int kA = kTileM * kBK * 2;  // this CTA's 128 rows of A: 16 KB
constexpr int kB = 128 * kBK * 2;     // this CTA's half of B: 16 KB
constexpr int kStage = kA + kB;
constexpr int kN = 256;  // MMA N: both halves of B
constexpr int kBarriers = 2 * kStages + 5;
constexpr int kEpiWarps = 4;
constexpr int kStageBox = 32 * 64;  // one staging tile: 32 rows x 32 bf16 columns (64-byte rows)
constexpr int kStaging = kEpiWarps * 2 * kStageBox;

size_t pair_smem_bytes(int E) {
  return 1024 + static_cast<size_t>(kStages) * kStage + kStaging + kBarriers * 8 + 16 +
         static_cast<size_t>(3 * E + 2) * 4;
}

struct PairParams {
  const int* mt_base;  // [E+1] 128-row block prefix
  const int* pt_base;  // [E+1] 256-row pair prefix
  const int* cnt;
  int E;
  int num_kb;
  int n_tiles;
  int b_rows_per_expert;
  int b_tile_stride;
  int b_second_offset;  // B rows from the leader's half to the peer's half
  __nv_bfloat16* out;
  int out_ld;
  int out_tile_cols;
  int* dev_status;
  unsigned long long timeout_ns;
};

struct PairCoord {
  int e, n, row0, valid;  // row0 / valid: this CTA's 128 rows
};

__device__ __forceinline__ PairCoord pair_coord(int tile, const int* s_pt, const int* s_mt, const int* s_cnt, int E,
                                                int NT, int rank) {
  PairCoord c;
  c.e = find_expert(s_pt, E, tile / NT);
  const int base = s_pt[c.e];
  const int np = s_pt[c.e + 1] - base;
  const int local = tile - base * NT;
  c.n = local / np;
  const int m = 2 * (local - c.n * np) + rank;
  c.row0 = (s_mt[c.e] + m) * kTileM;
  c.valid = max(0, min(kTileM, s_cnt[c.e] - m * kTileM));
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                  const __grid_constant__ CUtensorMap tmY, const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kA;
  uint8_t* sY = sB + kStages * kB;                                    // [4 warps][2][kStageBox]
  uint64_t* full = reinterpret_cast<uint64_t*>(sY + kStaging);  // used in the leader
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [2]
  uint64_t* tempty = tfull + 2;       // [2] used in the leader: 4 warps of each CTA arrive
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_mt = reinterpret_cast<int*>(s_tmem + 4);
  int* s_pt = s_mt + p.E + 1;
  int* s_cnt = s_pt + p.E + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  for (int i = threadIdx.x; i <= p.E; i += kThreads) {
    s_mt[i] = p.mt_base[i];
    s_pt[i] = p.pt_base[i];
  }
  for (int i = threadIdx.x; i < p.E; i += kThreads) s_cnt[i] = p.cnt[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, 2 * kN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int NT = p.n_tiles;
  const int total = s_pt[p.E] * NT;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        const PairCoord c = pair_coord(tile, s_pt, s_mt, s_cnt, p.E, NT, rank);
        const int brow = c.e * p.b_rows_per_expert + c.n * p.b_tile_stride + rank * p.b_second_offset;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kStage);
          const uint32_t bar = leader_addr(&full[stage]);
          tma_load_2d_pair(sA + stage * kA, &tmA, bar, kb * kBK, c.row0);
          tma_load_2d_pair(sB + stage * kB, &tmB, bar, kb * kBK, brow);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok && leader) {
        // let the copies already issued (of both CTAs) land before the pair can exit
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
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader only) ----------------
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kTileM, kN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        if (!mbar_wait_bounded(&tempty[acc], aph ^ 1, s_abort, p.dev_status, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * kN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], ph, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * kA);
          const uint32_t b0 = smem_u32(sB + stage * kB);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc,
                           (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      umma_commit_pair(drain);
      int never = 0;
      mbar_wait_bounded(drain, 0, &never, p.dev_status, p.timeout_ns);
    }
  } else {
    // ---------------- epilogue (both CTAs, own 128 rows) ----------------
    const int quad = warp & 3;
    uint8_t* stage0 = sY + (warp - 2) * 2 * kStageBox;
    int buf = 0;
    int acc = 0;
    uint32_t aph = 0;
    for (int tile = cluster; tile < total; tile += nclusters) {
      const PairCoord c = pair_coord(tile, s_pt, s_mt, s_cnt, p.E, NT, rank);
      const bool got = mbar_wait_bounded(&tfull[acc], aph, s_abort, p.dev_status, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * kN);
      // a block past the end of its expert (the peer's half of an odd last
      // pair) aliases the next expert's rows: never stored. Pad rows inside a
      // block hold garbage that no later stage reads, and are stored with it.
      const bool store = c.valid > 0;
#pragma unroll 1
      for (int cc = 0; cc < kN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tb + cc * 32, v);
        tmem_ld_wait();
        uint8_t* stg = stage0 + buf * kStageBox;
        if (lane == 0) bulk_wait_group_read<1>();  // the store that last read this buffer is done with it
        __syncwarp();
        const uint32_t sb = smem_u32(stg);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(sb + sw64_offset(lane, i), pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                       pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                       pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                       pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && store) {
          tma_store_2d(&tmY, stg, c.n * p.out_tile_cols + cc * 32, c.row0 + quad * 32);
          bulk_commit_group();
        }
        buf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_addr(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
    if (lane == 0) bulk_wait_group<0>();  // every store of this warp has landed
  }

  __syncthreads();
  cluster_sync();  // neither CTA frees TMEM while the pair still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kN);
  }
}

cudaError_t launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY, const PairParams& pp,
                        int nclusters, cudaStream_t st) {
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(grouped_gemm_bf16_pair_kernel), &done);
  if (err != cudaSuccess) return err;
  // every pair of the persistent grid must be resident at once: with an odd
  // SM count in a GPC, fewer than num_sms / 2 pairs fit
  const int maxc = max_active_clusters(reinterpret_cast<const void*>(grouped_gemm_bf16_pair_kernel), 2, kThreads,
                                       pair_smem_bytes(pp.E));
  if (maxc > 0) nclusters = std::min(nclusters, maxc);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * nclusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pair_smem_bytes(pp.E);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_bf16_pair_kernel, tmA, tmB, tmY, pp);
}

}  // namespace

// which = 1: down (h -> y, H % 256 == 0); no other projection runs here.
cudaError_t launch_gemm_bf16_pair(const moe_shape* s, const Plan& p, const void* /*w_gate_up*/, const void* w_down,
                                  uint8_t* ws, int which, int num_sms, cudaStream_t st) {
  const int H = s->H, I = s->I, E = s->E;
  PairParams pp{};
  pp.mt_base = reinterpret_cast<const int*>(ws + p.mt_base);
  pp.pt_base = reinterpret_cast<const int*>(ws + p.pt_base);
  pp.cnt = reinterpret_cast<const int*>(ws + p.cnt);
  pp.E = E;
  pp.dev_status = reinterpret_cast<int*>(ws + p.status);
  pp.timeout_ns = wait_limit_ns();
  // upper bound of the pair-tile count: every expert's pairs fit in (row blocks + E) / 2 + E
  const int max_pairs = static_cast<int>(p.m_rows / kTileM) / 2 + E;
  CUtensorMap tmA, tmB, tmY;
  if (which != 1) return cudaErrorNotSupported;
  if (H % 256 != 0) return cudaErrorNotSupported;
  if (pair_smem_bytes(E) > kSmemLimit) return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, p.m_rows, kBK, kTileM) ||
      !encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_down, I, static_cast<uint64_t>(E) * H, kBK,
                            128) ||
      !encode_tensor_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.y, H, p.m_rows, 32, 32,
                            CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  pp.num_kb = I / kBK;
  pp.n_tiles = H / 256;
  pp.b_rows_per_expert = H;
  pp.b_tile_stride = 256;
  pp.b_second_offset = 128;
  pp.out = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  pp.out_ld = H;
  pp.out_tile_cols = 256;
  const int nclusters = std::max(1, std::min(num_sms / 2, max_pairs * pp.n_tiles));
  return launch_pair(tmA, tmB, tmY, pp, nclusters, st);
}

}  // namespace moe

// FP4 (e2m1) expert GEMMs on the PREFILL path ("Experts backends", section
// "FP8 and FP4 quantized experts": FP4-packed expert weights with power-of-two
// UE8M0 scales, on Blackwell). Weights are e2m1 codes, two per byte, with one
// UE8M0 byte per row and 32 consecutive elements along K; activations are
// bf16. Every e2m1 value times a power of two is exact in bf16, so the weights
// are widened to bf16 in shared memory and the MMA is the bf16 one
// (tcgen05.mma kind::f16, fp32 accumulation in TMEM): the result is the bf16
// layer's on the dequantised weights, while HBM carries half a byte per
// weight.
//
//   gate/up:  h[rows of e, n..n+127] = act(X_e Wg_e^T) * (X_e Wu_e^T)
//   down:     y[rows of e, n..n+255] = h_e Wd_e^T
//
// Warp roles (448 threads, one CTA per SM):
//   warp 0       TMA producer: A tile [128 x 64] bf16 into the operand ring,
//                the B tile's packed codes [256 rows x 32 bytes] into the raw ring
//   warp 1       TMEM allocator and MMA issuer (one thread): 4 MMAs of K=16 per stage
//   warps 2..5   epilogue: TMEM -> act / bf16 -> 64-byte-swizzled staging tile
//                -> TMA tile store (one warp per TMEM lane quadrant)
//   warps 6..13  converters: each thread widens two 16-byte units (32 codes, one
//                scale block each) of the raw tile to bf16, scales them by
//                2^(b-127) and writes them, 128-byte-swizzled as a TMA load
//                would, into the operand ring's B slot. Both copies of a stage
//                complete on its raw barrier, so the stage is full once all
//                eight converter warps (which waited on that barrier) arrived.
// Tiles and their order are those of the bf16 kernel (tile_sched.cuh).
#include <cuda_fp4.h>

#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;  // K elements per stage: one 128-byte bf16 row
constexpr int kStages = 3;
constexpr int kEpiWarps = 4;
constexpr int kConvWarps = 8;
constexpr int kConvFirstWarp = 2 + kEpiWarps;
constexpr int kThreads = 32 * (2 + kEpiWarps + kConvWarps);
constexpr int kN = 256;                 // MMA N (B rows per tile)
constexpr int kA = kTileM * kBK * 2;    // 16 KB
constexpr int kB = kN * kBK * 2;        // 32 KB (bf16, after widening)
constexpr int kRaw = kN * kBK / 2;      // 8 KB of packed codes
constexpr int kStageBox = 32 * 64;      // staging tile: 32 rows x 64 bytes
constexpr int kStaging = kEpiWarps * 2 * kStageBox;
constexpr int kBarriers = 4 * kStages + 5;
constexpr size_t kFixedSmem = 1024 + static_cast<size_t>(kStages) * (kA + kB + kRaw) + kStaging + kBarriers * 8 + 16;

bool sched_in_smem(int E) { return kFixedSmem + static_cast<size_t>(2 * E + 1) * 4 <= kSmemLimit; }
size_t smem_bytes(int E) { return kFixedSmem + (sched_in_smem(E) ? static_cast<size_t>(2 * E + 1) * 4 : 0); }

struct Fp4Params {
  const int* mt_base;
  const int* cnt;
  int E;
  int num_kb;             // K / 64
  int n_tiles;            // N blocks per expert
  int b_rows_per_expert;  // rows of one expert's B matrix
  int b_tile_stride;      // B rows between consecutive N blocks
  int b_second_offset;    // B rows from the first 128-row half of a tile to the second
  const uint8_t* w_scale; // [E * b_rows_per_expert, K / 32] UE8M0
  int kscales;            // K / 32
  int out_tile_cols;      // output columns per tile (128 of h, 256 of y)
  int act;
  int sched_smem;
  int* dev_status;
  unsigned long long timeout_ns;
};

// 8 e2m1 codes (one 32-bit word, lowest nibble first) times `scale`, as 4
// packed bf16 pairs: exact (e2m1 -> f16 is exact, the power-of-two product
// is exact in fp32 and again in bf16).
__device__ __forceinline__ void widen8(uint32_t v, float scale, uint32_t (&out)[4]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const __half2 h2 =
        __half2(__nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>((v >> (8 * b)) & 0xFFu), __NV_E2M1));
    const float2 f = __half22float2(h2);
    out[b] = pack_bf16x2(f.x * scale, f.y * scale);
  }
}

__device__ __forceinline__ uint8_t* next_stage(uint8_t* stage0, int& buf, int lane) {
  if (lane == 0) bulk_wait_group_read<1>();
  __syncwarp();
  uint8_t* stg = stage0 + buf * kStageBox;
  buf ^= 1;
  return stg;
}

__device__ __forceinline__ void store_box(const CUtensorMap* map, uint8_t* stg, const uint32_t (&w)[16], int x, int y,
                                          int lane) {
  const uint32_t sb = smem_u32(stg);
#pragma unroll
  for (int i = 0; i < 4; ++i) st_shared_v4(sb + sw64_offset(lane, i), w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  fence_proxy_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, stg, x, y);
    bulk_commit_group();
  }
}

template <bool kGated, int kAct>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmR,
                            const __grid_constant__ CUtensorMap tmO, const Fp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kA;
  uint8_t* sR = sB + kStages * kB;
  uint8_t* sO = sR + kStages * kRaw;
  uint64_t* full = reinterpret_cast<uint64_t*>(sO + kStaging);
  uint64_t* empty = full + kStages;
  uint64_t* rfull = empty + kStages;
  uint64_t* rempty = rfull + kStages;
  uint64_t* tfull = rempty + kStages;  // [2]
  uint64_t* tempty = tfull + 2;        // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_sched = reinterpret_cast<int*>(s_tmem + 4);
  const int* s_mt = p.sched_smem ? s_sched : p.mt_base;
  const int* s_cnt = p.sched_smem ? s_sched + p.E + 1 : p.cnt;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.sched_smem) {
    for (int i = threadIdx.x; i <= p.E; i += kThreads) s_sched[i] = p.mt_base[i];
    for (int i = threadIdx.x; i < p.E; i += kThreads) s_sched[p.E + 1 + i] = p.cnt[i];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], kConvWarps);  // every converter warp, after the stage's copies landed
      mbar_init(&empty[s], 1);
      mbar_init(&rfull[s], 1);
      mbar_init(&rempty[s], kConvWarps);
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
    prefetch_tensormap(&tmR);
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
  const int total = s_mt[p.E] * NT;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_a = l2_policy_evict_last();  // A rows are re-read by every N block of the expert
      const uint64_t pol_b = l2_policy_evict_first();
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord c = tile_coord(tile, s_mt, s_cnt, p.E, NT);
        const int brow = c.e * p.b_rows_per_expert + c.n * p.b_tile_stride;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns) ||
              !mbar_wait_bounded(&rempty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&rfull[stage], kA + kRaw);
          tma_load_2d_hint(sA + stage * kA, &tmA, &rfull[stage], kb * kBK, c.row0, pol_a);
          tma_load_2d_hint(sR + stage * kRaw, &tmR, &rfull[stage], kb * (kBK / 2), brow, pol_b);
          tma_load_2d_hint(sR + stage * kRaw + 128 * (kBK / 2), &tmR, &rfull[stage], kb * (kBK / 2),
                           brow + p.b_second_offset, pol_b);
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
          mbar_wait_bounded(&rfull[stage], ph, &never, p.dev_status, 1000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_bf16_f32(kTileM, kN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
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
      umma_commit(drain);
      int never = 0;
      mbar_wait_bounded(drain, 0, &never, p.dev_status, p.timeout_ns);
    }
  } else if (warp < kConvFirstWarp) {
    // ---------------- epilogue: one warp per TMEM lane quadrant ----------------
    const int quad = warp & 3;
    uint8_t* stage0 = sO + (warp - 2) * 2 * kStageBox;
    int buf = 0, acc = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileCoord c = tile_coord(tile, s_mt, s_cnt, p.E, NT);
      const bool got = mbar_wait_bounded(&tfull[acc], aph, s_abort, p.dev_status, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * kN);
      const int y0 = c.row0 + quad * 32;  // pad rows of the expert's last block are stored too; nothing reads them
      if constexpr (kGated) {
        // gate columns 0..127, up columns 128..255: 128 h columns
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + cc * 32, g);
          tmem_ld32(tb + 128 + cc * 32, u);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(gated_act_t<kAct>(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                               gated_act_t<kAct>(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
          store_box(&tmO, next_stage(stage0, buf, lane), w, c.n * p.out_tile_cols + cc * 32, y0, lane);
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < kN / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tb + cc * 32, v);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          store_box(&tmO, next_stage(stage0, buf, lane), w, c.n * p.out_tile_cols + cc * 32, y0, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
    if (lane == 0) bulk_wait_group<0>();
  } else {
    // ---------------- converters: packed e2m1 -> scaled bf16, swizzled ----------------
    const int ct = threadIdx.x - 32 * kConvFirstWarp;  // 0 .. 255
    const int half = ct & 1;                            // which 32 of the stage's 64 K elements
    const int row0 = ct >> 1;                           // B rows row0 and row0 + 128
    int stage = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      const TileCoord c = tile_coord(tile, s_mt, s_cnt, p.E, NT);
      const size_t grow0 = static_cast<size_t>(c.e) * p.b_rows_per_expert + c.n * p.b_tile_stride + row0;
      const uint8_t* srow0 = p.w_scale + grow0 * p.kscales + half;
      const uint8_t* srow1 = p.w_scale + (grow0 + p.b_second_offset) * p.kscales + half;
      // the scale bytes of the next stage are in flight while this one converts
      uint32_t b0_next = __ldg(srow0), b1_next = __ldg(srow1);
      for (int kb = 0; kb < p.num_kb; ++kb) {
        const float sc0 = ue8m0_value(b0_next);
        const float sc1 = ue8m0_value(b1_next);
        if (kb + 1 < p.num_kb) {
          b0_next = __ldg(srow0 + 2 * (kb + 1));
          b1_next = __ldg(srow1 + 2 * (kb + 1));
        }
        const bool got = mbar_wait_bounded(&rfull[stage], ph, s_abort, p.dev_status, p.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint8_t* raw = sR + stage * kRaw;
        const uint4 v0 = *reinterpret_cast<const uint4*>(raw + row0 * (kBK / 2) + half * 16);
        const uint4 v1 = *reinterpret_cast<const uint4*>(raw + (row0 + 128) * (kBK / 2) + half * 16);
        __syncwarp();
        if (lane == 0) mbar_arrive(&rempty[stage]);
        const uint32_t bst = smem_u32(sB + stage * kB);
        const uint32_t wv0[4] = {v0.x, v0.y, v0.z, v0.w}, wv1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
          widen8(wv0[j], sc0, o);
          st_shared_v4(bst + sw128_offset(row0, half * 4 + j), o[0], o[1], o[2], o[3]);
          widen8(wv1[j], sc1, o);
          st_shared_v4(bst + sw128_offset(row0 + 128, half * 4 + j), o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_shared();  // the MMA reads this slot through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) {
          stage = 0;
          ph ^= 1;
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kN);
  }
}

template <bool kGated, int kAct>
cudaError_t launch_one(const CUtensorMap& tmA, const CUtensorMap& tmR, const CUtensorMap& tmO, Fp4Params fp,
                       int grid, cudaStream_t st) {
  fp.sched_smem = sched_in_smem(fp.E) ? 1 : 0;
  const size_t smem = smem_bytes(fp.E);
  if (smem > kSmemLimit) return cudaErrorInvalidValue;
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(grouped_gemm_fp4_kernel<kGated, kAct>), &done);
  if (err != cudaSuccess) return err;
  grouped_gemm_fp4_kernel<kGated, kAct><<<grid, kThreads, smem, st>>>(tmA, tmR, tmO, fp);
  return cudaGetLastError();
}

}  // namespace

bool fp4_gemm_available() { return true; }

// which = 0: gate/up (+ gated activation): xa -> h; which = 1: down: h -> y.
// The down tile spans 256 columns of y, so H must be a multiple of 256.
cudaError_t launch_gemm_fp4(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                            const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws, int which, int num_sms,
                            cudaStream_t st) {
  const int H = s->H, I = s->I, E = s->E;
  Fp4Params fp{};
  fp.mt_base = reinterpret_cast<const int*>(ws + p.mt_base);
  fp.cnt = reinterpret_cast<const int*>(ws + p.cnt);
  fp.E = E;
  fp.act = s->act;
  fp.dev_status = reinterpret_cast<int*>(ws + p.status);
  fp.timeout_ns = wait_limit_ns();
  const int max_mtiles = static_cast<int>(p.m_rows / kTileM);
  CUtensorMap tmA, tmR, tmO;
  if (which == 0) {
    if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.xa, H, p.m_rows, kBK, kTileM) ||
        !encode_tensor_map_2d(&tmR, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_gate_up, H / 2,
                              static_cast<uint64_t>(E) * 2 * I, kBK / 2, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, p.m_rows, 32, 32,
                              CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
    fp.num_kb = H / kBK;
    fp.n_tiles = I / 128;
    fp.b_rows_per_expert = 2 * I;
    fp.b_tile_stride = 128;
    fp.b_second_offset = I;
    fp.w_scale = sw_gate_up;
    fp.kscales = H / 32;
    fp.out_tile_cols = 128;
    const int grid = std::max(1, std::min(num_sms, max_mtiles * fp.n_tiles));
    switch (s->act) {
      case MOE_ACT_GELU: return launch_one<true, MOE_ACT_GELU>(tmA, tmR, tmO, fp, grid, st);
      case MOE_ACT_RELU: return launch_one<true, MOE_ACT_RELU>(tmA, tmR, tmO, fp, grid, st);
      default: return launch_one<true, MOE_ACT_SILU>(tmA, tmR, tmO, fp, grid, st);
    }
  }
  if (H % 256 != 0) return cudaErrorNotSupported;
  if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.h, I, p.m_rows, kBK, kTileM) ||
      !encode_tensor_map_2d(&tmR, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_down, I / 2, static_cast<uint64_t>(E) * H,
                            kBK / 2, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.y, H, p.m_rows, 32, 32,
                            CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  fp.num_kb = I / kBK;
  fp.n_tiles = H / 256;
  fp.b_rows_per_expert = H;
  fp.b_tile_stride = 256;
  fp.b_second_offset = 128;
  fp.w_scale = sw_down;
  fp.kscales = I / 32;
  fp.out_tile_cols = 256;
  const int grid = std::max(1, std::min(num_sms, max_mtiles * fp.n_tiles));
  return launch_one<false, MOE_ACT_SILU>(tmA, tmR, tmO, fp, grid, st);
}

}  // namespace moe

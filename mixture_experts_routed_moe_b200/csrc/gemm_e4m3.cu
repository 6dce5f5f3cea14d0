// FP8 (e4m3) expert GEMMs on tcgen05 (kind::f8f6f4), fed by TMA ("Experts
// backends", section "FP8 and FP4 quantized experts": FP8 experts with
// dynamic per-row activation scales; on Blackwell the expert weight scales are
// UE8M0 powers of two, one per 128x128 block).
//
//   gate/up:  h = act(Xg) * Xu with X = q_x * s_x (per row, per 128 columns) and
//             W = q_w * 2^(b-127) (per 128x128 block); h is quantised again per
//             row and 128 columns (e4m3 codes + fp32 scale)
//   down:     y = h W_d^T, rounded to bf16
//
// The activation scales are arbitrary fp32 numbers, so they cannot ride in the
// MMA's UE8M0 block scales. Instead every 128-wide K block goes through the
// tensor core on its own: 4 MMAs of K=32 write a fresh fp32 partial into one of
// two TMEM buffers, and 8 epilogue warps read it back and promote it into
// register accumulators with the combined scale s_x[row, kb] * 2^(b[nb, kb]-127).
// While they promote one partial, the tensor core fills the other.
//
// Warp roles (320 threads, one CTA per SM): warp 0 TMA producer, warp 1 TMEM
// allocator and MMA issuer, warps 2..9 promotion + epilogue. Warps w and w+4
// share TMEM lane quadrant w%4 (rows); warp group 2..5 takes the first half of
// each 128-column block pair, 6..9 the second. Tiles and their order are those
// of the bf16 kernel (tile_sched.cuh), handed out dynamically: the producer
// takes the next tile number from a counter as its CTA frees up, so CTAs
// running at the same time work on consecutive tiles (the row blocks of one
// expert and column block, which share the weight tile through L2) and the
// load evens out across SMs. A tile's results (h codes, or y) leave
// through 64-byte-swizzled staging tiles in shared memory and TMA tile stores,
// so the tile end issues a few shared-memory stores instead of scattered
// 16-byte global stores, one row per lane.
#include "moe_common.cuh"
#include "moe_internal.h"
#include "tile_sched.cuh"

namespace moe {
namespace {

constexpr int kBK = 128;  // e4m3 elements per 128-byte stage row = one scale block
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kA = kTileM * kBK;  // 16 KB
constexpr int kB = 256 * kBK;     // 32 KB
constexpr int kStage = kA + kB;
constexpr int kBarriers = 2 * kStages + 5 + 2 * kTileRing;
constexpr int kStageBox = 32 * 64;  // one staging tile: 32 rows of 64 bytes
constexpr int kStaging = kEpiWarps * 2 * kStageBox;

// The expert tile prefix and counts live in shared memory when they fit next
// to the ring and the staging tiles, else the kernel reads them from global
// memory (through L1).
constexpr size_t kFixedSmem =
    1024 + static_cast<size_t>(kStages) * kStage + kStaging + kBarriers * 8 + 16 + 2 * kTileM * 4 + kTileRing * 4;
bool sched_in_smem(int E) { return kFixedSmem + static_cast<size_t>(2 * E + 1) * 4 <= kSmemLimit; }
size_t smem_bytes(int E) { return kFixedSmem + (sched_in_smem(E) ? static_cast<size_t>(2 * E + 1) * 4 : 0); }

struct Fp8Params {
  const int* mt_base;
  const int* cnt;
  int E;
  int num_kb;             // K / 128
  int n_tiles;            // column blocks per expert
  int b_rows_per_expert;  // rows of one expert's B matrix
  int b_tile_stride;      // B rows between consecutive column blocks
  int b_second_offset;    // B rows from the first 128-row half to the second
  const float* a_scale;   // [m_rows, num_kb]
  const uint8_t* w_scale; // [E, b_rows_per_expert/128, num_kb]
  float* hs;              // gate/up: h scales [m_rows, I/128]
  int out_ld;             // I (gate/up) or H (down)
  int sched_smem;         // 1: expert prefix and counts copied to shared memory
  int* tile_counter;      // next tile to hand out (zero at launch)
  int act;                // gate activation (moe_activation)
  int* dev_status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory"); }

// Staging-buffer rotation of one epilogue warp (two buffers): wait until the
// TMA store that last read the next buffer is done with it.
__device__ __forceinline__ uint8_t* next_stage(uint8_t* stage0, int& buf, int lane) {
  if (lane == 0) bulk_wait_group_read<1>();
  __syncwarp();
  uint8_t* stg = stage0 + buf * kStageBox;
  buf ^= 1;
  return stg;
}

// Stores the warp's 32 rows x 64 bytes (4 x 16 bytes per lane, one row per
// lane) at (x, y) of `map` through staging buffer `stg`.
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

// End of a gate/up tile for one thread's row: h = act(gate) * up on its 64
// columns, the row's amax over the 128-column group (this warp's half and the
// partner warp's, exchanged through shared memory), then the 1x128 e4m3 codes
// (stored with the warp's other rows at (x0, y0) of the h-code map) and the
// group scale. The activation is fixed at compile time.
template <int kAct>
__device__ __forceinline__ void finish_gate_up(float (&acc)[128], float* s_amax, int hf, int r, bool valid,
                                               const CUtensorMap* map, uint8_t* stg, int x0, int y0, int lane,
                                               float* hs) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    acc[i] = gated_act_t<kAct>(acc[i], acc[64 + i]);
    amax = fmaxf(amax, fabsf(acc[i]));
  }
  s_amax[hf * kTileM + r] = amax;
  epi_bar_sync();
  amax = fmaxf(s_amax[r], s_amax[kTileM + r]);
  epi_bar_sync();
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const GroupDivisor dv = make_group_divisor(sc);
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(group_div(dv, acc[4 * i]), group_div(dv, acc[4 * i + 1])), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(group_div(dv, acc[4 * i + 2]), group_div(dv, acc[4 * i + 3])), __NV_SATFINITE, __NV_E4M3);
    w[i] = lo | (hi << 16);
  }
  // pad rows of the expert's last block are stored too (nothing reads them)
  store_box(map, stg, w, x0, y0, lane);
  if (valid && hf == 0) *hs = sc;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_e4m3_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmO, const Fp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kA;
  uint8_t* sO = sB + kStages * kB;  // [8 warps][2][kStageBox]
  uint64_t* full = reinterpret_cast<uint64_t*>(sO + kStaging);
  uint64_t* empty = full + kStages;
  uint64_t* pfull = empty + kStages;  // [2] partial accumulator ready
  uint64_t* pempty = pfull + 2;       // [2] partial accumulator consumed
  uint64_t* drain = pempty + 2;
  TileRing ring;
  ring.full = drain + 1;                // [kTileRing]
  ring.empty = ring.full + kTileRing;   // [kTileRing]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(ring.empty + kTileRing);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_amax = reinterpret_cast<float*>(s_tmem + 4);  // [2][128]
  ring.ids = reinterpret_cast<int*>(s_amax + 2 * kTileM);  // [kTileRing]
  int* s_sched = ring.ids + kTileRing;
  const int* s_mt = p.sched_smem ? s_sched : p.mt_base;
  const int* s_cnt = p.sched_smem ? s_sched + p.E + 1 : p.cnt;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.sched_smem) {
    for (int i = threadIdx.x; i <= p.E; i += kThreads) s_sched[i] = p.mt_base[i];
    for (int i = threadIdx.x; i < p.E; i += kThreads) s_sched[p.E + 1 + i] = p.cnt[i];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kEpiWarps);
    }
    for (int i = 0; i < kTileRing; ++i) {
      mbar_init(&ring.full[i], 1);
      mbar_init(&ring.empty[i], 1 + kEpiWarps);  // the MMA issuer and every epilogue warp read each tile
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
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int NT = p.n_tiles;
  const int KB = p.num_kb;
  const int total = s_mt[p.E] * NT;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      // weights stream through L2 once; the activation tile is re-read by
      // every column block of the expert: keep it, drop the weights first
      const uint64_t pol_a = l2_policy_evict_last();
      const uint64_t pol_b = l2_policy_evict_first();
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        const int tile = tiles_publish(ring, seq, p.tile_counter, total, s_abort, p.dev_status, p.timeout_ns);
        if (tile < 0) break;
        const TileCoord c = tile_coord(tile, s_mt, s_cnt, p.E, NT);
        const int brow = c.e * p.b_rows_per_expert + c.n * p.b_tile_stride;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], ph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStage);
          tma_load_2d_hint(sA + stage * kA, &tmA, &full[stage], kb * kBK, c.row0, pol_a);
          tma_load_2d_hint(sB + stage * kB, &tmB, &full[stage], kb * kBK, brow, pol_b);
          tma_load_2d_hint(sB + stage * kB + 128 * kBK, &tmB, &full[stage], kb * kBK, brow + p.b_second_offset, pol_b);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
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
      // ---------------- MMA issuer: one fresh partial per 128-wide K block ----------------
      constexpr uint32_t idesc = idesc_e4m3_f32(kTileM, 256);
      int stage = 0, pb = 0;
      uint32_t ph = 0, pph = 0;
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        if (tiles_take(ring, seq, s_abort, p.dev_status, p.timeout_ns) < 0) break;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], ph, s_abort, p.dev_status, p.timeout_ns) ||
              !mbar_wait_bounded(&pempty[pb], pph ^ 1, s_abort, p.dev_status, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(pb * 256);
          const uint32_t a0 = smem_u32(sA + stage * kA);
          const uint32_t b0 = smem_u32(sB + stage * kB);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            umma_e4m3(d, sdesc_kmajor_sw128(a0 + k * 32), sdesc_kmajor_sw128(b0 + k * 32), idesc, k != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          umma_commit(&pfull[pb]);
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1;
          }
          pb ^= 1;
          if (pb == 0) pph ^= 1;
        }
      }
      umma_commit(drain);
      int never = 0;
      mbar_wait_bounded(drain, 0, &never, p.dev_status, p.timeout_ns);
    }
  } else {
    // ---------------- promotion + epilogue ----------------
    const int quad = warp & 3;
    const int hf = (warp - 2) >> 2;  // 0: warps 2..5, 1: warps 6..9
    const int r = quad * 32 + lane;
    const int wrows = p.b_rows_per_expert / 128;  // weight scale rows per expert
    uint8_t* stage0 = sO + (warp - 2) * 2 * kStageBox;
    int buf = 0;
    int pb = 0;
    uint32_t pph = 0;
    bool ok = true;
    for (int seq = 0; ok; ++seq) {
      const int tile = tiles_take_warp(ring, seq, lane, s_abort, p.dev_status, p.timeout_ns);
      if (tile < 0) break;
      const TileCoord c = tile_coord(tile, s_mt, s_cnt, p.E, NT);
      const int row = c.row0 + r;
      // weight scale rows of the two 128-column halves this thread promotes
      int nb0, nb1;
      if (kGateUp) {
        nb0 = c.n;                                 // gate block
        nb1 = p.b_second_offset / 128 + c.n;       // up block
      } else {
        nb0 = nb1 = 2 * c.n + hf;
      }
      const uint8_t* ws0 = p.w_scale + (static_cast<size_t>(c.e) * wrows + nb0) * KB;
      const uint8_t* ws1 = p.w_scale + (static_cast<size_t>(c.e) * wrows + nb1) * KB;
      const float* xsr = p.a_scale + static_cast<size_t>(row) * KB;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      float sx_next = __ldg(xsr);
      for (int kb = 0; kb < KB; ++kb) {
        const float sx = sx_next;
        if (kb + 1 < KB) sx_next = __ldg(xsr + kb + 1);
        const float sc0 = sx * ue8m0_value(__ldg(ws0 + kb));
        const float sc1 = sx * ue8m0_value(__ldg(ws1 + kb));
        const bool got = mbar_wait_bounded(&pfull[pb], pph, s_abort, p.dev_status, p.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(pb * 256);
        // gate/up: columns [64hf, 64hf+64) of the gate half and the same of the up half;
        // down: columns [128hf, 128hf+128)
        // two 16-column loads in flight per wait
#pragma unroll
        for (int q = 0; q < 8; q += 2) {
          uint32_t v[2][16];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int qq = q + j;
            const uint32_t col =
                kGateUp ? ((qq < 4 ? 0u : 128u) + 64u * hf + 16u * (qq & 3)) : (128u * hf + 16u * qq);
            tmem_ld16(tb + col, v[j]);
          }
          tmem_ld_wait();
          if (q == 6) {
            // every column of this partial is in registers: hand the buffer
            // back to the tensor core before the last multiply-adds
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[pb]);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int qq = q + j;
            const float sc = (kGateUp && qq >= 4) ? sc1 : sc0;
#pragma unroll
            for (int i = 0; i < 16; i += 2)
              ffma2(acc[16 * qq + i], acc[16 * qq + i + 1], __uint_as_float(v[j][i]), __uint_as_float(v[j][i + 1]), sc);
          }
        }
        pb ^= 1;
        if (pb == 0) pph ^= 1;
      }
      if (!ok) break;
      // a warp that gave up on a wait raised the abort flag before leaving; never
      // enter the named barrier below without it
      if (__any_sync(0xffffffffu, *s_abort != 0)) break;
      const bool valid = r < c.valid;
      const int y0 = c.row0 + quad * 32;
      if constexpr (kGateUp) {
        // h for columns n*128 + 64hf + i, i < 64: acc[i] is the gate, acc[64+i] the up projection
        float* hs = p.hs + static_cast<size_t>(row) * (p.out_ld / 128) + c.n;
        uint8_t* stg = next_stage(stage0, buf, lane);
        const int x0 = c.n * 128 + hf * 64;
        switch (p.act) {
          case MOE_ACT_GELU: finish_gate_up<MOE_ACT_GELU>(acc, s_amax, hf, r, valid, &tmO, stg, x0, y0, lane, hs); break;
          case MOE_ACT_RELU: finish_gate_up<MOE_ACT_RELU>(acc, s_amax, hf, r, valid, &tmO, stg, x0, y0, lane, hs); break;
          default: finish_gate_up<MOE_ACT_SILU>(acc, s_amax, hf, r, valid, &tmO, stg, x0, y0, lane, hs); break;
        }
      } else {
        // y columns n*256 + 128hf + 32q .. +31, one staging tile each
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(acc[32 * q + 2 * i], acc[32 * q + 2 * i + 1]);
          uint8_t* stg = next_stage(stage0, buf, lane);
          store_box(&tmO, stg, w, c.n * 256 + hf * 128 + q * 32, y0, lane);
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // every store of this warp has landed
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <bool kGateUp>
cudaError_t launch_one(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmO, Fp8Params fp, int grid,
                       cudaStream_t st) {
  fp.sched_smem = sched_in_smem(fp.E) ? 1 : 0;
  const size_t smem = smem_bytes(fp.E);
  if (smem > kSmemLimit) return cudaErrorInvalidValue;
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(grouped_gemm_e4m3_kernel<kGateUp>), &done);
  if (err != cudaSuccess) return err;
  grouped_gemm_e4m3_kernel<kGateUp><<<grid, kThreads, smem, st>>>(tmA, tmB, tmO, fp);
  return cudaGetLastError();
}

}  // namespace

bool e4m3_path_available() { return true; }

// which = 0: gate/up (+SwiGLU, h quantised); which = 1: down. The activation
// quantisation of x happens in the permute stage.
cudaError_t launch_gemm_e4m3(const moe_shape* s, const Plan& p, const void* /*x*/, const void* w_gate_up,
                             const void* w_down, const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws,
                             int which, int num_sms, cudaStream_t st) {
  const int H = s->H, I = s->I, E = s->E;
  Fp8Params fp{};
  fp.mt_base = reinterpret_cast<const int*>(ws + p.mt_base);
  fp.cnt = reinterpret_cast<const int*>(ws + p.cnt);
  fp.E = E;
  fp.dev_status = reinterpret_cast<int*>(ws + p.status);
  fp.timeout_ns = wait_limit_ns();
  fp.act = s->act;
  // one tile counter per launch, zeroed with the status word by the permute stage
  fp.tile_counter = reinterpret_cast<int*>(ws + p.status) + kStatusTileCounter + which;
  const int max_mtiles = static_cast<int>(p.m_rows / kTileM);
  CUtensorMap tmA, tmB, tmO;
  if (which == 0) {
    if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + p.xa, H, p.m_rows, kBK, kTileM) ||
        !encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_gate_up, H, static_cast<uint64_t>(E) * 2 * I,
                              kBK, 128) ||
        !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + p.h, I, p.m_rows, 64, 32,
                              CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
    fp.num_kb = H / kBK;
    fp.n_tiles = I / 128;
    fp.b_rows_per_expert = 2 * I;
    fp.b_tile_stride = 128;
    fp.b_second_offset = I;
    fp.a_scale = reinterpret_cast<const float*>(ws + p.xs);
    fp.w_scale = sw_gate_up;
    fp.hs = reinterpret_cast<float*>(ws + p.hs);
    fp.out_ld = I;
    const int grid = std::max(1, std::min(num_sms, max_mtiles * fp.n_tiles));
    return launch_one<true>(tmA, tmB, tmO, fp, grid, st);
  }
  if (H % 256 != 0) return cudaErrorNotSupported;  // the down tile spans two 128-column scale blocks
  if (!encode_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + p.h, I, p.m_rows, kBK, kTileM) ||
      !encode_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_down, I, static_cast<uint64_t>(E) * H, kBK,
                            128) ||
      !encode_tensor_map_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.y, H, p.m_rows, 32, 32,
                            CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  fp.num_kb = I / kBK;
  fp.n_tiles = H / 256;
  fp.b_rows_per_expert = H;
  fp.b_tile_stride = 256;
  fp.b_second_offset = 128;
  fp.a_scale = reinterpret_cast<const float*>(ws + p.hs);
  fp.w_scale = sw_down;
  fp.out_ld = H;
  const int grid = std::max(1, std::min(num_sms, max_mtiles * fp.n_tiles));
  return launch_one<false>(tmA, tmB, tmO, fp, grid, st);
}

}  // namespace moe

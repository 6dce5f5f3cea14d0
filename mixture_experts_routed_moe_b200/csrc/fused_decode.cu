// The whole small-token forward in one launch: permute, gate/up with the gated
// activation, down projection and the weighted combine ("Experts backends",
// section "Fused Mega MoE on Blackwell": one fused kernel for the up
// projection, SwiGLU, the down projection and the combine; here on one GPU,
// without the expert-parallel dispatch, for bf16 experts on the weight-streaming
// path of the decode-stage switch).
//
// The stages that run as separate launches on the DECODE path become phases of
// one persistent kernel, linked by per-expert completion counters instead of
// kernel boundaries:
//
//   0  every block builds the expert-major permutation of the (at most
//      kFusedMaxAssignments) assignments in its own shared memory, with the same
//      deterministic ranks as the permute kernels; block 0 also writes it to
//      the workspace for inspection
//   1  gate/up tasks (touched expert, 4 rows of I): stream the weight rows and
//      write h; each finished task counts on done_gu[e]
//   2  down tasks (touched expert, 8 rows of H): wait until done_gu[e] holds
//      all I/4 gate/up tasks of expert e, then stream and write y; count on done_dn[e]
//   3  combine, one warp per token: wait until done_dn of the token's k
//      experts is full, then out[t] = bf16(sum_j w[t,j] * y[row(t,j)]) in fp32
//      fused multiply-adds, j ascending (the same bits as the combine kernel)
//
// Warps take tasks from one atomic queue per phase, so a warp only waits on
// tasks that running warps have already taken: no co-residency is assumed and
// the phases overlap (the down projection of the first experts streams while
// the last gate/up rows are still being read). Every wait is bounded; one that
// gives up records MOE_ERR_DEVICE_TIMEOUT in the status word and goes on.
// Rows written in this launch (h, y) are read back through L2 (ld.global.cg).
#include <algorithm>

#include "decode_core.cuh"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBlock = 256;
constexpr int kWarps = kBlock / 32;

struct FusedParams {
  const __nv_bfloat16* x;
  const int* idx;
  const float* topk_w;
  const __nv_bfloat16* wgu;
  const __nv_bfloat16* wd;
  __nv_bfloat16* out;
  int* status;
  int* hdr;
  int* cnt;
  int* row_off;
  int* row_src;
  int* slot_row;
  int* touched;
  int* sync;  // [3 queues][E done_gu][E done_dn], zero at launch
  __nv_bfloat16* h;
  __nv_bfloat16* y;
  int T, H, I, E, k, act;
  unsigned long long timeout_ns;
  int stall;  // failure-detection test: gate/up tasks publish no completions
};

size_t fused_smem_bytes(int E, int A) {
  // masks [kWarps][E], cnt [E], off [E+1], touched [E], row_src [A], slot [A], scan scratch, totals
  return static_cast<size_t>(kWarps) * E * 4 + static_cast<size_t>(3 * E + 1) * 4 + static_cast<size_t>(2 * A) * 4 +
         32 * 4 + 16;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Lane 0 polls *ctr until it reaches target (bounded); the warp then reads
// what the counted tasks wrote. Once any wait of the launch has given up, the
// others give up at once.
__device__ __forceinline__ void wait_count(const int* ctr, int target, int* status, unsigned long long limit,
                                           int lane) {
  if (lane == 0 && ld_acquire_gpu(ctr) < target) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(ctr) < target) {
      if ((*reinterpret_cast<volatile int*>(status) & kDevErrTimeout) != 0) break;
      if (globaltimer_ns() - t0 > limit) {
        atomicOr(status, kDevErrTimeout);
        break;
      }
      __nanosleep(64);
    }
  }
  __syncwarp();
  __threadfence();
}

// Next task of a phase's queue for the whole warp.
__device__ __forceinline__ int take(int* queue, int lane) {
  int t = 0;
  if (lane == 0) t = atomicAdd(queue, 1);
  return __shfl_sync(0xffffffffu, t, 0);
}

// Makes this warp's writes of one task visible device-wide, then counts it.
__device__ __forceinline__ void publish(int* ctr, int lane) {
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(ctr, 1);
}

// Inclusive scan of one value per thread over the block (kBlock threads).
__device__ __forceinline__ int block_scan(int v, int* s_warp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < kWarps) s_warp[lane] = w;
  }
  __syncthreads();
  const int r = v + (warp > 0 ? s_warp[warp - 1] : 0);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kBlock) fused_decode_kernel(const FusedParams p) {
  pdl_wait();  // the previous kernel on the stream has completed; its writes are visible
  pdl_trigger();
  extern __shared__ int smem_i[];
  const int E = p.E, T = p.T, k = p.k, H = p.H, I = p.I;
  const int A = T * k;
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_i);  // [kWarps][E]
  int* s_cnt = smem_i + kWarps * E;
  int* s_off = s_cnt + E;      // [E+1]
  int* s_touched = s_off + E + 1;
  int* s_row_src = s_touched + E;  // [A]
  int* s_slot = s_row_src + A;     // [A]
  int* s_warp = s_slot + A;        // [32]
  int* s_tot = s_warp + 32;        // [0] rows, [1] touched experts

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* queue = p.sync;
  int* done_gu = p.sync + 3;
  int* done_dn = done_gu + E;

  // ---------------- phase 0: the permutation, in every block ----------------
  for (int i = tid; i < kWarps * E; i += kBlock) s_mask[i] = 0;
  __syncthreads();
  bool bad = false;
  if (tid < T) {  // one token per thread (T <= kBlock)
    for (int j = 0; j < k; ++j) {
      const int e = p.idx[static_cast<size_t>(tid) * k + j];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        if (atomicOr(&s_mask[warp * E + e], 1u << lane) & (1u << lane)) bad = true;  // repeated expert
      } else {
        bad = true;
      }
    }
  }
  if (bad && blockIdx.x == 0) atomicOr(p.status, kDevErrIndex);
  __syncthreads();
  // per-expert counts and offsets: thread tid owns experts 4*tid .. 4*tid+3 (E <= 4*kBlock)
  int c4[4], tsum = 0, usum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = 4 * tid + q;
    c4[q] = 0;
    if (e < E)
      for (int w = 0; w < kWarps; ++w) c4[q] += __popc(s_mask[w * E + e]);
    tsum += c4[q];
    usum += c4[q] > 0 ? 1 : 0;
  }
  const int tincl = block_scan(tsum, s_warp);
  const int uincl = block_scan(usum, s_warp);
  {
    int base = tincl - tsum, ub = uincl - usum;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = 4 * tid + q;
      if (e < E) {
        s_cnt[e] = c4[q];
        s_off[e] = base;
        base += c4[q];
        if (c4[q] > 0) s_touched[ub++] = e;
      }
    }
    if (tid == kBlock - 1) {
      s_off[E] = tincl;
      s_tot[0] = tincl;
      s_tot[1] = uincl;
    }
  }
  __syncthreads();
  // rank of token t among the tokens of its expert: earlier warps' tokens, then earlier lanes
  if (tid < T) {
    for (int j = 0; j < k; ++j) {
      const int a = tid * k + j;
      const int e = p.idx[a];
      int row = -1;
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        int r = 0;
        for (int w = 0; w < warp; ++w) r += __popc(s_mask[w * E + e]);
        row = s_off[e] + r + __popc(s_mask[warp * E + e] & ((1u << lane) - 1u));
        s_row_src[row] = a;
      }
      s_slot[a] = row;
    }
  }
  __syncthreads();
  const int n_touched = s_tot[1];
  if (blockIdx.x == 0) {  // the layout the unfused path leaves in the workspace (tests read it)
    for (int e = tid; e < E; e += kBlock) {
      p.cnt[e] = s_cnt[e];
      p.row_off[e] = s_off[e];
    }
    for (int u = tid; u < n_touched; u += kBlock) p.touched[u] = s_touched[u];
    if (tid == 0) {
      p.row_off[E] = s_off[E];
      p.hdr[kHdrMTiles] = s_tot[0];
      p.hdr[kHdrTouched] = n_touched;
      p.hdr[kHdrRows] = s_tot[0];
      p.hdr[kHdrPairs] = 0;
    }
    for (int r = tid; r < s_tot[0]; r += kBlock) p.row_src[r] = s_row_src[r];
    for (int a = tid; a < A; a += kBlock) p.slot_row[a] = s_slot[a];
  }

  // ---------------- phase 1: gate/up ----------------
  const int rg = I / 4;
  const int total1 = n_touched * rg;
  for (int task = take(&queue[0], lane); task < total1; task = take(&queue[0], lane)) {
    const int u = task / rg;
    const int n0 = (task - u * rg) * 4;
    const int e = s_touched[u];
    const int c_e = s_cnt[e], r_e = s_off[e];
    const __nv_bfloat16* wg = p.wgu + (static_cast<size_t>(e) * 2 * I + n0) * H;
    const __nv_bfloat16* w[8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      w[r] = wg + static_cast<size_t>(r) * H;
      w[4 + r] = wg + (static_cast<size_t>(I) + r) * H;
    }
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = p.x + static_cast<size_t>(s_row_src[r_e + g0 + min(q, ntok - 1)] / k) * H;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: dec::gate_up_group<1>(w, a, H / 8, lane, p.h, row0, I, n0, p.act); break;
        case 2: dec::gate_up_group<2>(w, a, H / 8, lane, p.h, row0, I, n0, p.act); break;
        case 3: dec::gate_up_group<3>(w, a, H / 8, lane, p.h, row0, I, n0, p.act); break;
        default: dec::gate_up_group<4>(w, a, H / 8, lane, p.h, row0, I, n0, p.act); break;
      }
    }
    if (!p.stall) publish(&done_gu[e], lane);
  }

  // ---------------- phase 2: down ----------------
  const int cgroups = H / 8;
  const int total2 = n_touched * cgroups;
  for (int task = take(&queue[1], lane); task < total2; task = take(&queue[1], lane)) {
    const int u = task / cgroups;
    const int c0 = (task - u * cgroups) * 8;
    const int e = s_touched[u];
    const int c_e = s_cnt[e], r_e = s_off[e];
    const __nv_bfloat16* w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = p.wd + (static_cast<size_t>(e) * H + c0 + r) * I;
    wait_count(&done_gu[e], rg, p.status, p.timeout_ns, lane);
    for (int g0 = 0; g0 < c_e; g0 += 4) {
      const int ntok = min(4, c_e - g0);
      const __nv_bfloat16* a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = p.h + static_cast<size_t>(r_e + g0 + min(q, ntok - 1)) * I;
      const size_t row0 = static_cast<size_t>(r_e + g0);
      switch (ntok) {
        case 1: dec::down_group<1, true>(w, a, I / 8, lane, p.y, row0, H, c0); break;
        case 2: dec::down_group<2, true>(w, a, I / 8, lane, p.y, row0, H, c0); break;
        case 3: dec::down_group<3, true>(w, a, I / 8, lane, p.y, row0, H, c0); break;
        default: dec::down_group<4, true>(w, a, I / 8, lane, p.y, row0, H, c0); break;
      }
    }
    publish(&done_dn[e], lane);
  }

  // ---------------- phase 3: combine ----------------
  for (int t = take(&queue[2], lane); t < T; t = take(&queue[2], lane)) {
    for (int j = 0; j < k; ++j) {
      const int e = p.idx[static_cast<size_t>(t) * k + j];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) wait_count(&done_dn[e], cgroups, p.status, p.timeout_ns, lane);
    }
    uint4* o = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(t) * H);
    for (int c = lane; c < H / 8; c += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int j = 0; j < k; ++j) {
        const int row = s_slot[t * k + j];
        if (row < 0) continue;  // rejected index (reported in the status word)
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.y + static_cast<size_t>(row) * H) + c);
        const float wj = __ldg(p.topk_w + static_cast<size_t>(t) * k + j);
        acc[0] = fmaf(wj, bf16_lo(v.x), acc[0]);
        acc[1] = fmaf(wj, bf16_hi(v.x), acc[1]);
        acc[2] = fmaf(wj, bf16_lo(v.y), acc[2]);
        acc[3] = fmaf(wj, bf16_hi(v.y), acc[3]);
        acc[4] = fmaf(wj, bf16_lo(v.z), acc[4]);
        acc[5] = fmaf(wj, bf16_hi(v.z), acc[5]);
        acc[6] = fmaf(wj, bf16_lo(v.w), acc[6]);
        acc[7] = fmaf(wj, bf16_hi(v.w), acc[7]);
      }
      o[c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                        pack_bf16x2(acc[6], acc[7]));
    }
  }
}

}  // namespace

bool fused_supported(const moe_shape* s) {
  return s->wdtype == MOE_DT_BF16 && s->T <= kFusedMaxTokens &&
         static_cast<long long>(s->T) * s->k <= kFusedMaxAssignments && s->E <= 4 * kBlock &&
         fused_smem_bytes(s->E, s->T * s->k) <= kSmemLimit;
}

cudaError_t launch_fused_decode(const moe_shape* s, const Plan& p, const void* x, const int* topk_idx,
                                const float* topk_w, const void* w_gate_up, const void* w_down, void* out,
                                uint8_t* ws, int num_sms, cudaStream_t st) {
  FusedParams fp{};
  fp.x = static_cast<const __nv_bfloat16*>(x);
  fp.idx = topk_idx;
  fp.topk_w = topk_w;
  fp.wgu = static_cast<const __nv_bfloat16*>(w_gate_up);
  fp.wd = static_cast<const __nv_bfloat16*>(w_down);
  fp.out = static_cast<__nv_bfloat16*>(out);
  fp.status = reinterpret_cast<int*>(ws + p.status);
  fp.hdr = reinterpret_cast<int*>(ws + p.hdr);
  fp.cnt = reinterpret_cast<int*>(ws + p.cnt);
  fp.row_off = reinterpret_cast<int*>(ws + p.mt_base);
  fp.row_src = reinterpret_cast<int*>(ws + p.row_src);
  fp.slot_row = reinterpret_cast<int*>(ws + p.slot_row);
  fp.touched = reinterpret_cast<int*>(ws + p.touched);
  fp.sync = reinterpret_cast<int*>(ws + p.sync);
  fp.h = reinterpret_cast<__nv_bfloat16*>(ws + p.h);
  fp.y = reinterpret_cast<__nv_bfloat16*>(ws + p.y);
  fp.T = s->T;
  fp.H = s->H;
  fp.I = s->I;
  fp.E = s->E;
  fp.k = s->k;
  fp.act = s->act;
  fp.timeout_ns = wait_limit_ns();
  fp.stall = stall_gate_up_loads() ? 1 : 0;
  const size_t smem = fused_smem_bytes(s->E, s->T * s->k);
  static unsigned long long done = 0;
  cudaError_t err = ensure_max_smem(reinterpret_cast<const void*>(fused_decode_kernel), &done);
  if (err != cudaSuccess) return err;
  // one wave of resident blocks (more would only wait for tasks to run out)
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_decode_kernel, kBlock, smem);
  if (err != cudaSuccess) return err;
  err = cudaMemsetAsync(fp.status, 0, sizeof(int), st);
  if (err != cudaSuccess) return err;
  err = cudaMemsetAsync(fp.sync, 0, static_cast<size_t>(3 + 2 * s->E) * sizeof(int), st);
  if (err != cudaSuccess) return err;
  return launch_pdl(fused_decode_kernel, dim3(num_sms * std::max(1, per_sm)), dim3(kBlock), smem, st, fp);
}

}  // namespace moe

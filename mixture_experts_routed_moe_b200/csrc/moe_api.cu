// C ABI of the library (declared in include/moe_b200.h): host-side argument
// validation, the workspace plan, tensor-map encoding and the launch sequence
//   permute -> gate/up (+SwiGLU) -> down -> combine
// for the PREFILL (tcgen05 grouped GEMM) and DECODE (weight streaming) paths.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <limits>
#include <mutex>
#include <vector>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr size_t kAlign = 1024;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

constexpr int kMaxDevices = 64;

std::atomic<unsigned long long> g_wait_limit_ns{kDefaultTimeoutNs};
std::atomic<int> g_stall_gate_up{0};
std::atomic<int> g_sm_count[kMaxDevices];

}  // namespace

bool encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes, const void* base,
                          uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDevices) {
    const int cached = g_sm_count[dev].load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t ensure_max_smem(const void* kernel, unsigned long long* done) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const unsigned long long bit = (dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (__atomic_load_n(done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  int optin = 0;
  err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (err == cudaSuccess && bit != 0) __atomic_fetch_or(done, bit, __ATOMIC_ACQ_REL);
  return err;
}

bool validate_shape(const moe_shape* s) {
  if (s == nullptr) return false;
  if (s->T < 0 || s->H < 128 || s->I < 128 || s->H % 128 != 0 || s->I % 128 != 0) return false;
  if (s->H > 65536 || s->I > 65536) return false;
  if (s->E < 1 || s->E > 1024 || s->k < 1 || s->k > s->E) return false;
  if (s->wdtype != MOE_DT_BF16 && s->wdtype != MOE_DT_E4M3 && s->wdtype != MOE_DT_E2M1) return false;
  if (s->path != MOE_PATH_AUTO && s->path != MOE_PATH_PREFILL && s->path != MOE_PATH_DECODE &&
      s->path != MOE_PATH_FUSED)
    return false;
  if (s->act != MOE_ACT_SILU && s->act != MOE_ACT_GELU && s->act != MOE_ACT_RELU) return false;
  const long long A = static_cast<long long>(s->T) * s->k;
  const long long rows = A + static_cast<long long>(std::min<long long>(s->E, A)) * (kTileM - 1) + kTileM;
  if (rows >= (1ll << 31) || static_cast<long long>(s->E) * 2 * s->I >= (1ll << 31) ||
      static_cast<long long>(s->E) * s->H >= (1ll << 31))
    return false;
  return true;
}

// Decode-stage switch: the DECODE path while the assignments per expert stay
// at or below the crossover with the grouped GEMMs measured on B200 (sweeps
// of T on the decode- and large-layer shapes): 32 per expert for bf16
// experts (tensor-core GEMMs with the tokens as N, which stream the weights
// at HBM rate up to 128 tokens per expert), two for FP4 experts and one half
// for e4m3 experts, whose DECODE kernels widen codes on the CUDA cores.
int resolve_path(const moe_shape* s) {
  if (s->path != MOE_PATH_AUTO) return s->path;
  const long long A = static_cast<long long>(s->T) * s->k;
  const bool small = s->wdtype == MOE_DT_E4M3   ? 2 * A <= s->E
                     : s->wdtype == MOE_DT_E2M1 ? A <= 2ll * s->E
                                                : A <= 32ll * s->E;
  if (small) return MOE_PATH_DECODE;
  return MOE_PATH_PREFILL;
}

bool make_plan(const moe_shape* s, Plan* p) {
  if (!validate_shape(s)) return false;
  const long long T = s->T, H = s->H, I = s->I, E = s->E, k = s->k;
  const long long A = T * k;
  const bool fp8 = s->wdtype == MOE_DT_E4M3;
  p->path = resolve_path(s);
  const bool streaming = p->path == MOE_PATH_DECODE || p->path == MOE_PATH_FUSED;  // tile size 1, x read in place
  p->bm = streaming ? 1 : kTileM;
  if (p->bm == 1) {
    p->m_rows = A;
  } else {
    const long long rows = A + std::min(E, A) * (kTileM - 1);
    p->m_rows = std::max<long long>(kTileM, (rows + kTileM - 1) / kTileM * kTileM);
  }
  p->nblk = static_cast<int>(std::max<long long>(1, (T + kPermuteTokens - 1) / kPermuteTokens));
  const size_t none = std::numeric_limits<size_t>::max();
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + std::max<size_t>(bytes, 1), kAlign);
    return at;
  };
  const size_t M = static_cast<size_t>(p->m_rows);
  p->status = take(256);
  p->hdr = take(256);
  p->block_counts = take(static_cast<size_t>(p->nblk) * E * 4);
  p->cnt = take(E * 4);
  p->mt_base = take((E + 1) * 4);
  p->pt_base = take((E + 1) * 4);
  p->touched = take(E * 4);
  p->local_rank = take(std::max<long long>(A, 1) * 4);
  p->row_src = take(std::max<size_t>(M, 1) * 4);
  p->slot_row = take(std::max<long long>(A, 1) * 4);
  p->sync = take((3 + E * 2) * 4);
  const size_t act = fp8 ? 1 : 2;
  // permuted x: bf16 copy (bf16 PREFILL) or e4m3 codes (both e4m3 paths);
  // bf16 DECODE reads the token rows of x in place
  // (e4m3 DECODE: one row per token, not per assignment)
  const size_t xrows = (fp8 && streaming) ? static_cast<size_t>(T) : M;
  p->tc_stream = p->path == MOE_PATH_DECODE && small_gemm_supported(s);
  p->xa = (p->path == MOE_PATH_PREFILL || fp8 || p->tc_stream) ? take(xrows * H * act) : none;
  p->xs = fp8 ? take(xrows * (H / 128) * 4) : none;
  p->h = take(M * I * act);
  p->hs = fp8 ? take(M * (I / 128) * 4) : none;
  p->hf = (fp8 && streaming) ? take(M * I * 4) : none;
  p->y = take(M * H * 2);
  p->total = off;
  return true;
}

int max_active_clusters(const void* kernel, int cluster, int threads, size_t smem) {
  struct Entry {
    const void* kernel;
    int cluster, threads, dev;
    size_t smem;
    int n;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : cache)
    if (e.kernel == kernel && e.cluster == cluster && e.threads == threads && e.dev == dev && e.smem == smem)
      return e.n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();  // clear the query's error; callers fall back to their own bound
    n = 0;
  }
  cache.push_back(Entry{kernel, cluster, threads, dev, smem, n});
  return n;
}

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
bool stall_gate_up_loads() { return g_stall_gate_up.load(std::memory_order_relaxed) != 0; }

}  // namespace moe

using namespace moe;

namespace {

// bf16 experts whose H and I are multiples of 64 but not both of 128: a valid
// layer (the boundary accepts 64-aligned bf16 sizes) that this build's
// 128-wide tiles do not cover.
bool bf16_64_not_128(const moe_shape* s) {
  if (s == nullptr || s->wdtype != MOE_DT_BF16 || s->H < 64 || s->I < 64) return false;
  return s->H % 64 == 0 && s->I % 64 == 0 && (s->H % 128 != 0 || s->I % 128 != 0);
}

moe_status forward_impl(const moe_shape* shape, const void* x, const int32_t* topk_idx, const float* topk_w,
                        const void* w_gate_up, const void* w_down, const uint8_t* sw_gate_up,
                        const uint8_t* sw_down, void* out, void* workspace, size_t workspace_bytes, void* stream,
                        void* const* events, int32_t n_events) {
  if (bf16_64_not_128(shape)) return MOE_ERR_UNSUPPORTED;
  if (!validate_shape(shape)) return MOE_ERR_INVALID_ARG;
  if (!(n_events == 0 || (n_events == 5 && events != nullptr))) return MOE_ERR_INVALID_ARG;
  const bool fp8 = shape->wdtype == MOE_DT_E4M3;
  const bool fp4 = shape->wdtype == MOE_DT_E2M1;
  if ((fp8 || fp4) && (sw_gate_up == nullptr || sw_down == nullptr)) return MOE_ERR_SCALE_FORMAT;
  Plan plan;
  if (!make_plan(shape, &plan)) return MOE_ERR_INVALID_ARG;
  // e2m1 PREFILL: the down tile spans 256 columns of y
  if (fp4 && plan.path == MOE_PATH_PREFILL && (!fp4_gemm_available() || shape->H % 256 != 0))
    return MOE_ERR_UNSUPPORTED;
  // e4m3 PREFILL: the down tile spans two 128-column scale blocks
  if (fp8 && plan.path == MOE_PATH_PREFILL && (!e4m3_path_available() || shape->H % 256 != 0))
    return MOE_ERR_UNSUPPORTED;
  if (plan.path == MOE_PATH_FUSED && !fused_supported(shape)) return MOE_ERR_UNSUPPORTED;
  if (shape->T == 0) return MOE_OK;
  if (x == nullptr || topk_idx == nullptr || topk_w == nullptr || w_gate_up == nullptr || w_down == nullptr ||
      out == nullptr || workspace == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(w_gate_up, 16) || !aligned(w_down, 16) ||
      !aligned(workspace, 256) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < plan.total) return MOE_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int sms = device_sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  auto mark = [&](int i) -> bool {
    return n_events == 0 || cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
  };

  if (!mark(0)) return MOE_ERR_CUDA;
  if (plan.path == MOE_PATH_FUSED) {
    // one launch: its time shows as the gate/up stage (events 1..2)
    if (!mark(1)) return MOE_ERR_CUDA;
    if (launch_fused_decode(shape, plan, x, topk_idx, topk_w, w_gate_up, w_down, out, ws, sms, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return mark(2) && mark(3) && mark(4) ? MOE_OK : MOE_ERR_CUDA;
  }
  if (launch_permute(shape, plan, topk_idx, x, ws, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(1)) return MOE_ERR_CUDA;
  cudaError_t err;
  if (plan.path == MOE_PATH_DECODE && fp4) {
    err = launch_decode_fp4(shape, plan, x, w_gate_up, w_down, sw_gate_up, sw_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = launch_decode_fp4(shape, plan, x, w_gate_up, w_down, sw_gate_up, sw_down, ws, 1, sms, st);
  } else if (plan.path == MOE_PATH_DECODE && fp8) {
    err = launch_decode_e4m3(shape, plan, w_gate_up, w_down, sw_gate_up, sw_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = launch_decode_e4m3(shape, plan, w_gate_up, w_down, sw_gate_up, sw_down, ws, 1, sms, st);
  } else if (plan.path == MOE_PATH_DECODE) {
    err = launch_small_gemm(shape, plan, w_gate_up, w_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = launch_small_gemm(shape, plan, w_gate_up, w_down, ws, 1, sms, st);
  } else if (fp4) {
    err = launch_gemm_fp4(shape, plan, w_gate_up, w_down, sw_gate_up, sw_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = launch_gemm_fp4(shape, plan, w_gate_up, w_down, sw_gate_up, sw_down, ws, 1, sms, st);
  } else if (!fp8) {
    // gate/up: single-CTA 128x256 tiles; down: CTA-pair 256x256 tiles when
    // H allows (each measured the faster of the two on the prefill-shaped and
    // skewed layers)
    err = launch_gemm_bf16(shape, plan, w_gate_up, w_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = shape->H % 256 == 0 ? launch_gemm_bf16_pair(shape, plan, w_gate_up, w_down, ws, 1, sms, st)
                              : launch_gemm_bf16(shape, plan, w_gate_up, w_down, ws, 1, sms, st);
  } else {
    err = launch_gemm_e4m3(shape, plan, x, w_gate_up, w_down, sw_gate_up, sw_down, ws, 0, sms, st);
    if (err != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;
    err = launch_gemm_e4m3(shape, plan, x, w_gate_up, w_down, sw_gate_up, sw_down, ws, 1, sms, st);
  }
  if (err != cudaSuccess || !mark(3)) return MOE_ERR_CUDA;
  if (launch_combine(shape, plan, topk_w, out, ws, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(4)) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* topk_idx, float* topk_w,
                     void* stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k >= (1ll << 31) || static_cast<long long>(T) * E >= (1ll << 40))
    return MOE_ERR_INVALID_ARG;
  return launch_route(logits, T, E, k, topk_idx, topk_w, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

size_t moe_workspace_size(const moe_shape* shape) {
  Plan p;
  if (!make_plan(shape, &p)) return 0;
  return p.total;
}

moe_status moe_forward(const moe_shape* shape, const void* x, const int32_t* topk_idx, const float* topk_w,
                       const void* w_gate_up, const void* w_down, const uint8_t* sw_gate_up, const uint8_t* sw_down,
                       void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(shape, x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out, workspace,
                      workspace_bytes, stream, nullptr, 0);
}

moe_status moe_forward_timed(const moe_shape* shape, const void* x, const int32_t* topk_idx, const float* topk_w,
                             const void* w_gate_up, const void* w_down, const uint8_t* sw_gate_up,
                             const uint8_t* sw_down, void* out, void* workspace, size_t workspace_bytes,
                             void* stream, void* const* events, int32_t n_events) {
  return forward_impl(shape, x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out, workspace,
                      workspace_bytes, stream, events, n_events);
}

moe_status moe_workspace_query(const moe_shape* shape, moe_workspace_layout* layout) {
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  Plan p;
  if (!make_plan(shape, &p)) return MOE_ERR_INVALID_ARG;
  layout->status = p.status;
  layout->hdr = p.hdr;
  layout->cnt = p.cnt;
  layout->mt_base = p.mt_base;
  layout->row_src = p.row_src;
  layout->slot_row = p.slot_row;
  layout->xa = p.xa;
  layout->xs = p.xs;
  layout->h = p.h;
  layout->hs = p.hs;
  layout->y = p.y;
  layout->total = p.total;
  layout->bm = p.bm;
  layout->path = p.path;
  layout->m_rows = static_cast<int32_t>(p.m_rows);
  layout->reserved = 0;
  return MOE_OK;
}

moe_status moe_router(const void* x, const void* w_router, int32_t T, int32_t H, int32_t E, int32_t k,
                      float* logits, int32_t* topk_idx, float* topk_w, void* stream) {
  if (T < 0 || H < 64 || H % 64 != 0 || H > 65536 || E < 1 || E > 256 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x == nullptr || w_router == nullptr || topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      !aligned(logits, 4))
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k >= (1ll << 31) || static_cast<long long>(T) * E >= (1ll << 40))
    return MOE_ERR_INVALID_ARG;
  return launch_router(x, w_router, T, H, E, k, logits, topk_idx, topk_w, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_set_test_hooks(int32_t stall_gate_up_loads, uint64_t wait_limit_ns) {
  if (stall_gate_up_loads != 0 && stall_gate_up_loads != 1) return MOE_ERR_INVALID_ARG;
  if (wait_limit_ns != 0 && (wait_limit_ns < 1000000ull || wait_limit_ns > 60000000000ull)) return MOE_ERR_INVALID_ARG;
  g_wait_limit_ns.store(wait_limit_ns == 0 ? kDefaultTimeoutNs : wait_limit_ns);
  g_stall_gate_up.store(stall_gate_up_loads);
  return MOE_OK;
}

moe_status moe_read_device_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (v & kDevErrTimeout) return MOE_ERR_DEVICE_TIMEOUT;
  if (v & kDevErrIndex) return MOE_ERR_DEVICE_INDEX;
  return MOE_OK;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK:
      return "ok";
    case MOE_ERR_INVALID_ARG:
      return "invalid argument (shape, null or misaligned pointer)";
    case MOE_ERR_UNSUPPORTED:
      return "unsupported combination of options";
    case MOE_ERR_SCALE_FORMAT:
      return "FP8 experts need UE8M0 (power-of-two) block scales";
    case MOE_ERR_WORKSPACE:
      return "workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA:
      return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT:
      return "a kernel gave up on a bounded wait";
    case MOE_ERR_DEVICE_INDEX:
      return "routing index out of range or repeated within a token";
    case MOE_ERR_SCRATCH_LIMIT:
      return "shape needs more scratch than the allocation-free entry point holds";
  }
  return "unknown status";
}

int32_t moe_version(void) { return 100; }

}  // extern "C"

// Host-side declarations shared by the library's translation units: the
// workspace plan and the kernel launchers. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kTileM = 128;        // rows per expert tile on the PREFILL path
constexpr int kPermuteTokens = 256;  // tokens per block in the permute kernels
constexpr int kSmallPermuteT = 256;  // T up to this uses the single-block permute
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // bounded waits give up after 2 s
constexpr size_t kSmemLimit = 232448;  // dynamic shared memory a B200 CTA may opt in to (227 KB)
constexpr int kFusedMaxTokens = 256;         // FUSED path: one token per thread of a block
constexpr int kFusedMaxAssignments = 2048;   // FUSED path: T*k held in every block's shared memory

// Limit of every bounded device wait (kDefaultTimeoutNs unless a test set
// another through moe_set_test_hooks), and that entry point's switch that makes
// the gate/up GEMM's producer issue no loads.
unsigned long long wait_limit_ns();
bool stall_gate_up_loads();

// Where every intermediate lives inside the caller's workspace.
struct Plan {
  int path;        // resolved moe_path (PREFILL or DECODE)
  int bm;          // rows per expert tile: kTileM (PREFILL) or 1 (DECODE)
  int64_t m_rows;  // row capacity of the permuted buffers
  int nblk;        // permute blocks of kPermuteTokens tokens
  size_t status, hdr, block_counts, cnt, mt_base, pt_base, touched, local_rank, row_src, slot_row;
  size_t sync;  // FUSED path: task queues and per-expert completion counters (3 + 2E ints)
  size_t xa, xs, h, hs, hf, y, total;  // hf: fp32 h of the e4m3 DECODE path
  bool tc_stream;  // bf16 DECODE: tensor-core GEMMs with the tokens as N, x rows staged into xa
};

// Words of the status block (workspace offset `status`), all zeroed by the
// permute stage before the expert GEMMs run: the device status word, then one
// dynamic tile counter per GEMM launch (gate/up, down).
constexpr int kStatusTileCounter = 1;
constexpr int kStatusWordsZeroed = 4;

// Header words written on the device by the permute stage.
enum HdrWord { kHdrMTiles = 0, kHdrTouched = 1, kHdrRows = 2, kHdrPairs = 3 };

bool validate_shape(const moe_shape* s);
int resolve_path(const moe_shape* s);
bool make_plan(const moe_shape* s, Plan* p);

// Launchers. Each returns the launch's cudaError_t.
cudaError_t launch_route(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st);

// Router GEMM + routing (E <= 256, H % 64 == 0); logits may be null.
cudaError_t launch_router(const void* x, const void* w_router, int T, int H, int E, int k, float* logits, int* idx,
                          float* w, cudaStream_t st);

cudaError_t launch_permute(const moe_shape* s, const Plan& p, const int* topk_idx, const void* x, uint8_t* ws,
                           cudaStream_t st);

cudaError_t launch_gemm_bf16(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                             uint8_t* ws, int which, int num_sms, cudaStream_t st);

// 2-CTA (cta_group::2) down projection (which = 1), for H % 256 == 0.
cudaError_t launch_gemm_bf16_pair(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                                  uint8_t* ws, int which, int num_sms, cudaStream_t st);

// which = 0 also quantises the permuted activations (x -> e4m3 codes + fp32 scales).
cudaError_t launch_gemm_e4m3(const moe_shape* s, const Plan& p, const void* x, const void* w_gate_up,
                             const void* w_down, const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws,
                             int which, int num_sms, cudaStream_t st);
bool e4m3_path_available();

// bf16 experts on the DECODE path with the expert's token rows as the MMA's N
// (which = 0 gate/up from the staged x rows, 1 down).
bool small_gemm_supported(const moe_shape* s);
cudaError_t launch_small_gemm(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                              uint8_t* ws, int which, int num_sms, cudaStream_t st);
// e4m3 experts on the DECODE path: which = 0 runs gate/up and the h
// quantisation, which = 1 the down projection.
cudaError_t launch_decode_e4m3(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                               const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws, int which,
                               int num_sms, cudaStream_t st);

cudaError_t launch_combine(const moe_shape* s, const Plan& p, const float* topk_w, void* out, uint8_t* ws,
                           cudaStream_t st);

// FP4 (e2m1) experts on the DECODE path: which = 0 gate/up, 1 down.
cudaError_t launch_decode_fp4(const moe_shape* s, const Plan& p, const void* x, const void* w_gate_up,
                              const void* w_down, const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws,
                              int which, int num_sms, cudaStream_t st);
// FP4 experts on the PREFILL path (weights widened to bf16 in shared memory).
bool fp4_gemm_available();
cudaError_t launch_gemm_fp4(const moe_shape* s, const Plan& p, const void* w_gate_up, const void* w_down,
                            const uint8_t* sw_gate_up, const uint8_t* sw_down, uint8_t* ws, int which, int num_sms,
                            cudaStream_t st);

// The FUSED path (bf16 experts): permute, gate/up, down and combine in one launch.
bool fused_supported(const moe_shape* s);
cudaError_t launch_fused_decode(const moe_shape* s, const Plan& p, const void* x, const int* topk_idx,
                                const float* topk_w, const void* w_gate_up, const void* w_down, void* out,
                                uint8_t* ws, int num_sms, cudaStream_t st);

// Tensor-map encoding through the driver entry point (no link-time libcuda dependency).
// 128-byte swizzle by default (every operand tile and bf16 output tile); the
// 64-byte swizzle for tiles of 64-byte rows.
bool encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes, const void* base,
                          uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

int device_sm_count();

// Sets a kernel's dynamic shared-memory limit to the device maximum once per
// device (a host call kept out of the per-launch path, so launches can be
// captured in CUDA graphs). `done` is one bitmask per kernel, bit = device.
cudaError_t ensure_max_smem(const void* kernel, unsigned long long* done);

// Clusters of `cluster` CTAs (each `threads` threads and `smem` bytes of
// dynamic shared memory) of `kernel` that the current device holds at once;
// cached per kernel, shape and device; 0 if the query fails. A persistent
// cluster grid larger than this leaves clusters waiting for a second wave.
int max_active_clusters(const void* kernel, int cluster, int threads, size_t smem);

// Launches `kernel` with programmatic stream serialization: it may become
// resident while the previous kernel on the stream finishes, and waits for it
// with pdl_wait() before touching memory (every kernel launched this way
// does so first). Saves the launch gap between short kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace moe

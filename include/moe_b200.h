/*
 * moe_b200.h -- C ABI of the routed mixture-of-experts expert forward for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (Hugging Face Transformers docs page "Experts backends",
 * introduction): a router chooses k experts per token, each chosen expert maps
 * the token's hidden state through its own weights, and the token's output is
 * the routing-weighted sum of those expert results. Each expert is a gated MLP
 * (backend table, row "deepgemm_megamoe"): up projection, SwiGLU, down
 * projection, with SwiGLU meaning silu(gate) * up (section "SonicMoE").
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates, frees or copies between host and device, and never
 *    synchronises the host, except where an entry point says so.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and runs asynchronously, in stream order.
 *  - Arguments are validated on the host before anything is enqueued; a
 *    rejected call returns a negative moe_status and enqueues nothing.
 *  - Errors found on the device (routing indices out of range, a bounded wait
 *    that gave up) are recorded in the workspace's status word; read them with
 *    moe_read_device_status.
 *  - Layouts are row-major with the last index contiguous. bf16 is IEEE
 *    bfloat16; e4m3 is OCP FP8 E4M3 (float8_e4m3fn); UE8M0 is an unsigned
 *    8-bit power-of-two exponent, byte b meaning 2^(b-127).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,    /* bad shape, null pointer or misaligned pointer */
  MOE_ERR_UNSUPPORTED = -2,    /* valid request this build does not implement */
  MOE_ERR_SCALE_FORMAT = -3,   /* FP8 experts without UE8M0 block scales */
  MOE_ERR_WORKSPACE = -4,      /* workspace smaller than moe_workspace_size() */
  MOE_ERR_CUDA = -5,           /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = -6, /* a kernel gave up waiting (device status) */
  MOE_ERR_DEVICE_INDEX = -7,   /* topk_idx held an index outside [0,E) or a repeated expert */
  MOE_ERR_SCRATCH_LIMIT = -8   /* moe_forward_noalloc: the shape needs more scratch than the library holds */
} moe_status;

/* Expert weight type. */
typedef enum {
  MOE_DT_BF16 = 0, /* bf16 weights */
  MOE_DT_E4M3 = 1, /* e4m3 codes, one UE8M0 scale per 128x128 block; activations quantised 1x128 */
  MOE_DT_E2M1 = 2  /* FP4: e2m1 codes two per byte (even element in the low nibble), one UE8M0
                      scale per row and 32 consecutive elements along the reduction
                      dimension; activations stay bf16 */
} moe_wdtype;

/* Which execution of the expert matmuls to use (the page's decode-stage switch:
 * small token counts run better on a per-token form than on grouped GEMM tiles). */
typedef enum {
  MOE_PATH_AUTO = 0,    /* DECODE when T*k <= 32*E (bf16), 2*E (e2m1), E/2 (e4m3); else PREFILL */
  MOE_PATH_PREFILL = 1, /* expert-major permute + tcgen05 grouped GEMMs */
  MOE_PATH_DECODE = 2,  /* weight-streaming kernels, no tile padding */
  MOE_PATH_FUSED = 3    /* the DECODE path's permute, gate/up, down and combine in one
                           launch (section "Fused Mega MoE on Blackwell", on one GPU);
                           bf16 experts, T <= 256 and T*k <= 2048, else MOE_ERR_UNSUPPORTED */
} moe_path;

/* Gate activation of the gated expert MLP (section "SonicMoE": SwiGLU, GeGLU
 * and ReGLU map to silu, gelu and relu). h = act(gate) * up. */
typedef enum {
  MOE_ACT_SILU = 0, /* SwiGLU: silu(g) = g / (1 + exp(-g)) */
  MOE_ACT_GELU = 1, /* GeGLU:  gelu(g) = g/2 * (1 + erf(g / sqrt 2)), the exact form */
  MOE_ACT_RELU = 2  /* ReGLU:  relu(g) = max(g, 0) */
} moe_activation;

/* Problem shape. T tokens, hidden size H, expert intermediate size I,
 * E experts, top-k. Requirements: T >= 0; H and I positive multiples of 128;
 * 1 <= E <= 1024; 1 <= k <= E; T*k < 2^31 and every buffer below 2^31 rows.
 * bf16 experts whose H and I are multiples of 64 but not both of 128 form a
 * valid layer that this build does not run: moe_forward returns
 * MOE_ERR_UNSUPPORTED for them (and moe_workspace_size 0); other sizes are
 * MOE_ERR_INVALID_ARG. */
typedef struct {
  int32_t T, H, I, E, k;
  int32_t wdtype; /* moe_wdtype */
  int32_t path;   /* moe_path */
  int32_t act;    /* moe_activation */
} moe_shape;

/*
 * moe_route -- router top-k ("Experts backends", introduction: the router
 * picks k experts per token). For each token t: softmax over the E fp32 logits, the k
 * experts with the largest logits (equal logits: lower index first), slot j
 * holding the j-th largest, and their probabilities renormalised to sum to 1.
 *
 *   logits    [T, E] fp32, finite values (a NaN logit gives an unspecified choice)
 *   topk_idx  [T, k] int32 out
 *   topk_w    [T, k] fp32 out
 * Requirements: T >= 0, 1 <= E <= 1024, 1 <= k <= E. T == 0 is a no-op.
 */
moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k,
                     int32_t* topk_idx, float* topk_w, void* stream);

/*
 * moe_router -- the router GEMM fused with moe_route (the step ahead of the
 * experts: "Experts backends", introduction, the router that picks k experts;
 * backend table, row "sonicmoe", which fuses the router dispatch with the
 * expert GEMMs). For each token t:
 *   logits[t, e] = sum_h x[t, h] * w_router[e, h]   (bf16 inputs, fp32 accumulation)
 * then exactly moe_route's selection and weights on those fp32 logits (the
 * same code: for equal logits both give the same bits).
 *
 *   x          [T, H] bf16, 16-byte aligned
 *   w_router   [E, H] bf16, 16-byte aligned
 *   logits     [T, E] fp32 out, or NULL when the logits are not wanted
 *   topk_idx   [T, k] int32 out
 *   topk_w     [T, k] fp32 out
 * Requirements: T >= 0; H a positive multiple of 64 (at most 65536);
 * 1 <= k <= E <= 256. T == 0 is a no-op. Errors: MOE_ERR_INVALID_ARG before
 * any launch; MOE_ERR_CUDA for a failed launch. A bounded device wait that
 * gives up (never in normal operation) writes topk_idx = -1 for the tokens of
 * the affected 128-token tile.
 */
moe_status moe_router(const void* x, const void* w_router, int32_t T, int32_t H, int32_t E, int32_t k,
                      float* logits, int32_t* topk_idx, float* topk_w, void* stream);

/* Bytes of device workspace moe_forward needs for `shape` (an upper bound
 * that depends only on the shape; host-only, enqueues nothing). Returns 0 for
 * an invalid shape. */
size_t moe_workspace_size(const moe_shape* shape);

/*
 * moe_forward -- the routed expert forward ("Experts backends", introduction;
 * the "eager" row of the backend table is its reference definition):
 *   out[t] = sum_j topk_w[t,j] * Wd[e] (act(Wg[e] x[t]) * (Wu[e] x[t])),  e = topk_idx[t,j]
 * with act = shape->act (silu for SwiGLU experts).
 *
 *   x          [T, H] bf16
 *   topk_idx   [T, k] int32, each row k distinct experts in [0, E)
 *   topk_w     [T, k] fp32
 *   w_gate_up  [E, 2I, H]: rows 0..I-1 of expert e are the gate projection,
 *              rows I..2I-1 the up projection. bf16, or e4m3 codes, or
 *              e2m1 codes packed two per byte ([E, 2I, H/2] bytes).
 *   w_down     [E, H, I], bf16 or e4m3 codes, or packed e2m1 ([E, H, I/2] bytes).
 *   sw_gate_up e4m3: [E, 2I/128, H/128] UE8M0, one per 128x128 block;
 *              e2m1: [E, 2I, H/32] UE8M0, one per row and 32 elements; bf16: NULL
 *   sw_down    e4m3: [E, H/128, I/128]; e2m1: [E, H, I/32]; bf16: NULL
 *   out        [T, H] bf16 out
 *   workspace  >= moe_workspace_size(shape) bytes, 256-byte aligned; its
 *              previous contents do not matter. Calls that share a workspace
 *              must not overlap in time.
 * On the FUSED path the permute, expert and combine stages share one launch;
 * its layout, intermediates and results are those of the DECODE path.
 * Intermediates: h = act(gate) * up is rounded to bf16 and the expert output
 * y to bf16 (e4m3 experts: x and h are quantised per token and per 128-column
 * group with an fp32 scale amax/448, the FP8 reading of section "FP8 and FP4
 * quantized experts"; y stays bf16). The weighted sum runs in fp32 over j in
 * ascending order, so results are deterministic run to run.
 * e2m1 experts (section "FP8 and FP4 quantized experts": FP4-packed expert
 * weights with UE8M0 scales) keep bf16 activations: every e2m1 value times a
 * power of two is exact in bf16, so the layer is the bf16 layer on the
 * dequantised weights. On the PREFILL path (weights widened to bf16 in shared
 * memory ahead of the bf16 tensor-core MMA) H must be a multiple of 256, else
 * MOE_ERR_UNSUPPORTED; the DECODE path takes any H that is a multiple of 128.
 * Errors: MOE_ERR_SCALE_FORMAT when wdtype is e4m3 or e2m1 and a scale pointer is NULL
 * (the page's note: Blackwell kernels need UE8M0 scales and refuse plain float
 * ones instead of silently corrupting the output); MOE_ERR_UNSUPPORTED for
 * e4m3 weights on the PREFILL path with H not a multiple of 256 (the DECODE
 * path takes any H that is a multiple of 128).
 */
moe_status moe_forward(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                       const float* topk_w, const void* w_gate_up, const void* w_down,
                       const uint8_t* sw_gate_up, const uint8_t* sw_down, void* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* moe_forward that also records caller-created CUDA events (cudaEvent_t passed
 * as void*) between its stages, on `stream`: events[0] before the permute,
 * [1] after it, [2] after the gate/up stage, [3] after the down stage, [4]
 * after the combine. n_events must be 5 (or 0 with events NULL). */
moe_status moe_forward_timed(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                             const float* topk_w, const void* w_gate_up, const void* w_down,
                             const uint8_t* sw_gate_up, const uint8_t* sw_down, void* out,
                             void* workspace, size_t workspace_bytes, void* stream,
                             void* const* events, int32_t n_events);

/* Byte offsets, inside the workspace, of the intermediate buffers of the last
 * moe_forward with this shape (for tests and inspection; host-only).
 *   bm        rows per expert tile (128 for PREFILL, 1 for DECODE); path: resolved path
 *   cnt       int32 [E]    assignments per expert
 *   mt_base   int32 [E+1]  expert e owns rows [mt_base[e]*bm, mt_base[e+1]*bm)
 *   row_src   int32 [m_rows] assignment t*k+j held by each row, -1 for padding
 *   slot_row  int32 [T*k]  row of assignment t*k+j
 *   xa        permuted activations: bf16 [m_rows, H] (bf16 PREFILL only), e4m3
 *             codes [m_rows, H] (e4m3 PREFILL) or e4m3 codes [T, H] in token
 *             order (e4m3 DECODE: each token quantised once)
 *   xs        fp32 activation scales [rows of xa, H/128] (e4m3 only)
 *   h         bf16 [m_rows, I] (or e4m3 with fp32 scales hs [m_rows, I/128])
 *   y         bf16 [m_rows, H] expert outputs
 * m_rows is the allocated row capacity; only rows below mt_base[E]*bm are used.
 * An offset of SIZE_MAX means the buffer is not used by that path. */
typedef struct {
  size_t status, hdr, cnt, mt_base, row_src, slot_row, xa, xs, h, hs, y, total;
  int32_t bm, path, m_rows, reserved;
} moe_workspace_layout;

moe_status moe_workspace_query(const moe_shape* shape, moe_workspace_layout* layout);

/* Synchronises `stream`, then reads the device status word the last
 * moe_forward on this workspace wrote: MOE_OK, MOE_ERR_DEVICE_INDEX or
 * MOE_ERR_DEVICE_TIMEOUT (MOE_ERR_CUDA if the copy itself fails). */
moe_status moe_read_device_status(const void* workspace, void* stream);

/*
 * moe_set_test_hooks -- the failure-detection test's switches. Not for
 * production use; the page has no counterpart.
 *
 *  - wait_limit_ns: how long every bounded wait inside the GEMM kernels spins
 *    before it gives up, records MOE_ERR_DEVICE_TIMEOUT in the status word,
 *    lets its CTA's copies and MMAs in flight finish, frees its tensor memory
 *    and returns. 0 restores the default of 2 s; otherwise 1 ms to 60 s.
 *  - stall_gate_up_loads: 1 makes the prefill gate/up GEMM's producer issue no
 *    loads, so the MMA issuer waits on a barrier nothing completes and gives up
 *    after wait_limit_ns (on the FUSED path the gate/up tasks count no
 *    completions, so the down tasks' waits give up); the rest of the call then
 *    runs on stale intermediates and its output is garbage. 0 turns it off.
 *
 * Both are process-wide and read when a call is enqueued; do not change them
 * while other threads enqueue calls. Returns MOE_ERR_INVALID_ARG (and changes
 * nothing) for values outside those ranges.
 */
moe_status moe_set_test_hooks(int32_t stall_gate_up_loads, uint64_t wait_limit_ns);

/*
 * moe_forward_noalloc -- moe_forward for callers that cannot allocate device
 * memory. The page has no counterpart to this entry point; it exists for
 * callers that are handed only their input and output buffers (a plugin loaded
 * by a host framework that gives it no allocator) and for latency-critical
 * paths that must not call cudaMalloc, which can synchronise the device.
 *
 * Arguments and results are those of moe_forward, without the workspace: the
 * scratch space lives in a fixed array of MOE_NOALLOC_SCRATCH_BYTES bytes in
 * the library's own device memory (every GPU that loads the library holds it
 * until the process exits). Nothing is allocated or freed.
 *  - A shape whose moe_workspace_size() exceeds MOE_NOALLOC_SCRATCH_BYTES is
 *    rejected with MOE_ERR_SCRATCH_LIMIT before anything is enqueued.
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - All calls share the one array and leave their intermediates in it. Calls
 *    whose GPU work overlaps in time race on it: order them, for example by
 *    issuing them on one stream. Device-side errors are read with
 *    moe_forward_noalloc_status (moe_read_device_status takes a workspace).
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20) /* 8 MiB */
moe_status moe_forward_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                               const float* topk_w, const void* w_gate_up, const void* w_down,
                               const uint8_t* sw_gate_up, const uint8_t* sw_down, void* out, void* stream);

/* The device status of the last moe_forward_noalloc on the current device
 * (the counterpart of moe_read_device_status for the library's own scratch):
 * synchronises `stream`, then returns MOE_OK, MOE_ERR_DEVICE_INDEX or
 * MOE_ERR_DEVICE_TIMEOUT (MOE_ERR_CUDA if the read fails). Allocates nothing.
 * Like the forward's scratch, the word is shared by every call on the device:
 * read it after the call it should describe and before the next one. */
moe_status moe_forward_noalloc_status(void* stream);

/* Static description of a status code (never NULL). */
const char* moe_status_string(moe_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

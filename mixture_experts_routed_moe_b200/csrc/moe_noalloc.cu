// moe_forward_noalloc: moe_forward for callers that cannot allocate device
// memory.
//
// Some callers never get to call cudaMalloc: code loaded as a plugin by a host
// framework that hands it only its input and output buffers (no allocator
// handle), and latency-critical serving paths that forbid cudaMalloc because it
// can synchronise the device and take an unbounded time. For them this entry
// point runs the same forward with its scratch space in a fixed array that
// lives in the library's own device memory, so the caller passes inputs and
// outputs only.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes; every
// GPU that loads the library holds it until the process exits. Host code may
// not pass the array's name to a kernel (on the host it is only a stand-in for
// the symbol), so the device address is looked up with cudaGetSymbolAddress,
// once per device, with that device current; the first call on each device does
// this lookup and should therefore come before any stream capture. Every call
// shares the one array and leaves its contents behind: the forward clears what
// must start at zero (its status word) itself, and calls whose GPU work
// overlaps in time race on the array and must be ordered by the caller (for
// example by issuing them on one stream).
#include <atomic>
#include <mutex>

#include "moe_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (nullptr on error).
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                                          const float* topk_w, const void* w_gate_up, const void* w_down,
                                          const uint8_t* sw_gate_up, const uint8_t* sw_down, void* out,
                                          void* stream) {
  const size_t need = moe_workspace_size(shape);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return MOE_ERR_SCRATCH_LIMIT;
  void* scratch = scratch_address();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  return moe_forward(shape, x, topk_idx, topk_w, w_gate_up, w_down, sw_gate_up, sw_down, out, scratch,
                     kNoAllocScratchBytes, stream);
}

// The status word of the last moe_forward_noalloc on the current device: the
// forward writes device-side errors (a routing index out of range, a bounded
// wait that gave up) to the first word of its scratch, as moe_forward does to
// its workspace.
extern "C" moe_status moe_forward_noalloc_status(void* stream) {
  void* scratch = scratch_address();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  return moe_read_device_status(scratch, stream);
}

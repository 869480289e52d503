// moe_fp4_forward_noalloc: the MoE layer for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs inside a
// CUDA graph that was captured once and must not call cudaMalloc again, plugins whose
// host framework owns every allocation, or real-time loops where an allocator call
// could block.  This entry point runs the same kernels as moe_fp4_forward but takes its
// scratch from a fixed buffer that lives in this library's own device memory (a
// file-scope __device__ array), so the caller passes only inputs and outputs and the
// library calls no allocator.
#include <mutex>

#include "kernels.cuh"

namespace {

// The scratch buffer: allocated with the module on every device that loads this
// library and held until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch buffer on the current device.  The first call on a
// device looks it up with cudaGetSymbolAddress (the host-side name of a __device__
// array is only a stand-in and must never be passed to a kernel) and clears the
// workspace control block once, on the caller's stream so that it is ordered before
// the kernels the call launches; later calls reuse the cached address.
fp4_status scratch_for_current_device(void** out, cudaStream_t st) {
  int dev = 0;
  FP4_TRY_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return FP4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    FP4_TRY_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    FP4_TRY_CUDA(cudaMemsetAsync(p, 0, 256, st));   // control block (status word, timing counters)
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FP4_OK;
}

}  // namespace

namespace fp4 {
// The scratch of the current device (set up on first use), for the library's own
// entry points that act on it (status word, the bounded-wait self-test).
fp4_status noalloc_scratch(void** out, cudaStream_t st) { return scratch_for_current_device(out, st); }
}  // namespace fp4

extern "C" size_t moe_fp4_noalloc_capacity(void) { return kNoAllocScratchBytes; }

extern "C" fp4_status moe_fp4_forward_noalloc(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                                              const float* router_bias, int32_t T, int32_t k, void* y_bf16,
                                              void* stream) {
  const size_t need = moe_fp4_workspace_size(w, T, k);
  if (need == 0) {
    // invalid arguments: let the regular entry point name the refusal (it launches nothing)
    return moe_fp4_forward(w, x_bf16, router_w, router_bias, T, k, y_bf16, nullptr, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) return FP4_ERR_WORKSPACE;   // larger than the fixed buffer
  void* scratch = nullptr;
  FP4_TRY(scratch_for_current_device(&scratch, static_cast<cudaStream_t>(stream)));
  return moe_fp4_forward(w, x_bf16, router_w, router_bias, T, k, y_bf16, nullptr, scratch,
                         kNoAllocScratchBytes, stream);
}

extern "C" fp4_status moe_fp4_noalloc_status(void* stream) {
  void* scratch = nullptr;
  FP4_TRY(scratch_for_current_device(&scratch, static_cast<cudaStream_t>(stream)));
  return fp4_workspace_status(scratch, stream);
}

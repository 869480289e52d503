#include <atomic>
// C-ABI plumbing: status strings, CUDA error capture, device queries, tensor maps,
// and the workspace status word.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "kernels.cuh"

namespace fp4 {

static thread_local char g_last_error[256] = "";

fp4_status record_cuda_error(cudaError_t e, const char* where) {
  (void)cudaGetLastError();   // clear a non-sticky error so the next call starts clean
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
                static_cast<int>(e));
  return FP4_ERR_CUDA;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

fp4_status make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner_elems,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                        CUtensorMapSwizzle swz) {
  auto enc = get_encode();
  if (enc == nullptr) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return FP4_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner_elems, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return FP4_ERR_CUDA;
  }
  return FP4_OK;
}

fp4_status make_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                           CUtensorMapSwizzle swz) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner_bytes, rows, row_stride_bytes, box_inner,
                      box_rows, swz);
}

}  // namespace fp4

using namespace fp4;

extern "C" const char* fp4_status_string(fp4_status s) {
  switch (s) {
    case FP4_OK: return "FP4_OK";
    case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG";
    case FP4_ERR_EMPTY_SHAPE: return "FP4_ERR_EMPTY_SHAPE";
    case FP4_ERR_SHAPE_OVERFLOW: return "FP4_ERR_SHAPE_OVERFLOW";
    case FP4_ERR_ALIGNMENT: return "FP4_ERR_ALIGNMENT";
    case FP4_ERR_UNSUPPORTED: return "FP4_ERR_UNSUPPORTED";
    case FP4_ERR_WORKSPACE: return "FP4_ERR_WORKSPACE";
    case FP4_ERR_CUDA: return "FP4_ERR_CUDA";
    case FP4_ERR_TIMEOUT: return "FP4_ERR_TIMEOUT";
  }
  return "FP4_ERR_UNKNOWN";
}

extern "C" const char* fp4_last_error_string(void) { return g_last_error; }

extern "C" const char* fp4_version(void) { return "0.1.0"; }

namespace fp4 {
static std::atomic<unsigned long long> g_launches{0};
void note_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace fp4

extern "C" unsigned long long fp4_launch_count(void) { return fp4::g_launches.load(std::memory_order_relaxed); }

extern "C" fp4_status fp4_workspace_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return FP4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FP4_TRY_CUDA(cudaStreamSynchronize(st));
  uint32_t word = 0;
  FP4_TRY_CUDA(cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost));
  const uint32_t zero = 0;
  FP4_TRY_CUDA(cudaMemcpy(const_cast<void*>(workspace), &zero, sizeof(zero), cudaMemcpyHostToDevice));
  return (word & kStatusTimeout) ? FP4_ERR_TIMEOUT : FP4_OK;
}

extern "C" fp4_status fp4_workspace_kernel_stats(void* workspace, int reset, fp4_kernel_stats* out, void* stream) {
  if (workspace == nullptr) return FP4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FP4_TRY_CUDA(cudaStreamSynchronize(st));
  WsControl c;
  FP4_TRY_CUDA(cudaMemcpy(&c, workspace, sizeof(c), cudaMemcpyDeviceToHost));
  if (out != nullptr) {
    out->gate_up_ns = c.slot[0].total_ns;
    out->gate_up_launches = c.slot[0].launches;
    out->down_ns = c.slot[1].total_ns;
    out->down_launches = c.slot[1].launches;
  }
  if (reset) {
    for (int i = 0; i < 2; ++i) {
      c.slot[i].total_ns = 0ull;
      c.slot[i].launches = 0ull;
      c.slot[i].start_min = ~0ull;
      c.slot[i].end_max = 0ull;
      c.slot[i].done = 0u;
    }
    FP4_TRY_CUDA(cudaMemcpy(workspace, &c, sizeof(c), cudaMemcpyHostToDevice));
  }
  return FP4_OK;
}

extern "C" fp4_status fp4_mma_scales(const uint8_t* scales, int64_t rows, int64_t k, int64_t pair, uint8_t* out,
                                     void* stream) {
  int64_t n;
  FP4_TRY(checked_count({rows, k}, &n));
  if (pair < 0) return FP4_ERR_INVALID_ARG;
  if (k % 128 != 0) return FP4_ERR_UNSUPPORTED;
  if (pair == 0 && rows % 128 != 0) return FP4_ERR_UNSUPPORTED;
  if (pair > 0 && (pair % 64 != 0 || rows % (2 * pair) != 0)) return FP4_ERR_UNSUPPORTED;
  if (scales == nullptr || out == nullptr) return FP4_ERR_INVALID_ARG;
  if (!aligned16(scales) || !aligned16(out)) return FP4_ERR_ALIGNMENT;
  return launch_mma_scales(scales, rows, k, pair, out, static_cast<cudaStream_t>(stream));
}

extern "C" fp4_status fp4_nvfp4_mma_scales(const uint8_t* scales, int64_t rows, int64_t k, int64_t pair,
                                           uint8_t* out, void* stream) {
  int64_t n;
  FP4_TRY(checked_count({rows, k}, &n));
  if (pair < 0) return FP4_ERR_INVALID_ARG;
  if (k % 64 != 0) return FP4_ERR_UNSUPPORTED;
  if (pair == 0 && rows % 128 != 0) return FP4_ERR_UNSUPPORTED;
  if (pair > 0 && (pair % 64 != 0 || rows % (2 * pair) != 0)) return FP4_ERR_UNSUPPORTED;
  if (scales == nullptr || out == nullptr) return FP4_ERR_INVALID_ARG;
  if (!aligned16(scales) || !aligned16(out)) return FP4_ERR_ALIGNMENT;
  return launch_nv_scales(scales, rows, k, pair, out, static_cast<cudaStream_t>(stream));
}

namespace fp4 {
namespace {
// One CTA waits on an mbarrier phase that nothing completes; the bounded wait gives up
// after limit_ns, records the timeout in the status word and the kernel returns.
__global__ void wait_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_for(b, 0, status, limit_ns);
}
}  // namespace
}  // namespace fp4

extern "C" fp4_status fp4_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 2000000000ll) return FP4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace == nullptr) FP4_TRY(noalloc_scratch(&workspace, st));   // the no-alloc entry point's scratch
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP4_ERR_ALIGNMENT;
  wait_selftest_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(workspace),
                                         static_cast<unsigned long long>(limit_ns));
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch();
  return FP4_OK;
}

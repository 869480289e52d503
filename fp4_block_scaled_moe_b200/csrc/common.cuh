// Shared host and device helpers of the fp4moe CUDA library (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fp4moe.h"

namespace fp4 {

// ------------------------------------------------------------------------------------
// host side: status handling and checked arithmetic
// ------------------------------------------------------------------------------------

fp4_status record_cuda_error(cudaError_t e, const char* where);
// Count one accepted kernel launch (process-wide; read by fp4_launch_count).
void note_launch(unsigned n = 1);

#define FP4_TRY_CUDA(call)                                         \
  do {                                                             \
    cudaError_t e__ = (call);                                      \
    if (e__ != cudaSuccess) return fp4::record_cuda_error(e__, #call); \
  } while (0)

#define FP4_TRY(expr)                 \
  do {                                \
    fp4_status s__ = (expr);          \
    if (s__ != FP4_OK) return s__;    \
  } while (0)

// a * b and a + b on int64 with overflow detection
inline bool mul_ok(int64_t a, int64_t b, int64_t* out) { return !__builtin_mul_overflow(a, b, out); }
inline bool add_ok(int64_t a, int64_t b, int64_t* out) { return !__builtin_add_overflow(a, b, out); }

// product of dims, all > 0, without overflow; EMPTY_SHAPE / SHAPE_OVERFLOW otherwise
inline fp4_status checked_count(std::initializer_list<int64_t> dims, int64_t* out) {
  int64_t acc = 1;
  for (int64_t d : dims)
    if (d <= 0) return FP4_ERR_EMPTY_SHAPE;
  for (int64_t d : dims)
    if (!mul_ok(acc, d, &acc)) return FP4_ERR_SHAPE_OVERFLOW;
  *out = acc;
  return FP4_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int num_sms();                    // SM count of the current device (cached per device)
cudaError_t enable_pdl_attr(cudaLaunchAttribute* attr);

// Tensor maps (TMA descriptors) via the driver entry point, no libcuda link needed.
// inner_elems and box_inner count elements of dtype (for the 4-bit type, 4-bit elements).
fp4_status make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner_elems,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                        CUtensorMapSwizzle swz);
fp4_status make_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner_bytes, uint64_t rows,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                           CUtensorMapSwizzle swz);

// ------------------------------------------------------------------------------------
// device side
// ------------------------------------------------------------------------------------

constexpr uint32_t kStatusTimeout = 1u;   // bit set in the workspace status word
constexpr int kV2aLibBytes = 32 * 16 * 2;  // a V2a library: 32 codebooks of 16 fp16 entries

// Control block at the start of every workspace (first 256 bytes).
struct KernelSlot {
  unsigned long long start_min;   // per launch: earliest CTA start (reset by the router)
  unsigned long long end_max;     // per launch: latest CTA end
  unsigned int done;              // CTAs finished in this launch
  unsigned int pad;
  unsigned long long total_ns;    // accumulated over launches
  unsigned long long launches;
};
struct WsControl {
  uint32_t status;
  uint32_t unit_next[2];          // dynamic work-unit counters of the grouped kernels (gate_up, down)
  uint32_t pad;
  KernelSlot slot[2];             // 0: gate_up, 1: down
};
static_assert(sizeof(WsControl) <= 256, "control block");
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s bound on any device wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase. After limit_ns of %globaltimer records
// kStatusTimeout in *status and returns false; the caller then stops issuing work and
// leaves.
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint32_t* status,
                                              unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) {
      if (status) atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t* status) {
  return mbar_wait_for(bar, parity, status, kWaitLimitNs);
}

// 1D bulk copy global -> shared, completion counted on an mbarrier (bytes % 16 == 0).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 2D tiled TMA load (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Per-launch timing into a KernelSlot: call slot_begin after the dependency wait (one
// thread per CTA) and slot_end once every warp of the CTA is done (one thread per CTA).
__device__ __forceinline__ void slot_begin(KernelSlot* s) {
  if (s) atomicMin(&s->start_min, global_ns());
}
__device__ __forceinline__ void slot_end(KernelSlot* s) {
  if (!s) return;
  atomicMax(&s->end_max, global_ns());
  __threadfence();
  if (atomicAdd(&s->done, 1u) == gridDim.x * gridDim.y * gridDim.z - 1u) {
    __threadfence();
    const unsigned long long st = atomicAdd(&s->start_min, 0ull), en = atomicAdd(&s->end_max, 0ull);
    if (en > st) s->total_ns += en - st;
    s->launches += 1ull;
    s->done = 0u;
    s->start_min = ~0ull;
    s->end_max = 0ull;
  }
}

// Per-call reset of a workspace control block, by threads 0 and 1 of one CTA of the
// call's first kernel (after its dependency wait): status word, work-unit counters, and
// the per-launch timing fields of both kernel slots (the accumulated totals are kept).
__device__ __forceinline__ void ctrl_reset_per_call(WsControl* ctrl) {
  if (ctrl == nullptr || threadIdx.x >= 2) return;
  if (threadIdx.x == 0) ctrl->status = 0u;
  ctrl->unit_next[threadIdx.x] = 0u;
  KernelSlot* s = &ctrl->slot[threadIdx.x];
  s->start_min = ~0ull;
  s->end_max = 0ull;
  s->done = 0u;
}

// Programmatic dependent launch: wait for the producer grid's memory / let the next grid start.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Four bytes of packed E2M1 pairs -> four f16x2 registers (low nibble -> low half).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2,
                                                uint32_t& h3) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n"
      " mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n"
      " cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n"
      " cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}

// Two E4M3 bytes (low 16 bits of w) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t h;
  asm("{\n .reg .b16 lo;\n cvt.u16.u32 lo, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}" : "=r"(h) : "r"(w));
  return h;
}

// a * b + c per f16 half, rounded once (fma)
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// D = A (16x16 f16, row) * B (16x8 f16, col) + C, f32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9},"
      " {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B with C = 0 (fresh fp32 partial sums).
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9},"
      " {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// UE8M0 byte -> float 2^(b-127) (b = 0 -> 2^-127, b = 255 -> NaN).
__device__ __forceinline__ float ue8m0_to_f32(uint32_t b) {
  uint32_t bits = b << 23;
  bits = (b == 0u) ? 0x00400000u : bits;
  bits = (b == 255u) ? 0x7FC00000u : bits;
  return __uint_as_float(bits);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace fp4

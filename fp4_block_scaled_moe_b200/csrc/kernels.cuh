// Internal interfaces between the library's translation units.
#pragma once

#include "common.cuh"

namespace fp4 {

// Launch with the programmatic-stream-serialization attribute (PDL) when `pdl` is set:
// the kernel may start while the previous kernel on the stream finishes, and must call
// pdl_wait() before reading that kernel's results.
template <typename... KArgs, typename... Args>
fp4_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return record_cuda_error(e, "cudaLaunchKernelEx");
  return FP4_OK;
}

// Per-expert work units {expert, row tile, first slot, tokens} for the grouped kernels.
struct WorkListSpec {
  int4* units_a;     // gate_up units (or null)
  int4* units_b;     // down units (or null)
  int tiles_a;       // row tiles per expert, list a
  int tiles_b;
  int tok_group;     // tokens per unit
  int* n_units;      // [2] unit counts written by the router tail
};

struct RouteArgs {
  const void* x;
  const float* router_w;
  const float* router_bias;
  int T, H, E, k;
  const float* logits_in;
  float* logits;
  int32_t* ids;
  float* gw;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  __half* x16;       // optional f16 copy of x with per-token power-of-two scale
  int* sexp;         // [T] the exponents
  WsControl* ctrl;   // workspace control block, reset by the first kernel (or null)
  WorkListSpec wl;
  bool pdl_first;
};

fp4_status launch_route(const RouteArgs& a, cudaStream_t st);

// x (bf16 [T, H]) -> f16 with a per-row power-of-two scale exponent (see route.cu).
__global__ void x_to_f16_kernel(const uint16_t* __restrict__ x, int T, int H, __half* __restrict__ x16,
                                int* __restrict__ sexp);

// Grouped decode GEMV (register dequantisation + warp-level MMA), see decode.cu.
enum DecodeEpi { kEpiSwiglu = 0, kEpiDown = 1, kEpiLinear = 2 };

struct DecodeArgs {
  int fmt;                       // FP4_MXFP4 / FP4_NVFP4
  int epi;                       // DecodeEpi
  const uint8_t* codes;          // [rows_total, K/2]
  const uint8_t* scales;         // [rows_total, K/B]
  const float* tscale;           // [E] (NVFP4) or null
  int64_t rows_total;
  int K;
  int rows_per_expert;           // 2I (swiglu) or H (down) or N (linear)
  int inter;                     // I (swiglu: up rows start at I)
  // units: device list (+ count) or the static linear mapping
  const int4* units;
  const int* n_units;
  int static_tiles;              // linear: N / 64
  int static_T;                  // linear: T
  // activations: f16 rows
  const __half* x16;             // [rows, K]
  const int* sexp;               // per token exponent (swiglu / linear) or null
  const int32_t* perm;           // swiglu/down: slot -> pair
  int topk;
  const float* gw;               // down: gate weights per pair
  float limit;                   // swiglu clamp
  // outputs
  __half* h_out;                 // swiglu: [P, I]
  float* o_out;                  // down: [P, H]
  uint16_t* y_out;               // linear: [T, N] bf16
  int ldo;                       // leading dim of the output rows
  uint32_t* status;
  KernelSlot* slot;              // per-launch device timing (or null)
};

fp4_status launch_decode(const DecodeArgs& a, cudaStream_t st, bool pdl);

__global__ void combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv, int T, int k,
                               int H, uint16_t* __restrict__ y);

}  // namespace fp4

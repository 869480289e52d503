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
  note_launch();
  return FP4_OK;
}

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
  bool logits_only;  // stop after R1 (the grouped kernel finishes routing itself)
  bool pdl_first;
};

fp4_status launch_route(const RouteArgs& a, cudaStream_t st);

// The fixed scratch buffer of moe_fp4_forward_noalloc on the current device (no_alloc.cu).
fp4_status noalloc_scratch(void** out, cudaStream_t st);

// x (bf16 [T, H]) -> f16 with a per-row power-of-two scale exponent (see route.cu).
// ctrl (optional): the call's workspace control block, reset per call (see ctrl_reset_per_call).
__global__ void x_to_f16_kernel(const uint16_t* __restrict__ x, int T, int H, __half* __restrict__ x16,
                                int* __restrict__ sexp, WsControl* __restrict__ ctrl);

// Grouped decode GEMV (register dequantisation + warp-level MMA), see decode.cu.
enum DecodeEpi { kEpiSwiglu = 0, kEpiDown = 1, kEpiLinear = 2 };
// Where a grouped kernel finds its work units:
//   kModeList:   counts / offsets / perm already in global memory;
//   kModeRoute:  finish routing in the prologue from the logits (top-k, counts, perm);
//   kModeStatic: dense layer, units follow from (N, T).
enum DecodeMode { kModeList = 0, kModeRoute = 1, kModeStatic = 2 };
constexpr int kRouteMaxPairs = 1024;   // kModeRoute limits (shared-memory routing state)
constexpr int kRouteMaxExperts = 512;

struct DecodeArgs {
  int fmt;                       // FP4_MXFP4 / FP4_NVFP4 / FP4_CB4
  int epi;                       // DecodeEpi
  int mode;                      // DecodeMode
  const uint8_t* codes;          // [rows_total, K/2] (CB4: 4-bit codebook indices)
  const uint8_t* scales;         // [rows_total, K/B] (CB4: fp16 codebooks [rows_total, K/128, 16];
                                 //  V2a: 8-byte group records [rows_total, K/128])
  const uint8_t* lib;            // V2a: libraries [E_local][32][16] fp16
  const int32_t* sp_rowptr;      // CB4 sparse term: CSR over rows_total rows (or null)
  const int32_t* sp_col;
  const uint16_t* sp_val;        // fp16 bits
  const float* tscale;           // [E] (NVFP4) or null
  int64_t rows_total;
  int K;
  int rows_per_expert;           // 2I (swiglu) or H (down) or N (linear)
  int inter;                     // I (swiglu: up rows start at I)
  int E, T, topk;
  int e_begin, e_end;            // experts whose weights the call holds (codes row 0 = expert e_begin)
  const float* logits;           // kModeRoute: [T, E]
  int32_t* ids;                  // kModeRoute: written by CTA 0
  float* gw;                     // gate weights per pair (written by CTA 0 in kModeRoute)
  int32_t* counts;               // [E]
  int32_t* offsets;              // [E + 1]
  int32_t* perm;                 // [P] slot -> pair
  int32_t* inv;                  // [P] pair -> slot (written by CTA 0 in kModeRoute)
  int static_tiles;              // linear: N / 64
  int scale_tma;                 // set by launch_decode: scale bytes by TMA boxes (else per-row copies)
  // mixed-format fused buffers (or null): per local expert its format and the byte offsets of
  // its rows in `codes` and `scales`; only experts of this kernel's format get units
  const uint8_t* ex_fmt;
  const int64_t* row_off;
  const int64_t* srow_off;
  int64_t scale_rows_total;      // mixed-format buffers: rows of the scale buffer (else rows_total)
  const __half* x16;             // activation rows, f16 [rows, K] (null: dense layer converting x_bf16)
  const uint16_t* x_bf16;        // dense layer: bf16 x [T, K] when x16 is null
  const int* sexp;               // per token exponent (swiglu / linear) or null
  float limit;                   // swiglu clamp
  __half* h_out;                 // swiglu: [P, I]
  float* o_out;                  // down: [P, H]
  uint16_t* y_out;               // linear: [T, N] bf16
  int ldo;                       // leading dim of the output rows
  uint32_t* status;
  KernelSlot* slot;              // per-launch device timing (or null)
  uint32_t* unit_next;           // dynamic scheduling counter (zeroed by the router), or null
  int ksplit;                    // linear: units per 64-row tile and token group along K (0, 1: none)
  float* part;                   // linear with ksplit > 1: fp32 partial sums [ksplit][T][N]
};

fp4_status launch_decode(const DecodeArgs& a, cudaStream_t st, bool pdl);
// Dense layer: how many K shares (a power of two dividing the stage count) keep the
// layer's units within one wave of CTAs while [ks][T][N] fp32 partials fit part_bytes
int linear_ksplit(int fmt, int64_t K, int64_t T, int64_t N, size_t part_bytes);
// y[t, n] = bf16( sum over ks = 0, 1, ... of part[ks][t][n] ), n_elems = T N (multiple of 4)
fp4_status launch_linear_reduce(const float* part, int ksplit, int64_t n_elems, uint16_t* y, cudaStream_t st);

// The bf16 experts of a mixed-format fused buffer (dense16.cu): same units and epilogues
// as the grouped GEMV; weights at weights + offset[e - e_begin], bf16 rows of K.
struct Dense16Args {
  int epi;
  const uint8_t* weights;
  const int64_t* offset;
  const uint8_t* ex_fmt;
  int e_begin, e_end, E, K, rows_per_expert, inter, topk;
  const int32_t* counts;
  const int32_t* perm;
  const __half* x16;          // gate_up: token rows (scaled by 2^sexp); down: h rows by slot
  const int* sexp;
  float limit;
  __half* h_out;
  const float* gw;
  float* o_out;
  int ldo;
};
fp4_status launch_dense16(const Dense16Args& a, cudaStream_t st);

// y[t, :] = bf16(sum_j o[inv[t k + j], :]) in j order.
__global__ void combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv, int T, int k, int H,
                               uint16_t* __restrict__ y);
// y[t, :] = sum over j with e_begin <= ids[t k + j] < e_end of o[inv[t k + j], :], fp32, j order.
__global__ void combine_partial_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv,
                                       const int32_t* __restrict__ ids, int T, int k, int H, int e_begin,
                                       int e_end, float* __restrict__ y);
// out[i] = bf16(in[i]) (round to nearest even).
fp4_status launch_f32_to_bf16(const float* in, int64_t n, uint16_t* out, cudaStream_t st);


// Block-scaled tensor-core expert GEMM (MXFP4 weights x two-term MXFP8 activations).
// Scale atoms: 512 bytes holding the UE8M0 scales of 128 rows x 128 K (four 32-blocks):
// row r, block b at byte (r % 32) * 16 + (r / 32) * 4 + b -- the layout the TMEM scale
// copy (tcgen05.cp 32x128b, warpx4) reads.  Weights: atom (tile, K block) at
// (tile * (K / 128) + k / 128) * 512, a tile being 128 consecutive rows (down) or the
// 64 gate rows and 64 matching up rows of one expert (gate_up).  Activation terms: two
// atoms (rows 0-127, 128-255) per (token group, K block) at (group * (K / 128) + k / 128)
// * 1024, rows 2i, 2i + 1 = the two terms of the group's i-th slot; groups are the
// per-expert runs of ntok_cap slots, numbered across experts in expert order.
struct BsArgs {
  int epi;                        // kEpiSwiglu (gate_up + SwiGLU) or kEpiDown
  const uint8_t* codes;           // A: [rows_total][K/2] E2M1 pairs
  const uint8_t* a_atoms;         // A: scale atoms of the weights
  int64_t rows_total;
  int K;
  int rows_per_expert;
  int inter;                      // I (gate rows, then up rows, per expert)
  int E;
  int e_begin, e_end;             // experts whose weights the call holds (codes row 0 = expert e_begin)
  int P;                          // routed slots T*k
  int ntok_cap;                   // slots per token group
  const int32_t* counts;
  const uint8_t* b_q;             // B: [2P][K] E4M3, rows 2i and 2i+1 = terms of slot i
  const uint8_t* b_atoms;         // B: scale atoms per token group
  float limit;
  uint8_t* hq;                    // gate_up out: h terms [2P][I] E4M3
  uint8_t* h_atoms;               //              scale atoms per token group (K = I)
  const float* gw;                // down: gate weights by pair, perm: slot -> pair
  const int32_t* perm;
  float* o_out;                   // down out: [P][ldo] fp32, slot order
  int ldo;
  uint32_t* status;
  KernelSlot* slot;
  uint32_t* unit_next;
};
// slots per token group of the tensor-core kernels for T tokens (0 when unsupported)
int bs_ntok_cap(int T, int E);
// bytes of the activation scale atoms for P slots over E experts at this K
size_t bs_group_atom_bytes(int P, int E, int ntok_cap, int K);
// pair = 0: tiles of 128 consecutive rows; pair = I: gate_up tiles of 64 gate + 64 up rows
fp4_status launch_mma_scales(const uint8_t* scales, int64_t rows, int64_t K, int64_t pair, uint8_t* atoms,
                             cudaStream_t st);
bool bs_supported(int T, int E, int H, int I);
fp4_status launch_bs(const BsArgs& a, int T, cudaStream_t st);
// top-k + counts + stable slot order + activation split in one launch (T k <= 1024, E <= 512)
fp4_status launch_route_split(const float* logits, int T, int E, int k, const uint16_t* x, int H, int ntok_cap,
                              int32_t* ids, float* gw, int32_t* counts, int32_t* offsets, int32_t* perm,
                              int32_t* inv, uint8_t* q, uint8_t* atoms, cudaStream_t st);
fp4_status launch_split_x(const uint16_t* x, const int32_t* inv, const int32_t* counts, const int32_t* offsets,
                          int E, int k, int P, int H, int ntok_cap, uint8_t* q, uint8_t* atoms, cudaStream_t st);

// NVFP4 expert GEMMs on the tensor cores (kind::f16, weights widened to f16 on chip).
// Scale atoms: 512 bytes per (tile, 64-K stage) holding the four E4M3 block scales of each
// of the tile's 128 rows at byte 4 r; atom (tile, k / 64) at (tile * (K / 64) + k / 64) * 512,
// tiles as for the MXFP4 kernels (gate_up: 64 gate rows + the matching 64 up rows).
struct NvArgs {
  int epi;                        // kEpiSwiglu or kEpiDown
  const uint8_t* codes;           // [rows_total][K/2] E2M1 pairs
  const uint8_t* a_atoms;         // the weights' scale atoms
  const float* tscale;            // [E] per-expert tensor scale
  int64_t rows_total;
  int K;
  int rows_per_expert;
  int inter;
  int E;
  int e_begin, e_end;             // experts whose weights the call holds (codes row 0 = expert e_begin)
  int P;
  int ntok_cap;
  const int32_t* counts;
  const __half* b_rows;           // activations [P][K] f16, slot order
  const int* sx;                  // gate_up: power-of-two exponent of each slot's row
  float limit;
  __half* h_out;                  // gate_up out: h [P][I] f16, slot order
  const float* gw;                // down: gate weights by pair
  const int32_t* perm;
  float* o_out;                   // down out: [P][ldo] fp32, slot order
  int ldo;
  uint32_t* status;
  KernelSlot* slot;
  uint32_t* unit_next;
};
int nv_ntok_cap(int T, int E);
bool nv_supported(int T, int E, int H, int I);
fp4_status launch_nv(const NvArgs& a, int T, cudaStream_t st);
fp4_status launch_nv_scales(const uint8_t* scales, int64_t rows, int64_t K, int64_t pair, uint8_t* atoms,
                            cudaStream_t st);
// xs[i] = f16(x[perm[i] / k] 2^-sx[i]) for the P routed slots, sx as x_to_f16_kernel picks it.
fp4_status launch_gather_x16(const uint16_t* x, const int32_t* perm, int k, int P, int H, __half* xs, int* sx,
                             cudaStream_t st);

}  // namespace fp4

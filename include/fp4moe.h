/*
 * fp4moe: routed-expert mixture-of-experts layer on 4-bit block-scaled weights,
 * for NVIDIA B200 (sm_100a).  C ABI.
 *
 * Formats (defined in "XFP：质量地板驱动的自适应码本量化——3.4 位在双卡工作站跑通 397B MoE",
 * section 路线二：硬件格式（NVFP4 / MXFP4）):
 *   MXFP4  E2M1 elements (1 sign, 2 exponent, 1 mantissa bit), 32 per block, one
 *          UE8M0 power-of-two scale byte per block (value 2^(byte-127); 255 = NaN).
 *   NVFP4  E2M1 elements, 16 per block, one FP8 E4M3 scale byte per block, times one
 *          float32 per-tensor ("global") scale.
 *   CB4    4-bit indices into a 16-entry fp16 codebook per 128-weight group of a row,
 *          plus a sparse fp16 outlier term in CSR (same page, sections V2, 离群值提取,
 *          Lloyd 迭代, 子字节打包).
 *   V2A    N-bit codes into one of a matrix's 32 shared fp16 codebooks of 2^N entries,
 *          chosen per 128-weight group, with an fp16 scale and mid-point per group, plus
 *          the same sparse outlier term (same page, section V2a：共享码本库).
 * Packing: two 4-bit values per byte, the element with the even index in the low
 * nibble ("The gate that missed by 0.0202 pp", section "A fused tensor with two
 * dtypes in it").  Every tensor is row-major and contiguous:
 *   codes  uint8 [rows, K/2];  scales uint8 [rows, K/B] (B = 32 MXFP4, 16 NVFP4).
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers unless stated; the caller allocates and owns
 *     every buffer, including workspaces.  The library allocates no device memory,
 *     with one exception: the fixed 16 MiB module buffer (a __device__ array held on
 *     every device that loads the library) that moe_fp4_forward_noalloc uses as scratch.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  Only the status and statistics readers
 *     (fp4_workspace_status, moe_fp4_noalloc_status, fp4_workspace_kernel_stats)
 *     synchronise.
 *   - Shapes are checked before any launch with checked 64-bit arithmetic: a zero
 *     dimension returns FP4_ERR_EMPTY_SHAPE, a width, element count, byte size or
 *     index that overflows returns FP4_ERR_SHAPE_OVERFLOW ("TensorFold" pull request
 *     #1050: format classification refuses empty and oversized shapes by name).
 *     A refused call launches nothing and writes nothing.
 *   - Device pointers must be 16-byte aligned (FP4_ERR_ALIGNMENT otherwise).
 *   - CUDA errors are returned as FP4_ERR_CUDA; fp4_last_error_string() has the text.
 *   - Device-side waits are bounded; one that gives up records FP4_ERR_TIMEOUT in the
 *     workspace status word and the kernel returns (no trap, no hang).
 *   - No exceptions cross the ABI.  Entry points are reentrant; concurrent calls
 *     must not share a workspace.
 */
#ifndef FP4MOE_H
#define FP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef enum fp4_status {
  FP4_OK = 0,
  FP4_ERR_INVALID_ARG = 1,    /* null required pointer, bad enum, k > E, k > 32, ... */
  FP4_ERR_EMPTY_SHAPE = 2,    /* a dimension is zero (or negative) */
  FP4_ERR_SHAPE_OVERFLOW = 3, /* a derived width / count / byte size overflows */
  FP4_ERR_ALIGNMENT = 4,      /* K not a multiple of the block, or pointer misaligned */
  FP4_ERR_UNSUPPORTED = 5,    /* format / size combination this build does not run */
  FP4_ERR_WORKSPACE = 6,      /* workspace missing or smaller than required */
  FP4_ERR_CUDA = 7,           /* a CUDA runtime call failed */
  FP4_ERR_TIMEOUT = 8         /* a bounded device-side wait gave up */
} fp4_status;

typedef enum fp4_format {
  FP4_MXFP4 = 1,
  FP4_NVFP4 = 2,
  FP4_CB4 = 3,
  FP4_V2A = 4,
  FP4_DENSE_BF16 = 5 /* an expert kept in bf16 inside a mixed-format buffer (expert_format) */
} fp4_format;

typedef enum fp4_dtype { FP4_F32 = 0, FP4_BF16 = 1 } fp4_dtype;

/* Human-readable name of a status code (static storage). */
const char* fp4_status_string(fp4_status s);
/* Text of the last FP4_ERR_CUDA on the calling thread (static thread-local storage). */
const char* fp4_last_error_string(void);
/* Library version, e.g. "0.1.0". */
const char* fp4_version(void);
/* Number of CUDA kernel launches this library has issued in this process so far (all
 * entry points, all devices and streams; counted on the host when a launch is accepted,
 * whether it later runs or is captured into a graph).  Never fails. */
unsigned long long fp4_launch_count(void);

/*
 * fp4_pack: quantise `batch` matrices w [batch, n, k] (float32 or bf16, device) to
 * MXFP4 or NVFP4.  Outputs: codes [batch, n, k/2], scales [batch, n, k/B] and, for
 * NVFP4 only, tensor_scale [batch] (float32; one global scale per matrix; pass NULL
 * for MXFP4).
 *   MXFP4: per 32-block, e = clamp(floor(log2 amax) - 2, -127, 127) stored as e + 127
 *          (amax = 0 stores 0); element code = E2M1 round-to-nearest-even of v * 2^-e,
 *          saturating at 6, sign kept.  A block with a non-finite element stores scale
 *          0xFF and zero codes.
 *   NVFP4: ts = amax_tensor / 2688 (1 if amax_tensor = 0); per 16-block
 *          s = E4M3_rne_satfinite(amax_block / (6 ts)); code = E2M1_rne(v / (s ts)),
 *          all float32 operations correctly rounded, in that order; a block with s = 0
 *          stores zero codes; a block with a non-finite element stores scale 0x7F and
 *          zero codes; the tensor amax ignores non-finite elements.
 * Requirements: k % B == 0 (FP4_ERR_ALIGNMENT), batch, n, k > 0.
 * The result is bit-identical to the definition (integer outputs, exact).
 */
fp4_status fp4_pack(fp4_format fmt, const void* w, fp4_dtype w_dtype, int64_t batch, int64_t n,
                    int64_t k, uint8_t* codes, uint8_t* scales, float* tensor_scale, void* stream);

/*
 * fp4_unpack: inverse of fp4_pack.  out [batch, n, k] (float32 or bf16) receives
 * E2M1(code) * scale (* tensor_scale for NVFP4), rounded once to the output type
 * (round to nearest even).  Bit-identical to that definition.
 */
fp4_status fp4_unpack(fp4_format fmt, const uint8_t* codes, const uint8_t* scales,
                      const float* tensor_scale, int64_t batch, int64_t n, int64_t k, void* out,
                      fp4_dtype out_dtype, void* stream);

/*
 * CB4 packing: a 16-entry fp16 codebook per 128-weight group of each row plus a sparse
 * fp16 outlier term ("XFP：质量地板驱动的自适应码本量化", sections 离群值提取, Lloyd 迭代
 * and the V2 dense + sparse decomposition; 4-bit indices as in 子字节打包).
 * w [rows, k] float32 or bf16 (device), k % 128 == 0, rows * k < 2^31.  An outlier is
 * a weight with |w - mu| > threshold (float64 comparison).
 *   fp4_cb4_row_ptr: row_ptr [rows + 1] int32 (device) = exclusive scan of the outlier
 *     counts per row; row_ptr[rows] = nnz.  Call it first to size col and val.
 *   fp4_pack_cb4 (row_ptr from the first call): idx [rows, k/2] (even position in the low
 *     nibble), cb [rows, k/128, 16] fp16 bits, col [nnz] int32 (column within the row,
 *     ascending), val [nnz] fp16 bits.
 * Per group: outliers are replaced by mu; the entries start at the sorted values at
 * positions 8i + 4 (i = 0..15, the (i + 0.5)/16 quantiles); 20 Lloyd rounds assign each
 * weight to its nearest entry (ties to the lower index) and set each entry to the mean
 * of its members (summed in ascending position, float64; an empty entry is kept); the
 * entries are rounded to fp16 (nearest even) and every weight is assigned once more to
 * the nearest fp16 entry.  val = fp16(w - entry(idx)) at each outlier, so the dense
 * term plus the sparse term approximates w.  Deterministic.  col and val may be NULL
 * only when nnz == 0.  Errors: EMPTY_SHAPE, SHAPE_OVERFLOW, ALIGNMENT (k % 128, w, idx,
 * cb not 16-byte aligned), INVALID_ARG (threshold negative or not finite, mu not
 * finite, NULL pointers).
 */
fp4_status fp4_cb4_row_ptr(const void* w, fp4_dtype w_dtype, int64_t rows, int64_t k, double threshold,
                           double mu, int32_t* row_ptr, void* stream);
fp4_status fp4_pack_cb4(const void* w, fp4_dtype w_dtype, int64_t rows, int64_t k, double threshold, double mu,
                        const int32_t* row_ptr, uint8_t* idx, uint16_t* cb, int32_t* col, uint16_t* val,
                        void* stream);

/*
 * V2a packing ("XFP：质量地板驱动的自适应码本量化", section V2a：共享码本库, with 离群值提取 and
 * Lloyd 迭代): w [batch, rows, k] (float32 or bf16, device) holds `batch` matrices; each
 * gets one library of 32 fp16 codebooks of 2^n_bits entries (n_bits 2 or 4).
 *   - outliers |w - mu| > threshold leave the bulk (back-filled with mu) for an fp16
 *     residual CSR over the batch * rows rows; row_ptr [batch * rows + 1] comes from
 *     fp4_cb4_row_ptr with the same threshold and mu (call it first to size col / val);
 *   - per 128-group: mid = fp16((max + min) / 2), scale = fp16((max - min) / 2) of the
 *     bulk, z = (w - mid) / scale (0 when scale is 0);
 *   - LibFit: a Lloyd codebook per row over its z values (2^n_bits entries started at the
 *     sorted positions floor((2i + 1) k / 2^(n_bits + 1)), 20 rounds), then Lloyd over the
 *     rows' codebooks as vectors (32 entries started at the codebooks of span rank
 *     floor((2i + 1) rows / 64), 20 rounds, squared distance summed in entry order), the
 *     library rounded to fp16;
 *   - a group takes the library codebook with the least sum of squared distances to the
 *     nearest entry (in position order), each weight its nearest entry;
 *   - reconstruction fp16(mid + scale * entry), rounded once; val = fp16(w - it).
 * Float64 arithmetic, member means summed in ascending order, ties to the lower index:
 * deterministic.  Outputs: codes [batch * rows, k * n_bits / 8] (low bits first),
 * groups [batch * rows, k / 128] 8-byte records (mid fp16 | scale fp16 << 16 | library
 * index << 32), lib [batch, 32, 2^n_bits] fp16 bits, col / val [nnz] (may be NULL only
 * when nnz == 0).  workspace: fp4_pack_v2a_workspace_size bytes (256-byte aligned).
 * Limits: k % 128 == 0 (ALIGNMENT), k <= 4096, 32 <= rows <= 8192 (UNSUPPORTED).
 * fp4_unpack_v2a: the dense term as float32 (exact fp16 values) [batch, rows, k].
 */
size_t fp4_pack_v2a_workspace_size(int64_t batch, int64_t rows, int64_t k, int32_t n_bits);
fp4_status fp4_pack_v2a(const void* w, fp4_dtype w_dtype, int64_t batch, int64_t rows, int64_t k, int32_t n_bits,
                        double threshold, double mu, const int32_t* row_ptr, uint8_t* codes, uint64_t* groups,
                        uint16_t* lib, int32_t* col, uint16_t* val, void* workspace, size_t ws_bytes, void* stream);
fp4_status fp4_unpack_v2a(const uint8_t* codes, const uint64_t* groups, const uint16_t* lib, int64_t batch,
                          int64_t rows, int64_t k, int32_t n_bits, float* out, void* stream);

/*
 * moe_route: router of the MoE layer ("The gate that missed by 0.0202 pp", section
 * "A file is a census; a decode step is a sample": each token reads k of E experts).
 *   logits[t, e] = sum_h x[t, h] * router_w[e, h] + router_bias[e]   (float32 accumulate)
 *   topk_ids[t, :] = the k largest logits, descending, ties to the lower expert index
 *                    (a NaN logit ranks below every number)
 *   topk_w[t, :]   = softmax over those k logits (float32)
 *   counts[e]      = number of (t, j) routed to e;  offsets [E+1] = exclusive scan
 *   perm[slot]     = p = t*k + j, the pairs stably sorted by expert;  inv[p] = slot
 * x_bf16 [T, H] bf16, router_w [E, H] float32, router_bias [E] or NULL.
 * logits_in [T, E] (optional): when given, R1 is skipped and these logits are routed,
 * which makes every output of this call exactly reproducible.  logits_out [T, E] may
 * be NULL.  All outputs other than logits_out are required.
 * Requirements: 1 <= k <= min(E, 32), E <= 1024, T * k < 2^31.
 */
fp4_status moe_route(const void* x_bf16, const float* router_w, const float* router_bias, int32_t T,
                     int32_t H, int32_t E, int32_t k, const float* logits_in, float* logits_out,
                     int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                     int32_t* perm, int32_t* inv, void* stream);

/*
 * Expert weights of one MoE layer: gate_up [E, 2I, H] (rows 0..I-1 gate, I..2I-1 up)
 * and down [E, H, I], all experts of a matrix fused into one buffer with one stride.
 *   MXFP4 / NVFP4: *_codes, *_scales as in fp4_pack with batch = E; NVFP4 also
 *     *_tscale [E] (one global scale per expert matrix); MXFP4 leaves them NULL.
 *   CB4: *_codes are packed 4-bit indices [E, rows, K/2]; *_cb the fp16 codebooks
 *     [E, rows, K/128, 16] (uint16 bit patterns); the sparse term is one CSR over the
 *     E*rows rows of the fused matrix: *_rowptr [E*rows + 1], *_col [nnz] (column in
 *     the row), *_val [nnz] fp16 bits.  Forward = dense codebook term + sparse term.
 *   V2A (N = 4 in the layer): *_codes packed 4-bit codes [E, rows, K/2]; *_scales the
 *     8-byte group records [E, rows, K/128] (fp4_pack_v2a); *_cb the libraries
 *     [E, 32, 16] fp16 bits (one per expert matrix); the sparse term as for CB4.
 * swiglu_limit: L of h = silu(min(g, L)) * clamp(u, -L, L), finite, 0 < L <= 128.  Experts
 *   apply the model's gated SwiGLU together with its clamp ("GLM-5.3-Flash-MXFP4" model
 *   card, section "Verification compute and EAGLE"); the workload uses L = 7.
 */
typedef struct fp4_moe_weights {
  fp4_format fmt;
  int32_t num_experts; /* E */
  int32_t hidden;      /* H */
  int32_t inter;       /* I */
  float swiglu_limit;
  const uint8_t* gu_codes;
  const uint8_t* gu_scales;
  const float* gu_tscale;
  const uint8_t* dn_codes;
  const uint8_t* dn_scales;
  const float* dn_tscale;
  const uint16_t* gu_cb;
  const int32_t* gu_rowptr;
  const int32_t* gu_col;
  const uint16_t* gu_val;
  const uint16_t* dn_cb;
  const int32_t* dn_rowptr;
  const int32_t* dn_col;
  const uint16_t* dn_val;
  /* Expert-GEMM kernels: 0 = chosen per call (MXFP4: tensor cores when T*k >= 4E, i.e.
   * four or more tokens per expert on average, or whenever gu_mma_scales / dn_mma_scales
   * are given; NVFP4: tensor cores when T*k >= 64E; else the CUDA-core GEMV), 1 = CUDA-core
   * grouped GEMV, 2 = tensor-core GEMM (MXFP4: block-scaled kind::mxf8f6f4; NVFP4: weights widened to
   * f16 on chip, kind::f16; FP4_ERR_UNSUPPORTED for CB4 or unsupported shapes).
   * Any other value is FP4_ERR_INVALID_ARG. */
  int32_t kernel_variant;
  /* Tensor-core variant only (may be NULL): the gate_up / down scales re-laid by
   * fp4_mma_scales (MXFP4) or fp4_nvfp4_mma_scales (NVFP4).  When NULL, each call re-lays
   * them into the workspace. */
  const uint8_t* gu_mma_scales;
  const uint8_t* dn_mma_scales;
  /* Expert parallelism: the weight tensors hold experts [expert_begin, expert_begin +
   * local_experts) of the E routed experts (their first dimension is local_experts; the
   * router still covers all E).  local_experts = 0 (with expert_begin = 0) means all E.
   * moe_fp4_forward needs all E; moe_fp4_forward_partial takes any range.  A range
   * outside [0, E] is FP4_ERR_INVALID_ARG. */
  int32_t expert_begin;
  int32_t local_experts;
  /* Mixed formats in one fused buffer ("The gate that missed by 0.0202 pp", section "A fused
   * tensor with two dtypes in it": a fused MoE buffer packs every expert of a layer into one
   * tensor, an expert excluded from quantisation keeps its full-width bf16 rows beside the
   * half-width packed experts, so the format and the stride belong to the expert, not to the
   * tensor).  When expert_format is non-NULL (device uint8 [local experts]), fmt must be
   * FP4_MXFP4 and each expert is FP4_MXFP4 or FP4_DENSE_BF16:
   *   *_codes    one fused byte buffer of *_bytes bytes; expert e's rows start at byte
   *              *_offset[e] (device int64 [local experts], a multiple of K/2 with K = H for
   *              gate_up, I for down): MXFP4 codes [rows, K/2] or bf16 [rows, K];
   *   *_scales   one fused buffer of *_scale_bytes bytes holding the MXFP4 experts' scales
   *              [rows, K/32] at *_scale_offset[e] (a multiple of K/32; unused for bf16).
   * Such layers run on the CUDA-core kernels (kernel_variant 2 is FP4_ERR_UNSUPPORTED). */
  const uint8_t* expert_format;
  const int64_t* gu_offset;
  const int64_t* gu_scale_offset;
  const int64_t* dn_offset;
  const int64_t* dn_scale_offset;
  int64_t gu_bytes;
  int64_t gu_scale_bytes;
  int64_t dn_bytes;
  int64_t dn_scale_bytes;
} fp4_moe_weights;

/*
 * fp4_mma_scales: MXFP4 scales [rows, k/32] (UE8M0, row-major, as fp4_pack writes them)
 * re-laid for the tensor-core expert kernels: one 512-byte atom per tile of 128 rows and
 * 128 k, atom (tile, k/128) at (tile * (k/128) + k/128) * 512, the scale of tile row r
 * and 32-block b inside it at (r % 32) * 16 + (r / 32) * 4 + b % 4 -- the order the
 * tensor-memory scale copy reads.  pair = 0: tile t = rows 128t .. 128t+127 (down
 * weights; rows % 128 == 0).  pair = I > 0: rows are gate_up rows of experts with 2I rows
 * each (rows % 2I == 0, I % 64 == 0) and tile (e, t) = gate rows t*64 .. t*64+63 followed
 * by up rows I + t*64 .. I + t*64+63 of expert e, numbered e * (I/64) + t.  k % 128 == 0.
 * out: rows * k / 32 bytes.  FP4_ERR_UNSUPPORTED on other shapes; pointers 16-byte
 * aligned.  No counterpart in the pages: a layout of this library's MMA kernels.
 */
fp4_status fp4_mma_scales(const uint8_t* scales, int64_t rows, int64_t k, int64_t pair, uint8_t* out, void* stream);

/*
 * fp4_nvfp4_mma_scales: NVFP4 scales [rows, k/16] (E4M3, row-major, as fp4_pack writes
 * them) re-laid for the tensor-core NVFP4 expert kernels: one 512-byte atom per tile of
 * 128 rows and 64 k, atom (tile, k/64) at (tile * (k/64) + k/64) * 512, the four block
 * scales of tile row r at bytes 4r .. 4r+3 (block order).  Tiles as in fp4_mma_scales
 * (pair = 0: 128 consecutive rows, rows % 128 == 0; pair = I > 0: 64 gate rows then the
 * matching 64 up rows of each expert with 2I rows, I % 64 == 0).  k % 64 == 0.
 * out: rows * k / 16 bytes.  FP4_ERR_UNSUPPORTED on other shapes; pointers 16-byte
 * aligned.  No counterpart in the pages: a layout of this library's MMA kernels.
 */
fp4_status fp4_nvfp4_mma_scales(const uint8_t* scales, int64_t rows, int64_t k, int64_t pair, uint8_t* out,
                                void* stream);

/* Optional copies of the routing results of a forward call (each pointer may be NULL). */
typedef struct fp4_route_out {
  float* logits;     /* [T, E] */
  int32_t* topk_ids; /* [T, k] */
  float* topk_w;     /* [T, k] */
  int32_t* counts;   /* [E]    */
  int32_t* offsets;  /* [E+1]  */
  int32_t* perm;     /* [T*k]  */
  int32_t* inv;      /* [T*k]  */
} fp4_route_out;

/* Bytes of workspace moe_fp4_forward needs for these weights, T tokens and top-k
 * (0 when the arguments are invalid). */
size_t moe_fp4_workspace_size(const fp4_moe_weights* w, int32_t T, int32_t k);

/* The expert-GEMM kernels moe_fp4_forward runs for these weights, T tokens and top-k
 * (resolving kernel_variant 0): 1 = CUDA-core grouped GEMV, 2 = tensor-core GEMM;
 * 0 when the arguments are invalid.  Host only, launches nothing. */
int32_t moe_fp4_expert_kernels(const fp4_moe_weights* w, int32_t T, int32_t k);

/*
 * moe_fp4_forward: the routed-expert MoE layer.
 *   route (as moe_route) -> for every routed pair (t, j), e = topk_ids[t, j]:
 *   [g; u] = W_gu(e) x_t,  h = silu(min(g, L)) * clamp(u, -L, L),  o = W_d(e) h,
 *   y_t = bf16( sum_{j=0..k-1} topk_w[t, j] * o_{t, j} )   (fixed j order; deterministic)
 * x_bf16 [T, H], router_w [E, H] float32, router_bias [E] or NULL, y_bf16 [T, H].
 * workspace: device buffer of at least moe_fp4_workspace_size bytes, 256-byte aligned;
 * its first 64 bytes hold the status word read by fp4_workspace_status.
 * route: optional host struct of device pointers receiving the routing results.
 * Accuracy: float32 accumulation of exactly dequantised weights; against a float64
 * evaluation of the same definition, rel. Frobenius error <= 5e-3 and per-element
 * |err| <= 2e-2 (|ref| + 1).  The MXFP4 tensor-core variant feeds x and h to the
 * MMA as two E4M3 terms per value with a power-of-two scale per 32 (residual about
 * 2^-8 of each value); the NVFP4 tensor-core variant and the CUDA-core variant feed
 * them as float16, x with a power-of-two scale per row (h unscaled).
 */
fp4_status moe_fp4_forward(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                           const float* router_bias, int32_t T, int32_t k, void* y_bf16,
                           const fp4_route_out* route, void* workspace, size_t ws_bytes,
                           void* stream);

/*
 * moe_fp4_forward_partial: one rank's share of an expert-parallel MoE layer.  The experts
 * are split over ranks, each holding a contiguous range of them (expert_begin,
 * local_experts); every rank routes all T tokens over all E experts and computes
 *   y_partial[t, :] = sum over j with expert_begin <= e_tj < expert_begin + local_experts
 *                     of topk_w[t, j] * o_{t, j}        (float32, j order)
 * so that the layer output is bf16(sum over ranks of y_partial): the ranks' partial sums
 * are exchanged with an all-reduce (the expert-parallel placement of "GLM-5.3-Flash-MXFP4",
 * sections "Serving performance against AMD" and "Serving uplift versus the official FP8
 * checkpoint": TP4/EP4), and fp4_f32_to_bf16 rounds the sum.  y_partial [T, H] float32;
 * other arguments, workspace and errors as moe_fp4_forward.
 */
fp4_status moe_fp4_forward_partial(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                                   const float* router_bias, int32_t T, int32_t k, float* y_partial,
                                   const fp4_route_out* route, void* workspace, size_t ws_bytes, void* stream);

/* out[i] = bf16(in[i]), round to nearest even, for n float32 values (device pointers).
 * The last step of an expert-parallel layer after its partial sums are reduced. */
fp4_status fp4_f32_to_bf16(const float* in, int64_t n, void* out, void* stream);

/*
 * fp4_linear: dense W4A16 layer y [T, N] = bf16(x [T, K] . W^T), W [N, K] in MXFP4 or
 * NVFP4 (codes [N, K/2], scales [N, K/B], tensor_scale [1] for NVFP4, else NULL).
 * 4-bit weights read with bf16 activations ("TensorFold" pull request #1050,
 * W4A16_NVFP4).  workspace: at least fp4_linear_workspace_size(T, K) bytes, 256-byte
 * aligned; its first 256 bytes are a control block like moe_fp4_forward's, read by
 * fp4_workspace_status and by fp4_workspace_kernel_stats (gate_up_* = the linear kernel).
 * Up to 64 tokens the GEMV converts x itself (no separate conversion launch): it starts
 * streaming the weights before it waits for the previous kernel on the stream (so
 * consecutive layers overlap), and reads x and writes y only after that wait.  The
 * weights must therefore be complete when the call is made (not written by a kernel that
 * is still running on the stream and lets dependents start early); this library's packers
 * finish before any later kernel starts.  When the layer has too few 64-row tiles x
 * 8-token groups to fill the GPU, K is split over several CTAs and a second small kernel
 * adds their fp32 partial sums in a fixed order (y stays deterministic).  The timing
 * fields of the control block start valid when the workspace was zero-filled before its
 * first use (the Python binding's workspaces are).
 */
size_t fp4_linear_workspace_size(int32_t T, int64_t K);
fp4_status fp4_linear(fp4_format fmt, const void* x_bf16, int32_t T, int64_t K, const uint8_t* codes,
                      const uint8_t* scales, const float* tensor_scale, int64_t N, void* y_bf16,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * fp4_workspace_status: synchronise `stream`, then return the status word recorded in
 * `workspace` by the last call that used it (FP4_OK, or FP4_ERR_TIMEOUT when a bounded
 * device wait gave up), and clear it.  `workspace` is a device pointer.
 */
fp4_status fp4_workspace_status(const void* workspace, void* stream);

/*
 * fp4_selftest_wait_timeout: exercises the failure path of the library's bounded device
 * waits without faulting the GPU.  Launches one kernel that waits on a shared-memory
 * barrier phase nothing completes; after limit_ns (1 .. 2e9) of device time the wait
 * gives up, sets the timeout bit in the status word of `workspace` (a workspace of
 * moe_fp4_forward, 256-byte aligned; NULL = the scratch of moe_fp4_forward_noalloc on
 * the current device) and the kernel returns.  fp4_workspace_status (for NULL:
 * moe_fp4_noalloc_status) then reports FP4_ERR_TIMEOUT and clears the word; the context
 * stays usable.  No counterpart in the pages.
 */
fp4_status fp4_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream);

/*
 * moe_fp4_forward_noalloc: the same layer as moe_fp4_forward, for callers that cannot
 * allocate device memory (no counterpart in the pages: an addition of this library).
 * Some callers have no way to provide a workspace: a CUDA graph captured once that must
 * not allocate again, a plugin whose host framework owns every allocation, or a
 * real-time loop where an allocator call could block.  This entry point takes its
 * scratch from a fixed buffer inside the library's own device memory instead, so the
 * caller passes only inputs and outputs; it calls no cudaMalloc, no cudaFree and no
 * allocating library routine.
 *   - Capacity: moe_fp4_noalloc_capacity() bytes (16 MiB) on every device that loads the
 *     library, held until the process exits.  A call whose moe_fp4_workspace_size(w, T, k)
 *     exceeds it returns FP4_ERR_WORKSPACE and launches nothing.  16 MiB covers decode
 *     batches such as 64 tokens x top-8 at hidden 6144, intermediate 2048 on the CUDA-core
 *     expert kernels (14.8 MiB), and 16 tokens x top-8 at hidden 2048, intermediate 768
 *     on the tensor-core kernels (3.3 MiB with re-laid scale atoms); the tensor-core
 *     kernels at the larger shape need 36.6 MiB and are refused.
 *   - The first call on a device looks up the buffer's device address and clears its
 *     control block; make that first call before any stream capture on that device.
 *   - All calls on a device share the one buffer and it keeps the previous call's
 *     contents (each call rewrites everything it reads).  Calls that overlap on the GPU
 *     -- on two streams, or from two host threads -- race on it: serialise them.
 *   - Arguments, accuracy and errors otherwise as moe_fp4_forward (no routing outputs).
 *   - A bounded device wait that gives up records FP4_ERR_TIMEOUT in the buffer's status
 *     word, as for a workspace; read it with moe_fp4_noalloc_status.  Each call clears
 *     the word when it starts, so read it after the call it should report on.
 * moe_fp4_noalloc_status: synchronise `stream`, then return the status word of the
 * current device's buffer (FP4_OK or FP4_ERR_TIMEOUT) and clear it, as
 * fp4_workspace_status does for a caller's workspace.
 */
size_t moe_fp4_noalloc_capacity(void);
fp4_status moe_fp4_forward_noalloc(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                                   const float* router_bias, int32_t T, int32_t k, void* y_bf16, void* stream);
fp4_status moe_fp4_noalloc_status(void* stream);

/*
 * Per-kernel device time of the grouped expert kernels, accumulated in the workspace
 * by the kernels themselves from the device's global nanosecond timer: for each launch,
 * (last CTA finished) - (first CTA past its dependency wait).  Counters accumulate over
 * calls that use the same workspace until reset; fp4_workspace_kernel_stats synchronises
 * `stream`, copies them to *out (host), and zeroes them when `reset` is non-zero.
 * A freshly allocated workspace must be reset once before its counters mean anything.
 */
typedef struct fp4_kernel_stats {
  uint64_t gate_up_ns;        /* summed device time of the gate_up + SwiGLU kernel */
  uint64_t gate_up_launches;
  uint64_t down_ns;           /* summed device time of the down (gate-weighted) kernel */
  uint64_t down_launches;
} fp4_kernel_stats;

fp4_status fp4_workspace_kernel_stats(void* workspace, int reset, fp4_kernel_stats* out, void* stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* FP4MOE_H */

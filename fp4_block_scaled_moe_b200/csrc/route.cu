// Router of the MoE layer: logits, top-k with softmax gate weights, per-expert
// histogram and the stable token permutation; plus the per-expert work lists the
// grouped expert kernels consume.
//
// "The gate that missed by 0.0202 pp", section "A file is a census; a decode step is a
// sample": a decode step reads the trunk plus the k experts the router picks per token.
#include <algorithm>

#include "kernels.cuh"
#include "routing.cuh"

namespace fp4 {

// ---------------------------------------------------------------------------------
// x (bf16) -> f16 with a per-token power-of-two scale, so that every value fits the
// f16 range: x16 = x * 2^-s_t with max|x_t| * 2^-s_t in [2^14, 2^15).  One warp per row.
// ---------------------------------------------------------------------------------
__device__ void x_row_to_f16(const uint16_t* __restrict__ xrow, int H, __half* __restrict__ out,
                             int* __restrict__ sexp) {
  const int lane = threadIdx.x & 31;
  float amax = 0.f;
  for (int h = lane * 8; h < H; h += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(xrow + h);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  int s = 0;
  if (amax > 0.f && isfinite(amax)) {
    int e;
    frexpf(amax, &e);            // amax = f 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
    s = (e - 1) - 14;
  }
  for (int h = lane * 8; h < H; h += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(xrow + h);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half lo = __float2half_rn(ldexpf(__uint_as_float(w[j] << 16), -s));
      const __half hi = __float2half_rn(ldexpf(__uint_as_float(w[j] & 0xFFFF0000u), -s));
      o[j] = static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
    }
    *reinterpret_cast<uint4*>(out + h) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (lane == 0) *sexp = s;
}

__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t* __restrict__ x, int T, int H,
                                                       __half* __restrict__ x16, int* __restrict__ sexp,
                                                       WsControl* __restrict__ ctrl) {
  pdl_wait();
  if (blockIdx.x == 0) ctrl_reset_per_call(ctrl);
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row < T) x_row_to_f16(x + static_cast<int64_t>(row) * H, H, x16 + static_cast<int64_t>(row) * H, sexp + row);
  pdl_launch_dependents();
}

// Routed slots in slot order as f16 rows with their own power-of-two scale (one warp per
// slot): the activation operand of the NVFP4 tensor-core expert kernels.
__global__ void __launch_bounds__(256) gather_x16_kernel(const uint16_t* __restrict__ x,
                                                         const int32_t* __restrict__ perm, int k, int P, int H,
                                                         __half* __restrict__ xs, int* __restrict__ sx) {
  pdl_wait();
  const int warps = gridDim.x * 8;
  for (int i = blockIdx.x * 8 + (threadIdx.x >> 5); i < P; i += warps)
    x_row_to_f16(x + static_cast<int64_t>(perm[i] / k) * H, H, xs + static_cast<int64_t>(i) * H, sx + i);
  pdl_launch_dependents();
}

fp4_status launch_gather_x16(const uint16_t* x, const int32_t* perm, int k, int P, int H, __half* xs, int* sx,
                             cudaStream_t st) {
  const int grid = std::max(1, std::min((P + 7) / 8, num_sms() * 8));
  return launch_pdl(gather_x16_kernel, dim3(grid), dim3(256), 0, st, true, x, perm, k, P, H, xs, sx);
}

// ---------------------------------------------------------------------------------
// R1: logits[t, e] = sum_h x[t, h] w_r[e, h] + bias[e], float32 accumulation.
// CTA (e, token group of 16), 16 warps splitting H.  The router weights do not depend
// on the previous kernel, so the first slice of them is fetched before the dependency
// wait.  CTA (e, group) also converts row e (+ multiples of E) of the group to f16, and
// CTA (0, 0) clears the per-call counters of the grouped kernels.
// ---------------------------------------------------------------------------------
constexpr int kTokGroup = 16;
constexpr int kLogitsWarps = 16;
constexpr int kWrPrefetch = 4;   // float4 per lane fetched before the dependency wait

// f16 copy of one row with the whole CTA: x16 = x * 2^-s, max|x| * 2^-s in [2^14, 2^15)
__device__ void x_row_to_f16_cta(const uint16_t* __restrict__ xrow, int H, __half* __restrict__ out,
                                 int* __restrict__ sexp, float* red) {
  float amax = 0.f;
  for (int h = threadIdx.x * 8; h < H; h += blockDim.x * 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(xrow + h);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  __syncthreads();
  int s = 0;
  if (amax > 0.f && isfinite(amax)) {
    int e;
    frexpf(amax, &e);            // amax = f 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
    s = (e - 1) - 14;
  }
  for (int h = threadIdx.x * 8; h < H; h += blockDim.x * 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(xrow + h);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half lo = __float2half_rn(ldexpf(__uint_as_float(w[j] << 16), -s));
      const __half hi = __float2half_rn(ldexpf(__uint_as_float(w[j] & 0xFFFF0000u), -s));
      o[j] = static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
    }
    *reinterpret_cast<uint4*>(out + h) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (threadIdx.x == 0) *sexp = s;
}

__global__ void __launch_bounds__(kLogitsWarps * 32) logits_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ bias, int T, int H,
    int E, float* __restrict__ logits, __half* __restrict__ x16, int* __restrict__ sexp,
    WsControl* __restrict__ ctrl) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x;
  const int hspan = ((H + kLogitsWarps - 1) / kLogitsWarps + 3) & ~3;
  const int h0 = warp * hspan, h1 = min(H, h0 + hspan);
  const float* wrow = wr + static_cast<int64_t>(e) * H;
  float4 wpre[kWrPrefetch];
#pragma unroll
  for (int q = 0; q < kWrPrefetch; ++q) {
    const int h = h0 + lane * 4 + q * 128;
    wpre[q] = (h < h1) ? *reinterpret_cast<const float4*>(wrow + h) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  pdl_wait();
  if (ctrl != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 2) {
    if (threadIdx.x == 0) ctrl->status = 0u;
    ctrl->unit_next[threadIdx.x] = 0u;
    KernelSlot* s = &ctrl->slot[threadIdx.x];
    s->start_min = ~0ull;
    s->end_max = 0ull;
    s->done = 0u;
  }
  __shared__ float red[kLogitsWarps];
  const int t0 = blockIdx.y * kTokGroup;
  const int nt = min(kTokGroup, T - t0);
  if (x16 != nullptr)
    for (int i = e; i < nt; i += E)
      x_row_to_f16_cta(x + static_cast<int64_t>(t0 + i) * H, H, x16 + static_cast<int64_t>(t0 + i) * H,
                       sexp + t0 + i, red);
  float acc[kTokGroup];
#pragma unroll
  for (int i = 0; i < kTokGroup; ++i) acc[i] = 0.f;
  auto accumulate = [&](const float4 wv, int h) {
#pragma unroll
    for (int i = 0; i < kTokGroup; ++i) {
      if (i < nt) {
        const uint2 u = *reinterpret_cast<const uint2*>(x + static_cast<int64_t>(t0 + i) * H + h);
        acc[i] = fmaf(__uint_as_float(u.x << 16), wv.x, acc[i]);
        acc[i] = fmaf(__uint_as_float(u.x & 0xFFFF0000u), wv.y, acc[i]);
        acc[i] = fmaf(__uint_as_float(u.y << 16), wv.z, acc[i]);
        acc[i] = fmaf(__uint_as_float(u.y & 0xFFFF0000u), wv.w, acc[i]);
      }
    }
  };
#pragma unroll
  for (int q = 0; q < kWrPrefetch; ++q) {
    const int h = h0 + lane * 4 + q * 128;
    if (h < h1) accumulate(wpre[q], h);
  }
  for (int h = h0 + lane * 4 + kWrPrefetch * 128; h < h1; h += 128)
    accumulate(*reinterpret_cast<const float4*>(wrow + h), h);
#pragma unroll
  for (int i = 0; i < kTokGroup; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
  __shared__ float part_sum[kLogitsWarps][kTokGroup];
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < kTokGroup; ++i) part_sum[warp][i] = acc[i];
  __syncthreads();
  if (threadIdx.x < nt) {
    const int i = threadIdx.x;
    float sum = 0.f;
    for (int p = 0; p < kLogitsWarps; ++p) sum += part_sum[p][i];
    if (bias) sum += bias[e];
    logits[static_cast<int64_t>(t0 + i) * E + e] = sum;
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------------
// R2: top-k per token (one warp per token) and softmax over the selected logits.
// Order key: larger logit first; equal logits -> lower expert; NaN below every number.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int32_t* __restrict__ ids, float* __restrict__ gw) {
  pdl_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t < T)
    topk_warp(logits + static_cast<int64_t>(t) * E, E, k, ids + static_cast<int64_t>(t) * k,
              gw + static_cast<int64_t>(t) * k);
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------------
// R3: counts, offsets, stable permutation and inverse; optional work lists.
// One CTA of 1024 threads.  Warp w owns the contiguous pair chunk [w C, (w+1) C); the
// per-warp histograms give each warp its starting cursor per expert, and inside a warp
// pairs are placed in ascending order with a match/rank step, which keeps the sort stable.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) perm_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;                       // [32][E]
  int32_t* off = hist + 32 * E;             // [E + 1]
  int32_t* scan = off + E + 1;              // [1024] block scan scratch
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 32 * E; i += 1024) hist[i] = 0;
  __syncthreads();
  const int C = (P + 31) / 32;
  const int c0 = warp * C, c1 = min(P, c0 + C);
  for (int p = c0 + lane; p < c1; p += 32) atomicAdd(&hist[warp * E + ids[p]], 1);
  __syncthreads();
  // per expert: exclusive scan over warps, and total count
  int my_count = 0;
  for (int e = threadIdx.x; e < E; e += 1024) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int h = hist[w * E + e];
      hist[w * E + e] = run;
      run += h;
    }
    counts[e] = run;
    if (e == static_cast<int>(threadIdx.x)) my_count = run;
  }
  // exclusive scan of counts over experts (E <= 1024: one value per thread)
  const int v = (static_cast<int>(threadIdx.x) < E) ? my_count : 0;
  scan[threadIdx.x] = v;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int add = (static_cast<int>(threadIdx.x) >= o) ? scan[threadIdx.x - o] : 0;
    __syncthreads();
    scan[threadIdx.x] += add;
    __syncthreads();
  }
  if (static_cast<int>(threadIdx.x) < E) {
    off[threadIdx.x] = scan[threadIdx.x] - v;
    offsets[threadIdx.x] = scan[threadIdx.x] - v;
  }
  if (threadIdx.x == 0) { off[E] = P; offsets[E] = P; }
  __syncthreads();
  // cursors: hist[w][e] += off[e]
  for (int i = threadIdx.x; i < 32 * E; i += 1024) hist[i] += off[i % E];
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int base = c0; base < c1; base += 32) {
    const int p = base + lane;
    const bool live = p < c1;
    const int e = live ? ids[p] : -1 - lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(peers & lt);
    int slot = 0;
    if (live) slot = hist[warp * E + e] + rank;
    __syncwarp();
    if (live && rank == 0) hist[warp * E + e] += __popc(peers);
    __syncwarp();
    if (live) {
      perm[slot] = p;
      inv[p] = slot;
    }
  }
  pdl_launch_dependents();
}

// ---- R1 for many tokens: tensor-core tiles -------------------------------------------
// logits = x Wr^T + bias with x exactly bf16 and Wr float32 split exactly (to 2^-24 of
// each weight) into three bf16 terms, hi + mid + lo; bf16 x bf16 products are exact and
// accumulate in float32 on the tensor cores (mma.sync m16n8k16).  CTA tile: 128 tokens x
// 64 experts, K chunks of 32, two shared-memory stages; 8 warps of 32 x 32.
constexpr int kLgBM = 128, kLgBN = 64, kLgBK = 32, kLgLd = kLgBK + 8;   // row pitch 80 B
constexpr int kLgStage = (kLgBM + 3 * kLgBN) * kLgLd * 2;                // bytes per stage

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9},"
      " {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// bf16 (round to nearest even) of v and the exact remainder v - bf16(v)
__device__ __forceinline__ uint32_t bf16_split(float v, float& rest) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  rest = v - __bfloat162float(h);
  return static_cast<uint32_t>(__bfloat16_as_ushort(h));
}

__global__ void __launch_bounds__(256) logits_mma_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                                                         const float* __restrict__ bias, int T, int H, int E,
                                                         float* __restrict__ logits, WsControl* __restrict__ ctrl) {
  extern __shared__ __align__(16) uint8_t lg_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  const int t0 = blockIdx.x * kLgBM, e0 = blockIdx.y * kLgBN;
  const uint32_t sb = smem_u32(lg_smem);
  // loader assignment: x tile 128 rows x 4 chunks of 16 B; W tile 64 rows x 8 float4
  auto x_src = [&](int kt, int i) {
    const int c = tid + 256 * i, r = c >> 2, ch = c & 3;
    const int tr = min(t0 + r, T - 1);
    return x + static_cast<int64_t>(tr) * H + kt * kLgBK + ch * 8;
  };
  auto x_dst = [&](int stage, int i) {
    const int c = tid + 256 * i, r = c >> 2, ch = c & 3;
    return sb + stage * kLgStage + (r * kLgLd + ch * 8) * 2;
  };
  float4 wv[2];
  auto w_load = [&](int kt) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + 256 * i, r = c >> 3, ch = c & 7;
      const int er = min(e0 + r, E - 1);
      wv[i] = *reinterpret_cast<const float4*>(wr + static_cast<int64_t>(er) * H + kt * kLgBK + ch * 4);
    }
  };
  auto w_store = [&](int stage) {
    uint16_t* base = reinterpret_cast<uint16_t*>(lg_smem + stage * kLgStage) + kLgBM * kLgLd;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + 256 * i, r = c >> 3, ch = c & 7;
      const float v[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
      uint32_t hi[4], mid[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float r1, r2, r3;
        hi[j] = bf16_split(v[j], r1);
        mid[j] = bf16_split(r1, r2);
        lo[j] = bf16_split(r2, r3);
      }
      const int o = r * kLgLd + ch * 4;
      *reinterpret_cast<uint2*>(base + o) = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
      *reinterpret_cast<uint2*>(base + kLgBN * kLgLd + o) = make_uint2(mid[0] | (mid[1] << 16), mid[2] | (mid[3] << 16));
      *reinterpret_cast<uint2*>(base + 2 * kLgBN * kLgLd + o) = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
    }
  };

  const int nk = H / kLgBK;
  w_load(0);
#pragma unroll
  for (int i = 0; i < 2; ++i) cp_async16(x_dst(0, i), x_src(0, i));
  asm volatile("cp.async.commit_group;" ::: "memory");
  pdl_wait();
  if (ctrl != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 2) {
    if (threadIdx.x == 0) ctrl->status = 0u;
    ctrl->unit_next[threadIdx.x] = 0u;
    KernelSlot* s = &ctrl->slot[threadIdx.x];
    s->start_min = ~0ull;
    s->end_max = 0ull;
    s->done = 0u;
  }
  w_store(0);
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;

  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) {
      w_load(kt + 1);
#pragma unroll
      for (int i = 0; i < 2; ++i) cp_async16(x_dst(cur ^ 1, i), x_src(kt + 1, i));
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const uint32_t xs = sb + cur * kLgStage, ws = xs + kLgBM * kLgLd * 2;
    // this chunk's products accumulate on the tensor cores from zero; the running sums
    // take them with IEEE float adds, which bounds the tensor-core rounding to one chunk
    float part[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) part[i][j][c] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kLgBK; kk += 16) {
      uint32_t af[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int row = wm * 32 + i * 16 + (lane & 15), col = kk + (lane >> 4) * 8;
        ldsm_x4(xs + (row * kLgLd + col) * 2, af[i][0], af[i][1], af[i][2], af[i][3]);
      }
#pragma unroll
      for (int term = 0; term < 3; ++term) {
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
          const int n = wn * 32 + jp * 16 + (lane & 7) + ((lane >> 4) << 3), col = kk + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(ws + ((term * kLgBN + n) * kLgLd + col) * 2, b0, b1, b2, b3);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            mma_bf16_16816(part[i][2 * jp], af[i], b0, b1);
            mma_bf16_16816(part[i][2 * jp + 1], af[i], b2, b3);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][j][c] += part[i][j][c];
    if (kt + 1 < nk) {
      w_store(cur ^ 1);
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();
  }
  pdl_launch_dependents();
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + wn * 32 + j * 8 + 2 * tq;
    const float b_0 = (bias != nullptr && e < E) ? bias[e] : 0.f;
    const float b_1 = (bias != nullptr && e + 1 < E) ? bias[e + 1] : 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + wm * 32 + i * 16 + g + 8 * h;
        if (t < T) {
          float* out = logits + static_cast<int64_t>(t) * E;
          if (e < E) out[e] = acc[i][j][2 * h] + b_0;
          if (e + 1 < E) out[e + 1] = acc[i][j][2 * h + 1] + b_1;
        }
      }
    }
  }
}

size_t perm_smem_bytes(int E) { return (32 * static_cast<size_t>(E) + E + 1 + 1024) * sizeof(int32_t); }

fp4_status launch_route(const RouteArgs& a, cudaStream_t st) {
  const int P = a.T * a.k;
  if (a.logits_in == nullptr && a.x16 == nullptr && a.T >= 256 && a.H % kLgBK == 0) {
    static thread_local bool configured = false;
    if (!configured) {
      FP4_TRY_CUDA(cudaFuncSetAttribute(logits_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kLgStage));
      configured = true;
    }
    dim3 grid((a.T + kLgBM - 1) / kLgBM, (a.E + kLgBN - 1) / kLgBN);
    FP4_TRY(launch_pdl(logits_mma_kernel, grid, dim3(256), static_cast<size_t>(2 * kLgStage), st, a.pdl_first,
                       static_cast<const uint16_t*>(a.x), a.router_w, a.router_bias, a.T, a.H, a.E, a.logits,
                       a.ctrl));
  } else if (a.logits_in == nullptr) {
    dim3 grid(a.E, (a.T + kTokGroup - 1) / kTokGroup);
    FP4_TRY(launch_pdl(logits_kernel, grid, dim3(kLogitsWarps * 32), 0, st, a.pdl_first,
                       static_cast<const uint16_t*>(a.x), a.router_w, a.router_bias, a.T, a.H, a.E,
                       a.logits, a.x16, a.sexp, a.ctrl));
  } else if (a.x16 != nullptr) {
    FP4_TRY(launch_pdl(x_to_f16_kernel, dim3((a.T + 7) / 8), dim3(256), 0, st, a.pdl_first,
                       static_cast<const uint16_t*>(a.x), a.T, a.H, a.x16, a.sexp, a.ctrl));
  }
  if (a.logits_only) return FP4_OK;
  const float* lg = a.logits_in ? a.logits_in : a.logits;
  FP4_TRY(launch_pdl(topk_kernel, dim3((a.T + 7) / 8), dim3(256), 0, st, true, lg, a.T, a.E, a.k,
                     a.ids, a.gw));
  const size_t smem = perm_smem_bytes(a.E);
  static thread_local int configured_e = -1;
  if (smem > 48 * 1024 && configured_e < a.E) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(perm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(perm_smem_bytes(kMaxE))));
    configured_e = kMaxE;
  }
  FP4_TRY(launch_pdl(perm_kernel, dim3(1), dim3(1024), smem, st, true, a.ids, P, a.E, a.counts,
                     a.offsets, a.perm, a.inv));
  return FP4_OK;
}

}  // namespace fp4

using namespace fp4;

extern "C" fp4_status moe_route(const void* x_bf16, const float* router_w, const float* router_bias,
                                int32_t T, int32_t H, int32_t E, int32_t k, const float* logits_in,
                                float* logits_out, int32_t* topk_ids, float* topk_w, int32_t* counts,
                                int32_t* offsets, int32_t* perm, int32_t* inv, void* stream) {
  int64_t n;
  FP4_TRY(checked_count({T, E}, &n));
  if (k <= 0) return FP4_ERR_EMPTY_SHAPE;
  if (logits_in == nullptr) FP4_TRY(checked_count({T, H, E}, &n));
  int64_t P;
  if (!mul_ok(T, k, &P) || P >= (int64_t(1) << 31)) return FP4_ERR_SHAPE_OVERFLOW;
  if (k > E || k > 32 || E > kMaxE) return FP4_ERR_INVALID_ARG;
  if (!topk_ids || !topk_w || !counts || !offsets || !perm || !inv) return FP4_ERR_INVALID_ARG;
  if (logits_in == nullptr) {
    if (!x_bf16 || !router_w) return FP4_ERR_INVALID_ARG;
    if (H % 8 != 0) return FP4_ERR_ALIGNMENT;
    if (!aligned16(x_bf16) || !aligned16(router_w)) return FP4_ERR_ALIGNMENT;
    if (logits_out == nullptr) return FP4_ERR_INVALID_ARG;   // R1 needs somewhere to write
  }
  RouteArgs a{};
  a.x = x_bf16; a.router_w = router_w; a.router_bias = router_bias;
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.logits_in = logits_in; a.logits = logits_out;
  a.ids = topk_ids; a.gw = topk_w; a.counts = counts; a.offsets = offsets; a.perm = perm; a.inv = inv;
  a.pdl_first = false;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FP4_TRY(launch_route(a, st));
  if (logits_in != nullptr && logits_out != nullptr && logits_out != logits_in)
    FP4_TRY_CUDA(cudaMemcpyAsync(logits_out, logits_in, static_cast<size_t>(T) * E * sizeof(float),
                                 cudaMemcpyDeviceToDevice, st));
  return FP4_OK;
}

// fp4_pack / fp4_unpack: MXFP4 and NVFP4 block quantisation on the device.
//
// Formats: "XFP：质量地板驱动的自适应码本量化", section 路线二：硬件格式（NVFP4 / MXFP4）
// (E2M1 elements; 32-element blocks with a power-of-two UE8M0 scale for MXFP4;
// 16-element blocks with an FP8 E4M3 scale times a float32 per-tensor scale for
// NVFP4), two values per byte ("The gate that missed by 0.0202 pp", section "A fused
// tensor with two dtypes in it").  Every float32 operation that decides a code is a
// correctly rounded intrinsic (__fdiv_rn, __fmul_rn) in the order the header states,
// so the integer outputs are exact.
#include <algorithm>

#include "common.cuh"

namespace fp4 {
namespace {

constexpr int kThreads = 256;

// |a| -> E2M1 magnitude code by round-to-nearest, ties to the even mantissa, saturating.
// The midpoints between neighbouring magnitudes {0,.5,1,1.5,2,3,4,6} are
// .25 .75 1.25 1.75 2.5 3.5 5; at a midpoint the neighbour with mantissa bit 0 wins.
__device__ __forceinline__ uint32_t e2m1_code(float q) {
  const float a = fabsf(q);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) +
               (a > 5.0f);
  return c | (signbit(q) ? 8u : 0u);
}

// floor(log2(a)) of a finite a > 0, subnormals included.
__device__ __forceinline__ int ilog2_floor(float a) {
  const uint32_t b = __float_as_uint(a);
  const int ex = static_cast<int>(b >> 23);
  if (ex != 0) return ex - 127;
  return (31 - __clz(b & 0x7FFFFFu)) - 149;
}

// Non-negative float -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_code(float s) {
  if (s != s) return 0x7Fu;
  if (!(s < 448.0f)) return 0x7Eu;                    // s >= 448 (NaN is handled by the caller)
  if (s < 0.015625f) {                                // below 2^-6: subnormal grid of 2^-9
    return static_cast<uint32_t>(__float2int_rn(s * 512.0f));   // 0..8; 8 is 2^-6 = code 0x08
  }
  int e = ilog2_floor(s);                             // -6 .. 8
  const float m = s * __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // [1, 2), exact
  int q = __float2int_rn((m - 1.0f) * 8.0f);          // exact operands; RNE
  if (q == 8) { q = 0; ++e; }
  const uint32_t code = (static_cast<uint32_t>(e + 7) << 3) | static_cast<uint32_t>(q);
  return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  float v = (e == 0) ? static_cast<float>(m) * 0.001953125f
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) v = __uint_as_float(0x7FC00000u);
  return (code & 0x80u) ? -v : v;
}

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]);

template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(p);
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(u.x << 16);
  v[1] = __uint_as_float(u.x & 0xFFFF0000u);
  v[2] = __uint_as_float(u.y << 16);
  v[3] = __uint_as_float(u.y & 0xFFFF0000u);
}

// Group-of-G-lanes max (G a power of two dividing 32, groups aligned in the warp).
template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
template <int G>
__device__ __forceinline__ uint32_t group_or(uint32_t v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v |= __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// MXFP4: each lane quantises 4 consecutive elements; 8 lanes form one 32-element block.
template <typename T>
__global__ void __launch_bounds__(kThreads) mxfp4_pack_kernel(const T* __restrict__ w, int64_t n4,
                                                                uint16_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // every lane of a warp runs the same trip count so the shuffles stay convergent
  const int64_t base0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  for (int64_t base = base0; base < n4; base += stride) {
    const int64_t i = base + (threadIdx.x & 31);
    const bool live = i < n4;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (live) load4<T>(w + i * 4, v);
    float amax = 0.f;
    uint32_t bad = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool fin = isfinite(v[j]);
      bad |= fin ? 0u : 1u;
      amax = fin ? fmaxf(amax, fabsf(v[j])) : amax;
    }
    amax = group_max<8>(amax);
    bad = group_or<8>(bad);
    const int e_s = (amax > 0.f) ? max(min(ilog2_floor(amax) - 2, 127), -127) : -127;
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e_s) << 23);   // 2^-e_s, normal
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) packed |= e2m1_code(v[j] * inv) << (4 * j);
    if (bad) packed = 0;
    if (live) {
      codes[i] = static_cast<uint16_t>(packed);
      if ((threadIdx.x & 7) == 0) scales[i >> 3] = bad ? 0xFFu : static_cast<uint8_t>(e_s + 127);
    }
  }
}

// NVFP4 pass 1: per-matrix amax of the finite |w| (float bits, atomicMax on the ordered ints).
template <typename T>
__global__ void __launch_bounds__(kThreads) nvfp4_amax_kernel(const T* __restrict__ w, int64_t per4,
                                                                uint32_t* __restrict__ amax_bits) {
  const int64_t b = blockIdx.y;
  const T* wb = w + b * per4 * 4;
  float m = 0.f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < per4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[4];
    load4<T>(wb + i * 4, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) m = isfinite(v[j]) ? fmaxf(m, fabsf(v[j])) : m;
  }
  m = group_max<32>(m);
  __shared__ float red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = 1; j < kThreads / 32; ++j) m = fmaxf(m, red[j]);
    atomicMax(amax_bits + b, __float_as_uint(m));
  }
}

// NVFP4 pass 2: each lane quantises 4 elements; 4 lanes form one 16-element block.
template <typename T>
__global__ void __launch_bounds__(kThreads) nvfp4_pack_kernel(const T* __restrict__ w, int64_t per4,
                                                                const uint32_t* __restrict__ amax_bits,
                                                                uint16_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales) {
  const int64_t b = blockIdx.y;
  const float amax_t = __uint_as_float(amax_bits[b]);
  const float ts = (amax_t > 0.f) ? __fdiv_rn(amax_t, 2688.0f) : 1.0f;
  const float six_ts = __fmul_rn(6.0f, ts);
  const T* wb = w + b * per4 * 4;
  uint16_t* cb = codes + b * per4;
  uint8_t* sb = scales + b * (per4 >> 2);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t base0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  for (int64_t base = base0; base < per4; base += stride) {
    const int64_t i = base + (threadIdx.x & 31);
    const bool live = i < per4;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (live) load4<T>(wb + i * 4, v);
    float amax = 0.f;
    uint32_t bad = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool fin = isfinite(v[j]);
      bad |= fin ? 0u : 1u;
      amax = fin ? fmaxf(amax, fabsf(v[j])) : amax;
    }
    amax = group_max<4>(amax);
    bad = group_or<4>(bad);
    const float s = __fdiv_rn(amax, six_ts);
    const uint32_t sc = e4m3_code(s);
    const float denom = __fmul_rn(e4m3_value(sc), ts);
    uint32_t packed = 0;
    if (denom > 0.f) {
#pragma unroll
      for (int j = 0; j < 4; ++j) packed |= e2m1_code(__fdiv_rn(v[j], denom)) << (4 * j);
    }
    if (bad) packed = 0;
    if (live) {
      cb[i] = static_cast<uint16_t>(packed);
      if ((threadIdx.x & 3) == 0) sb[i >> 2] = bad ? 0x7Fu : static_cast<uint8_t>(sc);
    }
  }
}

__global__ void nvfp4_finalize_kernel(float* tensor_scale, int64_t batch) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b < batch) {
    const float amax_t = tensor_scale[b];   // holds the amax bits written by pass 1
    tensor_scale[b] = (amax_t > 0.f) ? __fdiv_rn(amax_t, 2688.0f) : 1.0f;
  }
}

// Round a double to the nearest bfloat16 (ties to even), subnormals and overflow included.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  if (x != x) return 0x7FC0u;
  if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
  const double a = fabs(x);
  int e = ilogb(a);
  if (e < -126) e = -126;
  const double q = rint(scalbn(a, 7 - e));            // exact scaling; ties to even
  const double r = scalbn(q, e - 7);
  uint32_t bits;
  if (r >= 0x1p128) bits = 0x7F800000u;
  else bits = __float_as_uint(static_cast<float>(r));   // r is a bf16 value: exact in float
  return static_cast<uint16_t>((bits >> 16) | (signbit(x) ? 0x8000u : 0u));
}

// Unpack: one thread per element; value computed exactly in double, rounded once.
template <int kFmt, int kOut>
__global__ void __launch_bounds__(kThreads) unpack_kernel(const uint8_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales,
                                                            const float* __restrict__ tscale,
                                                            int64_t per_batch, int64_t total,
                                                            void* __restrict__ out) {
  constexpr int B = (kFmt == FP4_MXFP4) ? 32 : 16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t byte = codes[i >> 1];
    const uint32_t c = (i & 1) ? (byte >> 4) : (byte & 15u);
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, static_cast<int>(e) - 1);
    if (c & 8u) v = -v;
    const uint32_t s = scales[i / B];
    double r;
    if (kFmt == FP4_MXFP4) {
      r = (s == 255u) ? __longlong_as_double(0x7FF8000000000000ll) : ldexp(v, static_cast<int>(s) - 127);
    } else {
      const int64_t b = i / per_batch;
      r = v * static_cast<double>(e4m3_value(s)) * static_cast<double>(tscale[b]);
    }
    if (kOut == FP4_F32) static_cast<float*>(out)[i] = __double2float_rn(r);
    else static_cast<uint16_t*>(out)[i] = f64_to_bf16_rne(r);
  }
}

int grid_for(int64_t work, int per_cta) {
  const int64_t want = (work + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" fp4_status fp4_pack(fp4_format fmt, const void* w, fp4_dtype w_dtype, int64_t batch,
                               int64_t n, int64_t k, uint8_t* codes, uint8_t* scales,
                               float* tensor_scale, void* stream) {
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4) return FP4_ERR_UNSUPPORTED;
  if (w_dtype != FP4_F32 && w_dtype != FP4_BF16) return FP4_ERR_INVALID_ARG;
  int64_t total;
  FP4_TRY(checked_count({batch, n, k}, &total));
  int64_t bytes_in;
  if (!mul_ok(total, w_dtype == FP4_F32 ? 4 : 2, &bytes_in)) return FP4_ERR_SHAPE_OVERFLOW;
  const int B = (fmt == FP4_MXFP4) ? 32 : 16;
  if (k % B != 0) return FP4_ERR_ALIGNMENT;
  if (!w || !codes || !scales) return FP4_ERR_INVALID_ARG;
  if (fmt == FP4_NVFP4 && !tensor_scale) return FP4_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) ||
      (tensor_scale && (reinterpret_cast<uintptr_t>(tensor_scale) & 3u)))
    return FP4_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n4 = total / 4;
  if (fmt == FP4_MXFP4) {
    const int grid = grid_for(n4, kThreads);
    if (w_dtype == FP4_F32)
      mxfp4_pack_kernel<float><<<grid, kThreads, 0, st>>>(static_cast<const float*>(w), n4,
                                                          reinterpret_cast<uint16_t*>(codes), scales);
    else
      mxfp4_pack_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(w), n4, reinterpret_cast<uint16_t*>(codes), scales);
    FP4_TRY_CUDA(cudaGetLastError());
    note_launch(1);
    return FP4_OK;
  }
  if (batch > 65535) return FP4_ERR_UNSUPPORTED;
  const int64_t per4 = (n * k) / 4;
  FP4_TRY_CUDA(cudaMemsetAsync(tensor_scale, 0, static_cast<size_t>(batch) * sizeof(float), st));
  const int gx = std::max(1, std::min(grid_for(per4, kThreads), std::max(1, num_sms() * 16 / (int)batch)));
  dim3 grid(gx, static_cast<unsigned>(batch));
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(tensor_scale);
  if (w_dtype == FP4_F32) {
    nvfp4_amax_kernel<float><<<grid, kThreads, 0, st>>>(static_cast<const float*>(w), per4, amax_bits);
    nvfp4_pack_kernel<float><<<grid, kThreads, 0, st>>>(static_cast<const float*>(w), per4, amax_bits,
                                                        reinterpret_cast<uint16_t*>(codes), scales);
  } else {
    nvfp4_amax_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(w),
                                                                per4, amax_bits);
    nvfp4_pack_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), per4, amax_bits, reinterpret_cast<uint16_t*>(codes),
        scales);
  }
  nvfp4_finalize_kernel<<<static_cast<unsigned>((batch + 255) / 256), 256, 0, st>>>(tensor_scale, batch);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch(3);
  return FP4_OK;
}

extern "C" fp4_status fp4_unpack(fp4_format fmt, const uint8_t* codes, const uint8_t* scales,
                                 const float* tensor_scale, int64_t batch, int64_t n, int64_t k,
                                 void* out, fp4_dtype out_dtype, void* stream) {
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4) return FP4_ERR_UNSUPPORTED;
  if (out_dtype != FP4_F32 && out_dtype != FP4_BF16) return FP4_ERR_INVALID_ARG;
  int64_t total;
  FP4_TRY(checked_count({batch, n, k}, &total));
  int64_t bytes_out;
  if (!mul_ok(total, 4, &bytes_out)) return FP4_ERR_SHAPE_OVERFLOW;
  const int B = (fmt == FP4_MXFP4) ? 32 : 16;
  if (k % B != 0) return FP4_ERR_ALIGNMENT;
  if (!codes || !scales || !out || (fmt == FP4_NVFP4 && !tensor_scale)) return FP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(out)) return FP4_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = grid_for(total, kThreads);
  const int64_t per = n * k;
  if (fmt == FP4_MXFP4) {
    if (out_dtype == FP4_F32)
      unpack_kernel<FP4_MXFP4, FP4_F32><<<grid, kThreads, 0, st>>>(codes, scales, tensor_scale, per, total, out);
    else
      unpack_kernel<FP4_MXFP4, FP4_BF16><<<grid, kThreads, 0, st>>>(codes, scales, tensor_scale, per, total, out);
  } else {
    if (out_dtype == FP4_F32)
      unpack_kernel<FP4_NVFP4, FP4_F32><<<grid, kThreads, 0, st>>>(codes, scales, tensor_scale, per, total, out);
    else
      unpack_kernel<FP4_NVFP4, FP4_BF16><<<grid, kThreads, 0, st>>>(codes, scales, tensor_scale, per, total, out);
  }
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch(1);
  return FP4_OK;
}

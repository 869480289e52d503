// Device twin of synth/draws.py: counter-based seeded weight draws.
//
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1,
// 2, 3", SC'11) turns (key, counter) into 32-bit words; a Student-t(4) variate comes
// from Bailey's polar method ("Polar generation of random variates with the
// t-distribution", Math. Comp. 62, 1994).  Every float operation is a correctly
// rounded intrinsic in the same order as the host code, so host and device draw the
// same bits.  This file holds input generation only, none of the FP4 method.
#include <cuda_runtime.h>
#include <stdint.h>

#define SYNTH_API extern "C" __attribute__((visibility("default")))

namespace {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__device__ __forceinline__ float signed_uniform(uint32_t r) {
  return static_cast<float>(static_cast<int32_t>(r >> 8) - (1 << 23)) * 0x1p-23f;
}
__device__ __forceinline__ float unit_uniform(uint32_t r) { return static_cast<float>(r >> 8) * 0x1p-24f; }

__device__ __forceinline__ float polar_t4(float u, float w) {
  float s = __fsqrt_rn(w);
  s = __fdiv_rn(1.0f, s);
  s = __fsub_rn(s, 1.0f);
  s = __fmul_rn(s, 4.0f);
  s = __fdiv_rn(s, w);
  s = __fsqrt_rn(s);
  return __fmul_rn(u, s);
}

__global__ void t4_kernel(float* __restrict__ out, int64_t start, int64_t count, uint32_t seed, uint32_t tid,
                          float scale, int with_outliers, float frac, float lo_s, float span_s, float sigma) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t idx = static_cast<uint64_t>(start + i);
    const uint32_t lo = static_cast<uint32_t>(idx), hi = static_cast<uint32_t>(idx >> 32);
    float t = 0.0f;
    bool done = false;
    for (uint32_t attempt = 0; attempt < 8 && !done; ++attempt) {
      const uint4 r = philox4x32_10(make_uint4(lo, hi, attempt, 0u), seed, tid);
      const uint32_t ra[2] = {r.x, r.z}, rb[2] = {r.y, r.w};
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        if (done) break;
        const float u = signed_uniform(ra[p]), v = signed_uniform(rb[p]);
        const float w = __fadd_rn(__fmul_rn(u, u), __fmul_rn(v, v));
        if (w > 0.0f && w <= 1.0f) {
          t = polar_t4(u, w);
          done = true;
        }
      }
    }
    float wv = __fmul_rn(t, scale);
    if (with_outliers) {
      const uint4 r = philox4x32_10(make_uint4(lo, hi, 0xFFFFFFFFu, 0u), seed, tid);
      if (unit_uniform(r.x) < frac) {
        float m = __fmul_rn(span_s, unit_uniform(r.y));
        m = __fadd_rn(lo_s, m);
        m = __fmul_rn(m, sigma);
        wv = (r.z & 1u) ? -m : m;
      }
    }
    out[i] = wv;
  }
}

}  // namespace

// Draws elements [start, start + count) of a flattened weight tensor into out (float32,
// device).  Returns 0 on success, else the cudaError_t of the launch.
SYNTH_API int synth_t4_weights(float* out, int64_t start, int64_t count, uint32_t seed, uint32_t tensor_id,
                               float scale, int with_outliers, float frac, float lo_sigma, float span_sigma,
                               float sigma, void* stream) {
  if (count <= 0) return 0;
  int blocks = static_cast<int>((count + 255) / 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  t4_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, start, count, seed, tensor_id, scale,
                                                                   with_outliers, frac, lo_sigma, span_sigma, sigma);
  return static_cast<int>(cudaGetLastError());
}

// CB4 packing on the GPU: a 16-entry fp16 codebook per 128-weight group of a row plus a
// sparse fp16 outlier term, following "XFP：质量地板驱动的自适应码本量化":
//   * 离群值提取 -- weights with |w - mu| > threshold leave the bulk for the sparse term
//     and their bulk position is back-filled with mu before any codebook is fitted;
//   * Lloyd 迭代 -- a scalar k-means codebook of 16 entries per group, started at the
//     CDF-uniform quantiles (the (i + 0.5)/16 order statistics: sorted position 8i + 4 of
//     128) and refined by 20 rounds of nearest-entry assignment (ties to the lower entry)
//     and member means (an empty entry keeps its value);
//   * V2 dense + sparse -- W = W_codebook + W_outlier, the sparse value being the fp16
//     residual w - entry(idx) at the outlier's position;
//   * 子字节打包 -- 4-bit indices, two per byte, even position in the low nibble.
// All arithmetic is float64; a member mean adds the members in ascending position order
// and divides once, and every fp16 value is one round-to-nearest-even of a float64, so
// the result is a deterministic function of the input weights.
#include <algorithm>

#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr int kGroup = 128, kEntries = 16, kRounds = 20;
constexpr int kWarpsPerCta = 8;

// float64 -> IEEE binary16 bits, round to nearest even, overflow to infinity.
__device__ __forceinline__ uint16_t f64_to_f16_rne(double x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  if (x != x) return 0x7E00u;
  const double a = fabs(x);
  if (a == 0.0) return sign;
  int e = ilogb(a);
  if (e < -14) e = -14;                               // subnormals share the exponent -14
  double q = rint(scalbn(a, 10 - e));                 // exact scaling; ties to even
  if (q >= 2048.0) {                                  // rounded up into the next binade
    q = 1024.0;
    e += 1;
  }
  if (e > 15) return sign | 0x7C00u;
  const uint32_t qi = static_cast<uint32_t>(q);
  if (qi < 1024u) return sign | static_cast<uint16_t>(qi);          // subnormal (e == -14)
  return sign | static_cast<uint16_t>(((e + 15) << 10) | (qi - 1024u));
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t b) {
  return static_cast<double>(__half2float(__ushort_as_half(b)));
}

// four consecutive weights of a row as float64
template <int kDt>
__device__ __forceinline__ void load4(const void* w, int64_t at, double (&v)[4]) {
  if (kDt == FP4_F32) {
    const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(w) + at);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(w) + at);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  }
}
template <int kDt>
__device__ __forceinline__ double load1(const void* w, int64_t at) {
  if (kDt == FP4_F32) return static_cast<const float*>(w)[at];
  return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(w)[at]) << 16);
}

// Outliers per row: one warp per row; counts land in row_ptr[1 + r].
template <int kDt>
__global__ void __launch_bounds__(256) cb4_count_kernel(const void* __restrict__ w, int64_t rows, int64_t K,
                                                        double thr, double mu, int32_t* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    int n = 0;
    for (int64_t c = 4 * lane; c < K; c += 128) {
      double v[4];
      load4<kDt>(w, r * K + c, v);
#pragma unroll
      for (int s = 0; s < 4; ++s) n += fabs(v[s] - mu) > thr;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
    if (lane == 0) row_ptr[1 + r] = n;
  }
}

// In-place inclusive scan of row_ptr[1..rows] (one CTA of 1024 threads); row_ptr[0] = 0.
__global__ void __launch_bounds__(1024) cb4_scan_kernel(int32_t* __restrict__ row_ptr, int64_t rows) {
  __shared__ int32_t part[1024];
  const int tid = threadIdx.x;
  const int64_t per = (rows + 1023) / 1024;
  const int64_t r0 = 1 + tid * per, r1 = (r0 + per < rows + 1) ? r0 + per : rows + 1;
  int32_t s = 0;
  for (int64_t r = r0; r < r1; ++r) s += row_ptr[r];
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int32_t v = (tid >= o) ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int32_t run = part[tid] - s;
  for (int64_t r = r0; r < r1; ++r) {
    run += row_ptr[r];
    row_ptr[r] = run;
  }
  if (tid == 0) row_ptr[0] = 0;
}

// Codebook fit: one warp per 128-weight group; lane l holds positions 4l .. 4l+3.
template <int kDt>
__global__ void __launch_bounds__(kWarpsPerCta * 32) cb4_fit_kernel(const void* __restrict__ w, int64_t rows,
                                                                    int64_t K, double thr, double mu,
                                                                    uint8_t* __restrict__ idx,
                                                                    uint16_t* __restrict__ cb) {
  __shared__ double init[kWarpsPerCta][kEntries];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const int64_t gpr = K / kGroup;
  const int64_t groups = rows * gpr;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
  for (int64_t gi = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + wl; gi < groups; gi += warps) {
    const int64_t r = gi / gpr, gc = gi % gpr;
    double g[4];
    load4<kDt>(w, r * K + gc * kGroup + 4 * lane, g);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (fabs(g[s] - mu) > thr) g[s] = mu;                 // outliers back-filled with mu

    // start: the order statistics at sorted positions 8i + 4 (stable rank)
    int rank[4] = {0, 0, 0, 0};
    for (int j4 = 0; j4 < 32; ++j4) {
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2) {
        const double v = __shfl_sync(0xFFFFFFFFu, g[s2], j4);
        const int pos = 4 * j4 + s2;
#pragma unroll
        for (int s = 0; s < 4; ++s) rank[s] += (v < g[s]) || (v == g[s] && pos < 4 * lane + s);
      }
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if ((rank[s] & 7) == 4) init[wl][rank[s] >> 3] = g[s];
    __syncwarp();
    double c[kEntries];
#pragma unroll
    for (int j = 0; j < kEntries; ++j) c[j] = init[wl][j];

    auto nearest = [&](double v) {
      int best = 0;
      double bd = fabs(v - c[0]);
#pragma unroll
      for (int j = 1; j < kEntries; ++j) {
        const double d = fabs(v - c[j]);
        if (d < bd) { bd = d; best = j; }
      }
      return best;
    };
    for (int round = 0; round < kRounds; ++round) {
      int a[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) a[s] = nearest(g[s]);
      // lane j < 16 forms the mean of entry j: members added in ascending position
      double sum = 0.0;
      int n = 0;
      for (int j4 = 0; j4 < 32; ++j4) {
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) {
          const double v = __shfl_sync(0xFFFFFFFFu, g[s2], j4);
          const int aj = __shfl_sync(0xFFFFFFFFu, a[s2], j4);
          if (aj == lane) { sum += v; ++n; }
        }
      }
      double mine = 0.0;
#pragma unroll
      for (int j = 0; j < kEntries; ++j) mine = (lane == j) ? c[j] : mine;
      const double cnew = (n > 0) ? sum / static_cast<double>(n) : mine;
#pragma unroll
      for (int j = 0; j < kEntries; ++j) c[j] = __shfl_sync(0xFFFFFFFFu, cnew, j);
    }
    // entries to fp16, then every weight to its nearest fp16 entry
    uint16_t bits[kEntries];
#pragma unroll
    for (int j = 0; j < kEntries; ++j) {
      bits[j] = f64_to_f16_rne(c[j]);
      c[j] = f16_bits_to_f64(bits[j]);
    }
    int a[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) a[s] = nearest(g[s]);
    const uint32_t packed = static_cast<uint32_t>(a[0] | (a[1] << 4) | (a[2] << 8) | (a[3] << 12));
    *reinterpret_cast<uint16_t*>(idx + r * (K / 2) + gc * (kGroup / 2) + 2 * lane) = static_cast<uint16_t>(packed);
    uint16_t mine = 0;
#pragma unroll
    for (int j = 0; j < kEntries; ++j) mine = (lane == j) ? bits[j] : mine;
    if (lane < kEntries) cb[gi * kEntries + lane] = mine;
  }
}

// Sparse term: one warp per row, outliers in ascending column order at row_ptr[r]..
template <int kDt>
__global__ void __launch_bounds__(256) cb4_outlier_kernel(const void* __restrict__ w, int64_t rows, int64_t K,
                                                          double thr, double mu, const int32_t* __restrict__ row_ptr,
                                                          const uint8_t* __restrict__ idx,
                                                          const uint16_t* __restrict__ cb, int32_t* __restrict__ col,
                                                          uint16_t* __restrict__ val) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    int32_t at = row_ptr[r];
    for (int64_t c0 = 0; c0 < K; c0 += 32) {
      const int64_t c = c0 + lane;
      const double v = load1<kDt>(w, r * K + c);
      const bool out = fabs(v - mu) > thr;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, out);
      if (out && col != nullptr && val != nullptr) {
        const int pos = at + __popc(bal & ((1u << lane) - 1u));
        const uint32_t byte = idx[r * (K / 2) + (c >> 1)];
        const uint32_t a = (c & 1) ? (byte >> 4) : (byte & 15u);
        const double entry = f16_bits_to_f64(cb[(r * (K / kGroup) + c / kGroup) * kEntries + a]);
        col[pos] = static_cast<int32_t>(c);
        val[pos] = f64_to_f16_rne(v - entry);
      }
      at += __popc(bal);
    }
  }
}

fp4_status check_cb4(const void* w, fp4_dtype dt, int64_t rows, int64_t k, double thr) {
  int64_t n;
  FP4_TRY(checked_count({rows, k}, &n));
  if (n >= (int64_t(1) << 31)) return FP4_ERR_SHAPE_OVERFLOW;
  if (k % kGroup != 0) return FP4_ERR_ALIGNMENT;
  if (dt != FP4_F32 && dt != FP4_BF16) return FP4_ERR_INVALID_ARG;
  if (!(thr >= 0.0) || !std::isfinite(thr)) return FP4_ERR_INVALID_ARG;
  if (w == nullptr) return FP4_ERR_INVALID_ARG;
  if (!aligned16(w)) return FP4_ERR_ALIGNMENT;
  return FP4_OK;
}

int grid_warps(int64_t items, int warps_per_cta) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + warps_per_cta - 1) / warps_per_cta,
                                                                    static_cast<int64_t>(num_sms()) * 16)));
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" fp4_status fp4_cb4_row_ptr(const void* w, fp4_dtype w_dtype, int64_t rows, int64_t k, double threshold,
                                      double mu, int32_t* row_ptr, void* stream) {
  FP4_TRY(check_cb4(w, w_dtype, rows, k, threshold));
  if (!std::isfinite(mu)) return FP4_ERR_INVALID_ARG;
  if (row_ptr == nullptr) return FP4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(row_ptr) & 3u) return FP4_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = grid_warps(rows, 8);
  if (w_dtype == FP4_F32)
    cb4_count_kernel<FP4_F32><<<grid, 256, 0, st>>>(w, rows, k, threshold, mu, row_ptr);
  else
    cb4_count_kernel<FP4_BF16><<<grid, 256, 0, st>>>(w, rows, k, threshold, mu, row_ptr);
  cb4_scan_kernel<<<1, 1024, 0, st>>>(row_ptr, rows);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch(2);
  return FP4_OK;
}

extern "C" fp4_status fp4_pack_cb4(const void* w, fp4_dtype w_dtype, int64_t rows, int64_t k, double threshold,
                                   double mu, const int32_t* row_ptr, uint8_t* idx, uint16_t* cb, int32_t* col,
                                   uint16_t* val, void* stream) {
  FP4_TRY(check_cb4(w, w_dtype, rows, k, threshold));
  if (!std::isfinite(mu)) return FP4_ERR_INVALID_ARG;
  if (!row_ptr || !idx || !cb) return FP4_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(cb) || (reinterpret_cast<uintptr_t>(row_ptr) & 3u)) return FP4_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t groups = rows * (k / kGroup);
  const int gfit = grid_warps(groups, kWarpsPerCta);
  const int grow = grid_warps(rows, 8);
  if (w_dtype == FP4_F32) {
    cb4_fit_kernel<FP4_F32><<<gfit, kWarpsPerCta * 32, 0, st>>>(w, rows, k, threshold, mu, idx, cb);
    cb4_outlier_kernel<FP4_F32><<<grow, 256, 0, st>>>(w, rows, k, threshold, mu, row_ptr, idx, cb, col, val);
  } else {
    cb4_fit_kernel<FP4_BF16><<<gfit, kWarpsPerCta * 32, 0, st>>>(w, rows, k, threshold, mu, idx, cb);
    cb4_outlier_kernel<FP4_BF16><<<grow, 256, 0, st>>>(w, rows, k, threshold, mu, row_ptr, idx, cb, col, val);
  }
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch(2);
  return FP4_OK;
}

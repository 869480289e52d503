// V2a packing on the GPU: codebook-plus-outlier weights whose codebooks come from one
// small shared library per matrix ("XFP：质量地板驱动的自适应码本量化", section V2a：共享
// 码本库, with 离群值提取 and Lloyd 迭代).
//   * outliers (|w - mu| > threshold) leave the bulk, back-filled with mu; they form an
//     fp16 residual CSR exactly as the CB4 packer's (the same row pointers);
//   * each 128-weight group keeps mid = fp16((max + min) / 2) and scale =
//     fp16((max - min) / 2) of its bulk values; z = (w - mid) / scale (0 if scale is 0);
//   * LibFit: a Lloyd codebook of 2^N entries per row over the row's z values (started at
//     the sorted positions floor((2i + 1) K / 2^(N+1)), 20 rounds), then Lloyd over those
//     codebooks as vectors: L = 32 library entries started at the codebooks of span rank
//     floor((2i + 1) R / 64) (span = largest - smallest entry, ties by row), 20 rounds,
//     squared distances summed in entry order; the library rounded to fp16;
//   * a group takes the library codebook with the least sum (in position order) of squared
//     distances to the nearest entry; each weight its nearest entry of that codebook;
//   * reconstruction fp16(mid + scale * entry), one rounding.
// All arithmetic is float64, member means add members in ascending order (positions for
// the row codebooks, rows for the library) and divide once, ties go to the lower index:
// the packed output is a deterministic function of the weights.
//
// Group record (8 bytes per 128 weights): mid fp16 | scale fp16 | library index | 3 zero
// bytes -- 64-bit records keep every per-stage copy of the decode kernels 16-byte aligned.
#include <algorithm>

#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr int kGroup = 128, kLib = 32, kRounds = 20;

__device__ __forceinline__ uint16_t v2a_f64_to_f16(double x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  if (x != x) return 0x7E00u;
  const double a = fabs(x);
  if (a == 0.0) return sign;
  int e = ilogb(a);
  if (e < -14) e = -14;
  double q = rint(scalbn(a, 10 - e));
  if (q >= 2048.0) {
    q = 1024.0;
    e += 1;
  }
  if (e > 15) return sign | 0x7C00u;
  const uint32_t qi = static_cast<uint32_t>(q);
  if (qi < 1024u) return sign | static_cast<uint16_t>(qi);
  return sign | static_cast<uint16_t>(((e + 15) << 10) | (qi - 1024u));
}
__device__ __forceinline__ double f16b(uint16_t b) { return static_cast<double>(__half2float(__ushort_as_half(b))); }

template <int kDt>
__device__ __forceinline__ double ld1(const void* w, int64_t at) {
  if (kDt == FP4_F32) return static_cast<const float*>(w)[at];
  return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(w)[at]) << 16);
}

// bulk value: an outlier position holds mu
__device__ __forceinline__ double bulk(double v, double thr, double mu) { return fabs(v - mu) > thr ? mu : v; }

// z of one weight from its group record
__device__ __forceinline__ double znorm(double b, uint64_t rec) {
  const double mid = f16b(static_cast<uint16_t>(rec & 0xFFFFu));
  const double sc = f16b(static_cast<uint16_t>((rec >> 16) & 0xFFFFu));
  return sc > 0.0 ? (b - mid) / sc : 0.0;
}

// ---- 1. group records (mid, scale): one warp per group --------------------------------
template <int kDt>
__global__ void __launch_bounds__(256) v2a_stats_kernel(const void* __restrict__ w, int64_t rows, int64_t K, double thr,
                                                        double mu, uint64_t* __restrict__ rec) {
  const int lane = threadIdx.x & 31;
  const int64_t gpr = K / kGroup, groups = rows * gpr;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t gi = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; gi < groups; gi += warps) {
    const int64_t base = (gi / gpr) * K + (gi % gpr) * kGroup;
    double lo = INFINITY, hi = -INFINITY;
    for (int s = 0; s < 4; ++s) {
      const double b = bulk(ld1<kDt>(w, base + 4 * lane + s), thr, mu);
      lo = fmin(lo, b);
      hi = fmax(hi, b);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    if (lane == 0) {
      const uint64_t mid = v2a_f64_to_f16((hi + lo) / 2.0), sc = v2a_f64_to_f16((hi - lo) / 2.0);
      rec[gi] = mid | (sc << 16);
    }
  }
}

// ---- 2. per-row Lloyd codebooks: one warp per row, the row's z values in shared memory ----
template <int kDt>
__global__ void __launch_bounds__(128) v2a_rowfit_kernel(const void* __restrict__ w, int64_t rows, int K, int Kp, int n,
                                                         double thr, double mu, const uint64_t* __restrict__ rec,
                                                         double* __restrict__ cbs) {
  extern __shared__ __align__(16) uint8_t v2a_smem[];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5, nw = blockDim.x >> 5;
  double* z = reinterpret_cast<double*>(v2a_smem) + static_cast<int64_t>(wl) * (K + Kp);
  double* srt = z + K;
  uint8_t* asg = v2a_smem + static_cast<size_t>(nw) * (K + Kp) * sizeof(double) + static_cast<size_t>(wl) * K;
  const int64_t gpr = K / kGroup;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * nw + wl; r < rows; r += static_cast<int64_t>(gridDim.x) * nw) {
    for (int p = lane; p < K; p += 32) {
      const double v = znorm(bulk(ld1<kDt>(w, r * K + p), thr, mu), rec[r * gpr + p / kGroup]);
      z[p] = v;
      srt[p] = v;
    }
    for (int p = K + lane; p < Kp; p += 32) srt[p] = INFINITY;
    __syncwarp();
    // bitonic sort of srt[0..Kp)
    for (int size = 2; size <= Kp; size <<= 1)
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = lane; i < Kp / 2; i += 32) {
          const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
          const bool up = (lo & size) == 0;
          const double a = srt[lo], b = srt[hi];
          if ((a > b) == up) {
            srt[lo] = b;
            srt[hi] = a;
          }
        }
        __syncwarp();
      }
    double c[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c[j] = (j < n) ? srt[static_cast<int64_t>(2 * j + 1) * K / (2 * n)] : 0.0;
    __syncwarp();
    for (int round = 0; round < kRounds; ++round) {
      for (int p = lane; p < K; p += 32) {
        const double v = z[p];
        int best = 0;
        double bd = fabs(v - c[0]);
#pragma unroll
        for (int j = 1; j < 16; ++j) {
          if (j >= n) break;
          const double d = fabs(v - c[j]);
          if (d < bd) { bd = d; best = j; }
        }
        asg[p] = static_cast<uint8_t>(best);
      }
      __syncwarp();
      double sum = 0.0;
      int cnt = 0;
      if (lane < n)
        for (int p = 0; p < K; ++p)
          if (asg[p] == lane) { sum += z[p]; ++cnt; }
      double mine = 0.0;
#pragma unroll
      for (int j = 0; j < 16; ++j) mine = (lane == j) ? c[j] : mine;
      const double cnew = (cnt > 0) ? sum / static_cast<double>(cnt) : mine;
#pragma unroll
      for (int j = 0; j < 16; ++j) c[j] = __shfl_sync(0xFFFFFFFFu, cnew, j);
      __syncwarp();
    }
    double mine = 0.0;
#pragma unroll
    for (int j = 0; j < 16; ++j) mine = (lane == j) ? c[j] : mine;
    if (lane < n) cbs[r * n + lane] = mine;
    __syncwarp();
  }
}

// ---- 3. LibFit: one CTA per matrix --------------------------------------------------------
__global__ void __launch_bounds__(256) v2a_libfit_kernel(const double* __restrict__ cbs_all, int R, int Rp, int n,
                                                         uint16_t* __restrict__ lib_out, double* __restrict__ lib_f64) {
  extern __shared__ __align__(16) uint8_t v2a_smem[];
  double* key = reinterpret_cast<double*>(v2a_smem);              // [Rp] span
  int* idx = reinterpret_cast<int*>(key + Rp);                   // [Rp] row
  int16_t* asg = reinterpret_cast<int16_t*>(idx + Rp);           // [R]
  __shared__ double lib[kLib][16];
  const int b = blockIdx.x, tid = threadIdx.x;
  const double* cbs = cbs_all + static_cast<int64_t>(b) * R * n;
  for (int r = tid; r < Rp; r += blockDim.x) {
    if (r < R) {
      double mx = cbs[r * n], mn = cbs[r * n];
      for (int j = 1; j < n; ++j) {
        mx = fmax(mx, cbs[r * n + j]);
        mn = fmin(mn, cbs[r * n + j]);
      }
      key[r] = mx - mn;
    } else {
      key[r] = INFINITY;
    }
    idx[r] = r;
  }
  __syncthreads();
  // bitonic sort by (span, row)
  for (int size = 2; size <= Rp; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < Rp / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const double ka = key[lo], kb = key[hi];
        const int ia = idx[lo], ib = idx[hi];
        const bool gt = (ka > kb) || (ka == kb && ia > ib);
        if (gt == up) {
          key[lo] = kb; key[hi] = ka;
          idx[lo] = ib; idx[hi] = ia;
        }
      }
      __syncthreads();
    }
  for (int t = tid; t < kLib * 16; t += blockDim.x) {
    const int l = t / 16, j = t % 16;
    lib[l][j] = (j < n) ? cbs[static_cast<int64_t>(idx[(2 * l + 1) * R / (2 * kLib)]) * n + j] : 0.0;
  }
  __syncthreads();
  for (int round = 0; round < kRounds; ++round) {
    for (int r = tid; r < R; r += blockDim.x) {
      int best = 0;
      double bd = 0.0;
      for (int l = 0; l < kLib; ++l) {
        double d = 0.0;
        for (int j = 0; j < n; ++j) {
          const double t = cbs[r * n + j] - lib[l][j];
          d += t * t;
        }
        if (l == 0 || d < bd) { bd = d; best = l; }
      }
      asg[r] = static_cast<int16_t>(best);
    }
    __syncthreads();
    if (tid < kLib) {
      double acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = 0.0;
      int cnt = 0;
      for (int r = 0; r < R; ++r)
        if (asg[r] == tid) {
          ++cnt;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < n) acc[j] += cbs[r * n + j];
        }
      if (cnt > 0)
        for (int j = 0; j < n; ++j) lib[tid][j] = acc[j] / static_cast<double>(cnt);
    }
    __syncthreads();
  }
  for (int t = tid; t < kLib * n; t += blockDim.x) {
    const uint16_t h = v2a_f64_to_f16(lib[t / n][t % n]);
    lib_out[static_cast<int64_t>(b) * kLib * n + t] = h;
    lib_f64[static_cast<int64_t>(b) * kLib * n + t] = f16b(h);
  }
}

// ---- 4. group choice and codes: one warp per group ------------------------------------------
template <int kDt>
__global__ void __launch_bounds__(256) v2a_assign_kernel(const void* __restrict__ w, int64_t rows_per_matrix,
                                                         int64_t rows, int64_t K, int n, int n_bits, double thr,
                                                         double mu, const double* __restrict__ lib_f64,
                                                         uint64_t* __restrict__ rec, uint8_t* __restrict__ codes) {
  const int lane = threadIdx.x & 31;
  const int64_t gpr = K / kGroup, groups = rows * gpr;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t gi = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; gi < groups; gi += warps) {
    const int64_t r = gi / gpr, base = r * K + (gi % gpr) * kGroup;
    const uint64_t rc = rec[gi];
    const double* lib = lib_f64 + (r / rows_per_matrix) * kLib * n;
    double zv[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) zv[s] = znorm(bulk(ld1<kDt>(w, base + 4 * lane + s), thr, mu), rc);
    // lane l: error of library codebook l over the group's positions in order
    double err = 0.0;
    for (int p = 0; p < kGroup; ++p) {
      const double v = __shfl_sync(0xFFFFFFFFu, zv[p & 3], p >> 2);
      double dm = INFINITY;
      for (int j = 0; j < n; ++j) {
        const double t = v - lib[lane * n + j];
        dm = fmin(dm, t * t);
      }
      err += dm;
    }
    // least error, ties to the lower index
    double be = err;
    int bl = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
      const int ol = __shfl_xor_sync(0xFFFFFFFFu, bl, o);
      if (oe < be || (oe == be && ol < bl)) { be = oe; bl = ol; }
    }
    uint32_t packed = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      int best = 0;
      double bd = fabs(zv[s] - lib[bl * n]);
      for (int j = 1; j < n; ++j) {
        const double d = fabs(zv[s] - lib[bl * n + j]);
        if (d < bd) { bd = d; best = j; }
      }
      packed |= static_cast<uint32_t>(best) << (n_bits * s);
    }
    if (n_bits == 4)
      *reinterpret_cast<uint16_t*>(codes + base / 2 + 2 * lane) = static_cast<uint16_t>(packed);
    else
      codes[base / 4 + lane] = static_cast<uint8_t>(packed);
    if (lane == 0) rec[gi] = rc | (static_cast<uint64_t>(bl) << 32);
  }
}

__device__ __forceinline__ int v2a_code(const uint8_t* codes, int64_t at, int n_bits) {
  return n_bits == 4 ? (codes[at >> 1] >> (4 * (at & 1))) & 15 : (codes[at >> 2] >> (2 * (at & 3))) & 3;
}

// fp16 reconstruction of one weight (exact float64 arithmetic, one rounding)
__device__ __forceinline__ uint16_t v2a_recon(uint64_t rc, const uint16_t* lib_bits, int n, int code) {
  const double mid = f16b(static_cast<uint16_t>(rc & 0xFFFFu));
  const double sc = f16b(static_cast<uint16_t>((rc >> 16) & 0xFFFFu));
  const int l = static_cast<int>((rc >> 32) & 31u);
  return v2a_f64_to_f16(mid + sc * f16b(lib_bits[l * n + code]));
}

// ---- 5. outlier residuals: one warp per row, ascending columns -------------------------------
template <int kDt>
__global__ void __launch_bounds__(256) v2a_outlier_kernel(const void* __restrict__ w, int64_t rows_per_matrix,
                                                          int64_t rows, int64_t K, int n, int n_bits, double thr,
                                                          double mu, const int32_t* __restrict__ row_ptr,
                                                          const uint8_t* __restrict__ codes,
                                                          const uint64_t* __restrict__ rec,
                                                          const uint16_t* __restrict__ lib,
                                                          int32_t* __restrict__ col, uint16_t* __restrict__ val) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    int32_t at = row_ptr[r];
    const uint16_t* lb = lib + (r / rows_per_matrix) * kLib * n;
    for (int64_t c0 = 0; c0 < K; c0 += 32) {
      const int64_t c = c0 + lane;
      const double v = ld1<kDt>(w, r * K + c);
      const bool out = fabs(v - mu) > thr;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, out);
      if (out) {
        const int slot = at + __popc(m & ((1u << lane) - 1u));
        const uint16_t hat = v2a_recon(rec[r * (K / kGroup) + c / kGroup], lb, n, v2a_code(codes, r * K + c, n_bits));
        col[slot] = static_cast<int32_t>(c);
        val[slot] = v2a_f64_to_f16(v - f16b(hat));
      }
      at += __popc(m);
    }
  }
}

// ---- dense term as float32 (exact fp16 values): one thread per weight -----------------------
__global__ void __launch_bounds__(256) v2a_unpack_kernel(const uint8_t* __restrict__ codes,
                                                         const uint64_t* __restrict__ rec,
                                                         const uint16_t* __restrict__ lib, int64_t rows_per_matrix,
                                                         int64_t rows, int64_t K, int n, int n_bits,
                                                         float* __restrict__ out) {
  const int64_t total = rows * K;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / K, c = i % K;
    const uint16_t h = v2a_recon(rec[r * (K / kGroup) + c / kGroup], lib + (r / rows_per_matrix) * kLib * n, n,
                                 v2a_code(codes, i, n_bits));
    out[i] = __half2float(__ushort_as_half(h));
  }
}

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

struct V2aWs {
  size_t cbs, lib, total;
};
V2aWs v2a_ws(int64_t batch, int64_t rows, int n) {
  V2aWs L;
  L.cbs = 0;
  L.lib = align_up(sizeof(double) * batch * rows * n, 256);
  L.total = L.lib + align_up(sizeof(double) * batch * kLib * n, 256);
  return L;
}

fp4_status check_v2a(int64_t batch, int64_t rows, int64_t k, int32_t n_bits) {
  int64_t cnt;
  FP4_TRY(checked_count({batch, rows, k}, &cnt));
  if (n_bits != 2 && n_bits != 4) return FP4_ERR_INVALID_ARG;
  if (k % kGroup != 0) return FP4_ERR_ALIGNMENT;
  if (cnt >= (int64_t(1) << 31)) return FP4_ERR_SHAPE_OVERFLOW;
  if (rows < kLib || k > 4096 || rows > 8192) return FP4_ERR_UNSUPPORTED;
  return FP4_OK;
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" size_t fp4_pack_v2a_workspace_size(int64_t batch, int64_t rows, int64_t k, int32_t n_bits) {
  if (check_v2a(batch, rows, k, n_bits) != FP4_OK) return 0;
  return v2a_ws(batch, rows, 1 << n_bits).total;
}

extern "C" fp4_status fp4_pack_v2a(const void* w, fp4_dtype w_dtype, int64_t batch, int64_t rows, int64_t k,
                                   int32_t n_bits, double threshold, double mu, const int32_t* row_ptr,
                                   uint8_t* codes, uint64_t* groups, uint16_t* lib, int32_t* col, uint16_t* val,
                                   void* workspace, size_t ws_bytes, void* stream) {
  FP4_TRY(check_v2a(batch, rows, k, n_bits));
  if (w_dtype != FP4_F32 && w_dtype != FP4_BF16) return FP4_ERR_INVALID_ARG;
  if (!(threshold >= 0.0) || !std::isfinite(threshold) || !std::isfinite(mu)) return FP4_ERR_INVALID_ARG;
  if (!w || !row_ptr || !codes || !groups || !lib) return FP4_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(groups) || !aligned16(lib)) return FP4_ERR_ALIGNMENT;
  const int n = 1 << n_bits;
  const V2aWs L = v2a_ws(batch, rows, n);
  if (workspace == nullptr || ws_bytes < L.total) return FP4_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP4_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* cbs = reinterpret_cast<double*>(ws + L.cbs);
  double* lib64 = reinterpret_cast<double*>(ws + L.lib);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t R = batch * rows;
  const int64_t groups_n = R * (k / kGroup);
  const int sms = num_sms();
  const int ggrid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((groups_n + 7) / 8, sms * 32)));
  const int rgrid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((R + 7) / 8, sms * 32)));
  const bool f32 = w_dtype == FP4_F32;
  // 1. group records
  if (f32) v2a_stats_kernel<FP4_F32><<<ggrid, 256, 0, st>>>(w, R, k, threshold, mu, groups);
  else v2a_stats_kernel<FP4_BF16><<<ggrid, 256, 0, st>>>(w, R, k, threshold, mu, groups);
  FP4_TRY_CUDA(cudaGetLastError());
  // 2. row codebooks
  const int K = static_cast<int>(k), Kp = next_pow2(K);
  const size_t per_warp = static_cast<size_t>(K + Kp) * sizeof(double) + K;
  const int nw = static_cast<int>(std::max<size_t>(1, std::min<size_t>(4, (96 * 1024) / per_warp)));
  const size_t smem2 = per_warp * nw;
  auto rowfit = f32 ? v2a_rowfit_kernel<FP4_F32> : v2a_rowfit_kernel<FP4_BF16>;
  FP4_TRY_CUDA(cudaFuncSetAttribute(rowfit, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem2)));
  const int fgrid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((R + nw - 1) / nw, sms * 8)));
  rowfit<<<fgrid, 32 * nw, smem2, st>>>(w, R, K, Kp, n, threshold, mu, groups, cbs);
  FP4_TRY_CUDA(cudaGetLastError());
  // 3. library per matrix
  const int Rm = static_cast<int>(rows), Rp = next_pow2(Rm);
  const size_t smem3 = static_cast<size_t>(Rp) * (sizeof(double) + sizeof(int)) + sizeof(int16_t) * Rm;
  FP4_TRY_CUDA(cudaFuncSetAttribute(v2a_libfit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem3)));
  v2a_libfit_kernel<<<static_cast<int>(batch), 256, smem3, st>>>(cbs, Rm, Rp, n, lib, lib64);
  FP4_TRY_CUDA(cudaGetLastError());
  // 4. library index and codes
  if (f32)
    v2a_assign_kernel<FP4_F32><<<ggrid, 256, 0, st>>>(w, rows, R, k, n, n_bits, threshold, mu, lib64, groups, codes);
  else
    v2a_assign_kernel<FP4_BF16><<<ggrid, 256, 0, st>>>(w, rows, R, k, n, n_bits, threshold, mu, lib64, groups, codes);
  FP4_TRY_CUDA(cudaGetLastError());
  // 5. outlier residuals
  if (col != nullptr && val != nullptr) {
    if (f32)
      v2a_outlier_kernel<FP4_F32><<<rgrid, 256, 0, st>>>(w, rows, R, k, n, n_bits, threshold, mu, row_ptr, codes,
                                                          groups, lib, col, val);
    else
      v2a_outlier_kernel<FP4_BF16><<<rgrid, 256, 0, st>>>(w, rows, R, k, n, n_bits, threshold, mu, row_ptr, codes,
                                                           groups, lib, col, val);
    FP4_TRY_CUDA(cudaGetLastError());
  }
  note_launch(col != nullptr && val != nullptr ? 5 : 4);
  return FP4_OK;
}

extern "C" fp4_status fp4_unpack_v2a(const uint8_t* codes, const uint64_t* groups, const uint16_t* lib,
                                     int64_t batch, int64_t rows, int64_t k, int32_t n_bits, float* out,
                                     void* stream) {
  int64_t cnt;
  FP4_TRY(checked_count({batch, rows, k}, &cnt));
  if (n_bits != 2 && n_bits != 4) return FP4_ERR_INVALID_ARG;
  if (k % kGroup != 0) return FP4_ERR_ALIGNMENT;
  if (!codes || !groups || !lib || !out) return FP4_ERR_INVALID_ARG;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((cnt + 255) / 256, num_sms() * 16)));
  v2a_unpack_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(codes, groups, lib, rows, batch * rows, k,
                                                                         1 << n_bits, n_bits, out);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch();
  return FP4_OK;
}

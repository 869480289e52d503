// Experts kept in bf16 inside a mixed-format fused expert buffer.
//
// "The gate that missed by 0.0202 pp", section "A fused tensor with two dtypes in it":
// a fused MoE buffer packs every expert of a layer into one tensor, and an expert
// excluded from quantisation keeps its full-width bf16 rows beside the half-width packed
// 4-bit experts, so each expert carries its own format and offset.  The 4-bit experts of
// such a buffer run on the grouped GEMV (its units skip the other format); this kernel
// runs the bf16 ones with the same units {expert, 64-row tile, <= 8 routed tokens} and
// the same epilogues (SwiGLU with its clamp into f16 h, or the gate-weighted fp32 output
// in slot order), so the combine sums both kinds alike.
//
// One CTA per unit at a time (8 warps, 8 rows each): a warp streams four of its rows' bf16
// weights at a time, 16 bytes per lane and two K chunks ahead (eight loads in flight per
// lane), and multiplies them with the unit's f16 activation rows in fp32; the lanes'
// partial sums meet in a fixed butterfly order (deterministic).
#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr int kD16Tok = 8;
constexpr int kD16Rows = 64;
constexpr int kD16Threads = 256;
constexpr int kD16MaxE = 1024;

__device__ __forceinline__ bool d16_mine(const Dense16Args& a, int e) {
  return e >= a.e_begin && e < a.e_end && a.ex_fmt[e - a.e_begin] == FP4_DENSE_BF16;
}

template <int kEpi>
__global__ void __launch_bounds__(kD16Threads, 1) dense16_kernel(const Dense16Args a) {
  __shared__ int cnt[kD16MaxE + 1], off[kD16MaxE + 1], pre[kD16MaxE + 1];
  __shared__ float red[kD16Rows][kD16Tok];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E;
  const int tiles = (kEpi == kEpiSwiglu) ? a.inter / 32 : a.rows_per_expert / kD16Rows;
  pdl_wait();
  for (int e = threadIdx.x; e < E; e += kD16Threads) cnt[e] = a.counts[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    int sc = 0, su = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = sc;
      pre[e] = su;
      sc += cnt[e];
      su += d16_mine(a, e) ? (cnt[e] + kD16Tok - 1) / kD16Tok * tiles : 0;
    }
    off[E] = sc;
    pre[E] = su;
  }
  __syncthreads();
  const int n_units = pre[E];
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    int lo = 0, hi = E - 1;                      // largest e with pre[e] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int e = lo, n = cnt[e];
    const int groups = (n + kD16Tok - 1) / kD16Tok;
    const int local = u - pre[e];
    const int tile = local / groups, grp = local - tile * groups;
    const int slot0 = off[e] + grp * kD16Tok, ntok = min(kD16Tok, n - grp * kD16Tok);
    const uint8_t* wbase = a.weights + a.offset[e - a.e_begin];
    int64_t xr[kD16Tok];                         // activation row of each token of the unit
#pragma unroll
    for (int i = 0; i < kD16Tok; ++i) {
      const int slot = slot0 + min(i, ntok - 1);
      xr[i] = (kEpi == kEpiSwiglu) ? a.perm[slot] / a.topk : slot;
    }
    // a warp's 8 rows in two groups of four; each step keeps 2 K chunks x 4 rows of weights
    // (eight 16-byte loads per lane) in flight
    for (int rg = 0; rg < 2; ++rg) {
      const uint16_t* wrow[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = warp * (kD16Rows / 8) + rg * 4 + q;   // row of the unit
        const int64_t row = (kEpi == kEpiSwiglu) ? (r < 32 ? tile * 32 + r : a.inter + tile * 32 + (r - 32))
                                                 : static_cast<int64_t>(tile) * kD16Rows + r;
        wrow[q] = reinterpret_cast<const uint16_t*>(wbase) + row * a.K;
      }
      float acc[4][kD16Tok];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kD16Tok; ++i) acc[q][i] = 0.f;
      for (int k0 = lane * 8; k0 < a.K; k0 += 512) {
        uint4 wv[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            wv[u][q] = (k0 + 256 * u < a.K) ? *reinterpret_cast<const uint4*>(wrow[q] + k0 + 256 * u)
                                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int k = k0 + 256 * u;
          if (k >= a.K) break;
#pragma unroll
          for (int i = 0; i < kD16Tok; ++i) {
            if (i >= ntok) break;
            const uint4 xv = *reinterpret_cast<const uint4*>(a.x16 + xr[i] * a.K + k);
            const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
            float xf[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xx[j]));
              xf[2 * j] = f.x;
              xf[2 * j + 1] = f.y;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t ww[4] = {wv[u][q].x, wv[u][q].y, wv[u][q].z, wv[u][q].w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                acc[q][i] = fmaf(__uint_as_float(ww[j] << 16), xf[2 * j], acc[q][i]);
                acc[q][i] = fmaf(__uint_as_float(ww[j] & 0xFFFF0000u), xf[2 * j + 1], acc[q][i]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kD16Tok; ++i) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[q][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[q][i], o);
        }
      if (lane == 0)
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int i = 0; i < kD16Tok; ++i) red[warp * (kD16Rows / 8) + rg * 4 + q][i] = acc[q][i];
    }
    __syncthreads();
    if (kEpi == kEpiSwiglu) {
      for (int idx = threadIdx.x; idx < 32 * ntok; idx += kD16Threads) {
        const int r = idx & 31, i = idx >> 5;
        const float sc = ldexpf(1.0f, a.sexp[a.perm[slot0 + i] / a.topk]);
        const float g = fminf(red[r][i] * sc, a.limit);
        const float uu = fminf(fmaxf(red[32 + r][i] * sc, -a.limit), a.limit);
        a.h_out[static_cast<int64_t>(slot0 + i) * a.inter + tile * 32 + r] = __float2half_rn(g / (1.0f + expf(-g)) * uu);
      }
    } else {
      for (int idx = threadIdx.x; idx < kD16Rows * ntok; idx += kD16Threads) {
        const int r = idx & 63, i = idx >> 6;
        a.o_out[static_cast<int64_t>(slot0 + i) * a.ldo + tile * kD16Rows + r] = red[r][i] * a.gw[a.perm[slot0 + i]];
      }
    }
    __syncthreads();
  }
  pdl_launch_dependents();
}

}  // namespace

fp4_status launch_dense16(const Dense16Args& a, cudaStream_t st) {
  if (a.E > kD16MaxE || a.K % 256 != 0) return FP4_ERR_UNSUPPORTED;
  const int grid = num_sms() * 4;
  if (a.epi == kEpiSwiglu) return launch_pdl(dense16_kernel<kEpiSwiglu>, dim3(grid), dim3(kD16Threads), 0, st, true, a);
  return launch_pdl(dense16_kernel<kEpiDown>, dim3(grid), dim3(kD16Threads), 0, st, true, a);
}

}  // namespace fp4

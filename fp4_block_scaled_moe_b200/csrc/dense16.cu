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
// One CTA per unit at a time, two per SM (8 warps, 8 rows each): every lane streams its
// share of the warp's rows through a ring of 16-byte asynchronous copies into shared memory
// (16 in flight per lane, 64 KB per CTA; a lane reads back only its own copies, so no
// barrier guards the ring), the unit's f16 activation rows sit in shared memory, and the
// products accumulate in fp32 in chunk order; the lanes' partial sums meet in a fixed
// butterfly order (deterministic).
#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr int kD16Tok = 8;
constexpr int kD16Rows = 64;
constexpr int kD16Threads = 256;
constexpr int kD16MaxE = 1024;
constexpr int kD16Depth = 16;             // 16-byte weight items in flight per lane

__device__ __forceinline__ bool d16_mine(const Dense16Args& a, int e) {
  return e >= a.e_begin && e < a.e_end && a.ex_fmt[e - a.e_begin] == FP4_DENSE_BF16;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// shared memory: the unit's activation rows [kD16Tok][K] f16, then the weight ring
// [kD16Depth][kD16Threads] of 16-byte items (each lane reads back only what it copied)
size_t d16_smem_bytes(int K) {
  return static_cast<size_t>(kD16Tok) * K * 2 + static_cast<size_t>(kD16Depth) * kD16Threads * 16;
}

template <int kEpi>
__global__ void __launch_bounds__(kD16Threads, 2) dense16_kernel(const Dense16Args a) {
  extern __shared__ __align__(16) uint8_t d16_smem[];
  __shared__ int cnt[kD16MaxE + 1], off[kD16MaxE + 1], pre[kD16MaxE + 1];
  __shared__ float red[kD16Rows][kD16Tok];
  __half* xs = reinterpret_cast<__half*>(d16_smem);
  uint4* ring = reinterpret_cast<uint4*>(d16_smem + static_cast<size_t>(kD16Tok) * a.K * 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, K = a.K;
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
  const int nck = K / 256;                      // 256-element chunks per row
  const int n_items = 8 * nck;                  // this lane's 16-byte weight items per unit
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
    // the warp's 8 rows
    const uint16_t* wrow[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = warp * 8 + q;                // row of the unit
      const int64_t row = (kEpi == kEpiSwiglu) ? (r < 32 ? tile * 32 + r : a.inter + tile * 32 + (r - 32))
                                               : static_cast<int64_t>(tile) * kD16Rows + r;
      wrow[q] = reinterpret_cast<const uint16_t*>(wbase) + row * K;
    }
    // item m of this lane: chunk m / 8 of row m % 8, 8 elements at 256 (m / 8) + 8 lane
    auto issue = [&](int m) {
      if (m < n_items)
        cp_async16(&ring[(m % kD16Depth) * kD16Threads + threadIdx.x], wrow[m & 7] + 256 * (m >> 3) + 8 * lane);
      cp_async_commit();                         // (an empty group past the end keeps the count)
    };
#pragma unroll
    for (int m = 0; m < kD16Depth; ++m) issue(m);
    // the unit's activation rows into shared memory (while the weights are on their way)
    for (int idx = threadIdx.x; idx < ntok * (K / 8); idx += kD16Threads) {
      const int i = idx / (K / 8), c8 = idx - i * (K / 8);
      const int slot = slot0 + i;
      const int64_t xr = (kEpi == kEpiSwiglu) ? a.perm[slot] / a.topk : slot;
      *reinterpret_cast<uint4*>(xs + static_cast<int64_t>(i) * K + 8 * c8) =
          *reinterpret_cast<const uint4*>(a.x16 + xr * K + 8 * c8);
    }
    __syncthreads();
    float acc[8][kD16Tok];
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int i = 0; i < kD16Tok; ++i) acc[q][i] = 0.f;
    for (int c = 0; c < nck; ++c) {
      uint4 xv[kD16Tok];
#pragma unroll
      for (int i = 0; i < kD16Tok; ++i)
        xv[i] = (i < ntok) ? *reinterpret_cast<const uint4*>(xs + static_cast<int64_t>(i) * K + 256 * c + 8 * lane)
                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int m = 8 * c + q;
        cp_async_wait<kD16Depth - 1>();          // item m has landed (groups complete in order)
        const uint4 wv = ring[(m % kD16Depth) * kD16Threads + threadIdx.x];
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < kD16Tok; ++i) {
          if (i >= ntok) break;
          const uint32_t xx[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&xx[j]));
            acc[q][i] = fmaf(__uint_as_float(ww[j] << 16), xf.x, acc[q][i]);
            acc[q][i] = fmaf(__uint_as_float(ww[j] & 0xFFFF0000u), xf.y, acc[q][i]);
          }
        }
        issue(m + kD16Depth);                    // refill the slot just consumed
      }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int i = 0; i < kD16Tok; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[q][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[q][i], o);
      }
    if (lane == 0)
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int i = 0; i < kD16Tok; ++i) red[warp * 8 + q][i] = acc[q][i];
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
  const size_t smem = d16_smem_bytes(a.K);
  if (smem > 190 * 1024) return FP4_ERR_UNSUPPORTED;
  auto k_gu = dense16_kernel<kEpiSwiglu>;
  auto k_dn = dense16_kernel<kEpiDown>;
  static thread_local size_t configured = 0;
  if (configured < smem) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(k_gu, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    FP4_TRY_CUDA(cudaFuncSetAttribute(k_dn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    configured = smem;
  }
  const int grid = num_sms() * 2;
  if (a.epi == kEpiSwiglu) return launch_pdl(k_gu, dim3(grid), dim3(kD16Threads), smem, st, true, a);
  return launch_pdl(k_dn, dim3(grid), dim3(kD16Threads), smem, st, true, a);
}

}  // namespace fp4

// Grouped W4A16 GEMV for the decode path: few tokens per expert, so the layer is
// bound by the weight stream from HBM.
//
// Design (B200): a persistent CTA per SM walks a list of work units {expert, 64-row
// weight tile, up to 16 routed tokens}.  One producer warp streams each unit's 4-bit
// codes with TMA (128-byte swizzled boxes, conflict-free for the fragment reads), its
// scale bytes with 4-byte async copies, and the f16 activation rows with 1D bulk copies
// into a multi-stage shared-memory ring guarded by mbarriers.  Eight consumer warps
// dequantise in registers (E2M1 pairs -> f16x2 with the sm_100 conversion instruction;
// NVFP4 E4M3 block scales folded in f16, exact; MXFP4 power-of-two scales applied per
// 32-block in fp32) and accumulate with warp-level f16 MMAs into fp32.  The two K
// halves meet in shared memory and a fused epilogue writes: the SwiGLU-with-clamp
// activation h (gate_up), the gate-weighted expert output (down), or y (dense layer).
//
// The per-element unpack-and-scale cost is the overhead the MXFP4 campaign measured
// ("The gate that missed by 0.0202 pp", section "Serving throughput": a constant loss
// paid once per weight element per step); here it runs in registers beside the stream.
#include <algorithm>

#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr int kRows = 64;                 // weight rows per unit
constexpr int kTok = 16;                  // tokens per unit
constexpr int kConsumers = 8;             // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kMaxStages = 4;
constexpr int kOutPitch = kTok + 1;       // fp32 staging row pitch (bank spread)

struct Layout {
  int kc;            // K elements per stage
  int nchunks;       // K / kc
  int scale_row;     // scale bytes per row per stage
  int codes_off, scales_off, x_off;
  int x_row;         // bytes per token row in the stage (padded)
  int stage_bytes;
  int stages;
  int out_off;       // fp32 staging for the K-half reduction
  int bar_off;
  int smem_bytes;
};

__device__ __forceinline__ void named_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

struct Unit {
  int e, tile, slot0, ntok;
};

__device__ __forceinline__ Unit load_unit(const DecodeArgs& a, int u) {
  Unit un;
  if (a.units != nullptr) {
    const int4 v = a.units[u];
    un.e = v.x; un.tile = v.y; un.slot0 = v.z; un.ntok = v.w;
  } else {
    un.e = 0;
    un.tile = u % a.static_tiles;
    un.slot0 = (u / a.static_tiles) * kTok;
    un.ntok = min(kTok, a.static_T - un.slot0);
  }
  return un;
}

// global weight row of unit row r (0..63)
template <int kEpi>
__device__ __forceinline__ int64_t unit_row(const DecodeArgs& a, const Unit& un, int r) {
  const int64_t base = static_cast<int64_t>(un.e) * a.rows_per_expert;
  if (kEpi == kEpiSwiglu)
    return base + (r < 32 ? un.tile * 32 + r : a.inter + un.tile * 32 + (r - 32));
  return base + static_cast<int64_t>(un.tile) * kRows + r;
}

// activation row feeding unit token i
template <int kEpi>
__device__ __forceinline__ int x_row_of(const DecodeArgs& a, const Unit& un, int i) {
  if (kEpi == kEpiSwiglu) return a.perm[un.slot0 + i] / a.topk;
  return un.slot0 + i;
}

template <int kFmt, int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a, const Layout L) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 128-byte swizzled TMA boxes need 1024-byte aligned destinations
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bar_full = sbase + L.bar_off;                 // [stages] x 8 bytes
  const uint32_t bar_empty = bar_full + 8 * kMaxStages;
  constexpr int B = (kFmt == FP4_MXFP4) ? 32 : 16;

  __shared__ unsigned int exit_count;
  if (threadIdx.x == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kConsumers);
    }
    fence_barrier_init();
    exit_count = 0u;
  }
  if (warp == kConsumers && lane == 0) prefetch_tmap(&tmap);
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) slot_begin(a.slot);
  // the last warp of the CTA to leave records the CTA's end time
  auto finish = [&]() {
    if (lane == 0 && atomicAdd(&exit_count, 1u) == kConsumers) slot_end(a.slot);
  };

  const int n_units = (a.n_units != nullptr) ? *a.n_units
                                             : a.static_tiles * ((a.static_T + kTok - 1) / kTok);
  const int ncb = L.kc / 256;                                  // 128-byte code boxes per row per stage

  if (warp == kConsumers) {
    // ------------------------------- producer -------------------------------------
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = load_unit(a, u);
      const int64_t y0 = unit_row<kEpi>(a, un, 0), y1 = unit_row<kEpi>(a, un, 32);
      const int xr = (lane < un.ntok) ? x_row_of<kEpi>(a, un, lane) : 0;
      const uint32_t tx = static_cast<uint32_t>(kRows * (L.kc / 2) + un.ntok * L.kc * 2);
      const int words = L.scale_row / 4;
      for (int c = 0; c < L.nchunks; ++c, ++it) {
        const int s = it % L.stages;
        if (it >= L.stages && !mbar_wait(bar_empty + 8 * s, ((it / L.stages) & 1) ^ 1, a.status)) {
          ok = false;
          break;
        }
        const uint32_t st_base = sbase + s * L.stage_bytes;
        const int k0 = c * L.kc;
        // scale bytes: 64 rows x scale_row, 4-byte async copies
        for (int w = lane; w < kRows * words; w += 32) {
          const int r = w / words, cw = w % words;
          const uint8_t* src = a.scales + unit_row<kEpi>(a, un, r) * (a.K / B) + k0 / B + cw * 4;
          cp_async4(st_base + L.scales_off + r * L.scale_row + cw * 4, src);
        }
        cp_async_arrive(bar_full + 8 * s);
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, tx);
        __syncwarp();
        for (int q = lane; q < 2 * ncb; q += 32) {
          const int rb = q & 1, cb = q >> 1;
          tma_load_2d(st_base + L.codes_off + (cb * kRows + rb * 32) * 128, &tmap, k0 / 2 + cb * 128,
                      static_cast<int32_t>(rb ? y1 : y0), bar_full + 8 * s);
        }
        if (lane < un.ntok)
          bulk_g2s(st_base + L.x_off + lane * L.x_row, a.x16 + static_cast<int64_t>(xr) * a.K + k0,
                   static_cast<uint32_t>(L.kc * 2), bar_full + 8 * s);
      }
    }
    // drain: never leave while copies into this CTA's shared memory are in flight
    for (int d = 1; d <= L.stages && d <= it; ++d) {
      const int j = it - d;
      mbar_wait(bar_full + 8 * (j % L.stages), (j / L.stages) & 1, a.status);
    }
    finish();
    return;
  }

  // --------------------------------- consumers --------------------------------------
  const int rg = warp & 3, kh = warp >> 2;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = rg * 16 + g, r1 = r0 + 8;
  float* outs = reinterpret_cast<float*>(smem + L.out_off);
  const int nreg = L.kc / 32;                                  // 32-K regions per stage
  const int j0 = kh * (nreg / 2), j1 = j0 + nreg / 2;
  int it = 0;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const Unit un = load_unit(a, u);
    const int ntiles = un.ntok > 8 ? 2 : 1;
    float acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
    for (int c = 0; c < L.nchunks; ++c, ++it) {
      const int s = it % L.stages;
      if (!mbar_wait(bar_full + 8 * s, (it / L.stages) & 1, a.status)) {
        finish();
        return;
      }
      const uint32_t st_base = sbase + s * L.stage_bytes;
      const uint32_t cbase = st_base + L.codes_off;
      const uint32_t sc_r0 = st_base + L.scales_off + r0 * L.scale_row;
      const uint32_t sc_r1 = st_base + L.scales_off + r1 * L.scale_row;
      const uint32_t xbase = st_base + L.x_off + g * L.x_row + t * 16;
      for (int j = j0; j < j1; ++j) {
        const uint32_t box = cbase + ((j >> 3) * kRows) * 128;
        const uint32_t w0 = lds32(box + r0 * 128 + (((j & 7) ^ (r0 & 7)) << 4) + 4 * t);
        const uint32_t w1 = lds32(box + r1 * 128 + (((j & 7) ^ (r1 & 7)) << 4) + 4 * t);
        uint32_t p0[4], p1[4];   // f16x2 of row r0 / r1: bytes 0..3 of the word
        e2m1x8_to_f16x8(w0, p0[0], p0[1], p0[2], p0[3]);
        e2m1x8_to_f16x8(w1, p1[0], p1[1], p1[2], p1[3]);
        if (kFmt == FP4_NVFP4) {
          // this thread's 8 K positions all lie in block 2j + (t >> 1)
          const int blk = 2 * j + (t >> 1);
          const uint32_t s01 = e4m3x2_to_f16x2(lds8(sc_r0 + blk) | (lds8(sc_r1 + blk) << 8));
          const uint32_t s0 = __byte_perm(s01, 0, 0x1010), s1 = __byte_perm(s01, 0, 0x3232);
#pragma unroll
          for (int q = 0; q < 4; ++q) { p0[q] = hmul2(p0[q], s0); p1[q] = hmul2(p1[q], s1); }
#pragma unroll
          for (int tl = 0; tl < 2; ++tl) {
            if (tl < ntiles) {
              const uint4 xq = lds128(xbase + tl * 8 * L.x_row + j * 64);
              mma_16816(acc[tl], p0[0], p1[0], p0[1], p1[1], xq.x, xq.y);
              mma_16816(acc[tl], p0[2], p1[2], p0[3], p1[3], xq.z, xq.w);
            }
          }
        } else {
          const float f0 = ue8m0_to_f32(lds8(sc_r0 + j)), f1 = ue8m0_to_f32(lds8(sc_r1 + j));
#pragma unroll
          for (int tl = 0; tl < 2; ++tl) {
            if (tl < ntiles) {
              const uint4 xq = lds128(xbase + tl * 8 * L.x_row + j * 64);
              float part[4] = {0.f, 0.f, 0.f, 0.f};
              mma_16816(part, p0[0], p1[0], p0[1], p1[1], xq.x, xq.y);
              mma_16816(part, p0[2], p1[2], p0[3], p1[3], xq.z, xq.w);
              acc[tl][0] = fmaf(f0, part[0], acc[tl][0]);
              acc[tl][1] = fmaf(f0, part[1], acc[tl][1]);
              acc[tl][2] = fmaf(f1, part[2], acc[tl][2]);
              acc[tl][3] = fmaf(f1, part[3], acc[tl][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }
    // ---- K halves meet in shared memory ----
    named_bar_sync();
    if (kh == 1) {
#pragma unroll
      for (int tl = 0; tl < 2; ++tl) {
        const int n = tl * 8 + 2 * t;
        outs[r0 * kOutPitch + n] = acc[tl][0];
        outs[r0 * kOutPitch + n + 1] = acc[tl][1];
        outs[r1 * kOutPitch + n] = acc[tl][2];
        outs[r1 * kOutPitch + n + 1] = acc[tl][3];
      }
    }
    named_bar_sync();
    if (kh == 0) {
#pragma unroll
      for (int tl = 0; tl < 2; ++tl) {
        const int n = tl * 8 + 2 * t;
        outs[r0 * kOutPitch + n] += acc[tl][0];
        outs[r0 * kOutPitch + n + 1] += acc[tl][1];
        outs[r1 * kOutPitch + n] += acc[tl][2];
        outs[r1 * kOutPitch + n + 1] += acc[tl][3];
      }
    }
    named_bar_sync();
    // ---- fused epilogue ----
    const float ts = (kFmt == FP4_NVFP4) ? a.tscale[un.e] : 1.0f;
    if (kEpi == kEpiSwiglu) {
      for (int idx = threadIdx.x; idx < 32 * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 31, i = idx >> 5;
        const int tok = a.perm[un.slot0 + i] / a.topk;
        const float sc = ldexpf(ts, a.sexp[tok]);
        const float gv = fminf(outs[r * kOutPitch + i] * sc, a.limit);
        const float uv = fminf(fmaxf(outs[(32 + r) * kOutPitch + i] * sc, -a.limit), a.limit);
        const float hv = gv / (1.0f + expf(-gv)) * uv;
        a.h_out[static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * 32 + r] = __float2half_rn(hv);
      }
    } else if (kEpi == kEpiDown) {
      for (int idx = threadIdx.x; idx < kRows * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 63, i = idx >> 6;
        const float wgt = a.gw[a.perm[un.slot0 + i]];
        a.o_out[static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * kRows + r] =
            outs[r * kOutPitch + i] * ts * wgt;
      }
    } else {
      for (int idx = threadIdx.x; idx < kRows * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 63, i = idx >> 6;
        const float v = ldexpf(outs[r * kOutPitch + i] * ts, a.sexp[un.slot0 + i]);
        a.y_out[static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * kRows + r] =
            __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
  }
  finish();
}

Layout make_layout(int fmt, int K) {
  Layout L{};
  const int B = (fmt == FP4_MXFP4) ? 32 : 16;
  const int smem_cap = 227 * 1024 - 256;    // leave room for the kernel's static shared memory
  const int extra = kRows * kOutPitch * 4 + 16 * kMaxStages + 1024;
  for (int kc : {1024, 768, 512, 256}) {
    if (K % kc != 0) continue;
    Layout c{};
    c.kc = kc;
    c.nchunks = K / kc;
    c.scale_row = kc / B;
    c.codes_off = 0;
    c.scales_off = kRows * kc / 2;
    c.x_off = c.scales_off + kRows * c.scale_row;
    c.x_row = 2 * kc + 64;
    c.stage_bytes = static_cast<int>(align_up(c.x_off + kTok * c.x_row, 1024));
    c.stages = std::min(kMaxStages, (smem_cap - extra) / c.stage_bytes);
    if (c.stages < 2) continue;
    c.out_off = c.stages * c.stage_bytes;
    c.bar_off = c.out_off + kRows * kOutPitch * 4;
    c.smem_bytes = c.bar_off + 16 * kMaxStages + 1024;   // + alignment slack
    return c;
  }
  return L;
}

template <int kFmt, int kEpi>
fp4_status launch_one(const DecodeArgs& a, const Layout& L, const CUtensorMap& map, int grid,
                      cudaStream_t st, bool pdl) {
  auto kern = decode_kernel<kFmt, kEpi>;
  static thread_local int configured = 0;
  if (configured < L.smem_bytes) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.smem_bytes));
    configured = L.smem_bytes;
  }
  return launch_pdl(kern, dim3(grid), dim3(kThreads), static_cast<size_t>(L.smem_bytes), st, pdl, map, a, L);
}

}  // namespace

fp4_status launch_decode(const DecodeArgs& a, cudaStream_t st, bool pdl) {
  const Layout L = make_layout(a.fmt, a.K);
  if (L.kc == 0) return FP4_ERR_UNSUPPORTED;
  CUtensorMap map;
  FP4_TRY(make_tmap_2d_u8(&map, a.codes, static_cast<uint64_t>(a.K / 2), static_cast<uint64_t>(a.rows_total),
                          static_cast<uint64_t>(a.K / 2), 128, 32, CU_TENSOR_MAP_SWIZZLE_128B));
  int grid = num_sms();
  if (a.units == nullptr) {
    const int n = a.static_tiles * ((a.static_T + kTok - 1) / kTok);
    grid = std::min(grid, n);
  }
  const int key = (a.fmt == FP4_NVFP4 ? 3 : 0) + a.epi;
  switch (key) {
    case 0: return launch_one<FP4_MXFP4, kEpiSwiglu>(a, L, map, grid, st, pdl);
    case 1: return launch_one<FP4_MXFP4, kEpiDown>(a, L, map, grid, st, pdl);
    case 2: return launch_one<FP4_MXFP4, kEpiLinear>(a, L, map, grid, st, pdl);
    case 3: return launch_one<FP4_NVFP4, kEpiSwiglu>(a, L, map, grid, st, pdl);
    case 4: return launch_one<FP4_NVFP4, kEpiDown>(a, L, map, grid, st, pdl);
    default: return launch_one<FP4_NVFP4, kEpiLinear>(a, L, map, grid, st, pdl);
  }
}

// y[t, n] = bf16( sum_{j = 0..k-1} o[inv[t k + j], n] ), fixed j order.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv,
                                                      int T, int k, int H, uint16_t* __restrict__ y) {
  pdl_wait();
  const int64_t n4 = static_cast<int64_t>(T) * (H / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int tt = static_cast<int>(i / (H / 4));
    const int h = static_cast<int>(i % (H / 4)) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(o + static_cast<int64_t>(inv[tt * k + j]) * H + h);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(s.x)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.y))) << 16);
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(s.z)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.w))) << 16);
    *reinterpret_cast<uint2*>(y + static_cast<int64_t>(tt) * H + h) = make_uint2(lo, hi);
  }
  pdl_launch_dependents();
}

}  // namespace fp4

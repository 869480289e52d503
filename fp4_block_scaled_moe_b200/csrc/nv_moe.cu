// Grouped NVFP4 expert GEMMs on the tensor cores (tcgen05.mma kind::f16).
//
// Format: NVFP4 as "XFP：质量地板驱动的自适应码本量化" (section 路线二) describes it, E2M1
// elements with one FP8 E4M3 scale per 16 and one float32 scale per tensor.  The block-
// scaled MMA kinds take power-of-two (UE8M0) scales per 32 or FP4 activations, neither of
// which fits bf16 activations with E4M3 scales per 16, so here the weights are widened
// on chip: E2M1 x E4M3 is exact in f16 (at most 6 significant bits, magnitudes in
// [2^-10, 2688]), and x enters as f16 with a power-of-two scale per routed slot (exact
// for bf16 values within the 2^15 range below the row's largest).  The tensor scale and
// the activation scale multiply the fp32 accumulator in the epilogue.
//
// A work unit is (expert, tile, token group): one 128-row weight tile times up to 256
// activation rows into one fp32 accumulator in TMEM (double-buffered against the
// epilogue).  gate_up tiles are 64 gate rows and the 64 up rows of the same intermediate
// indices; down tiles are 128 output rows.  K advances 64 per stage (one 128-byte
// swizzle row of f16).
//
// Warp roles of a persistent CTA (one per SM, two for units of <= 64 columns):
//   warp 0     weight producer: TMA of the tile's 4-bit codes (two 64-row boxes, 32 bytes
//              of K each) and one bulk copy of its 512-byte E4M3 scale atom per stage into
//              a deep ring, and the unit sequence (taken from the work counter) for warp 1.
//   warp 1     activation producer: TMA of the unit's f16 rows (128-byte swizzle).
//   warp 2     MMA issuer and TMEM owner: 4 MMAs of K = 16 per stage.
//   warps 3-6  converters, one weight row per thread: codes -> f16 pairs (cvt e2m1x2),
//              times the block's E4M3 scale (exact), stored in the 128-byte swizzled
//              K-major layout the MMA reads.
//   warps 7-10 epilogue, one TMEM lane quadrant each.  gate_up: up rows reach the gate
//              warps through shared memory; h = silu(min(g, L)) clamp(u, -L, L) is written
//              as f16 in slot order for the down GEMM.  down: rows times the gate weight
//              and the tensor scale, fp32 in slot order for the combine.
#include <algorithm>

#include "kernels.cuh"
#include "tcgen05.cuh"

namespace fp4 {
namespace {

constexpr int kNvKS = 64;                         // K per stage
constexpr int kNvCodes = 128 * kNvKS / 2;         // 4 KB of codes per 128-row tile and stage
constexpr int kNvRawBytes = kNvCodes + 512;       // + the stage's scale atom
constexpr int kNvATile = 128 * 128;               // f16 A tile (128 rows x 128 B)
constexpr int kNvMaxCols = 256;
constexpr int kNvWarps = 11;
constexpr int kNvThreads = kNvWarps * 32;
constexpr int kNvMaxR = 16, kNvMaxQA = 4, kNvMaxQB = 8, kNvUQ = 8;
constexpr int kNvMaxExperts = 1024;
constexpr int kWConv0 = 3, kWEpi0 = 7;

struct NvLayout {
  int cap;           // tokens per unit
  int ncols;         // B rows per unit = accumulator columns (16-multiple, <= 256)
  int R, QA, QB;     // ring depths: raw weights, f16 weights, activations
  int b_stage;       // bytes of one activation stage
  int raw_off, a_off, b_off, xch_off, cnt_off, off_off, pre_off, bar_off, int_off;
  int smem_bytes, tmem_cols, ctas_per_sm;
};

struct NvUnit {
  int e, tile, slot0, ntok;
};

__device__ __forceinline__ NvUnit nv_unit_of(int u, const int* cnt, const int* off, const int* pre, int E,
                                             int tiles, int cap) {
  int lo = 0, hi = E - 1;                  // largest e with pre[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid - 1;
  }
  NvUnit un;
  un.e = lo;
  const int n = cnt[lo];
  const int groups = (n + cap - 1) / cap;
  const int local = u - pre[lo];
  un.tile = local / groups;
  const int grp = local - un.tile * groups;
  un.slot0 = off[lo] + grp * cap;
  un.ntok = min(cap, n - grp * cap);
  return un;
}

// v[m] for a warp-uniform m in 0..7, from registers (no local-memory indexing); a 16-column
// chunk starting at c0 (a multiple of 16) lies in the lane group c0 >> 5.
__device__ __forceinline__ float pick8(const float (&v)[8], int m) {
  float r = v[0];
#pragma unroll
  for (int j = 1; j < 8; ++j) r = (m == j) ? v[j] : r;
  return r;
}

__device__ __forceinline__ void nv_epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// f16 pair (lo, hi) from the two E4M3 bytes of v -> the lo / hi value broadcast to both halves
__device__ __forceinline__ uint32_t bcast_lo(uint32_t h2) { return __byte_perm(h2, 0u, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h2) { return __byte_perm(h2, 0u, 0x3232); }

template <int kEpi, int kCtas>
__global__ void __launch_bounds__(kNvThreads, kCtas)
    nv_moe_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const NvArgs a, const NvLayout L) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - sraw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = L.R, QA = L.QA, QB = L.QB;
  // barriers (8 bytes each)
  const uint32_t b_full_raw = sbase + L.bar_off;
  const uint32_t b_empty_raw = b_full_raw + 8 * kNvMaxR;
  const uint32_t b_full_a = b_empty_raw + 8 * kNvMaxR;
  const uint32_t b_empty_a = b_full_a + 8 * kNvMaxQA;
  const uint32_t b_full_b = b_empty_a + 8 * kNvMaxQA;
  const uint32_t b_empty_b = b_full_b + 8 * kNvMaxQB;
  const uint32_t b_unit_full = b_empty_b + 8 * kNvMaxQB;
  const uint32_t b_unit_empty = b_unit_full + 8 * kNvUQ;
  const uint32_t b_accf = b_unit_empty + 8 * kNvUQ;
  const uint32_t b_acce = b_accf + 16;
  const uint32_t b_final = b_acce + 16;
  int* ints = reinterpret_cast<int*>(smem + L.int_off);
  int* raw_unit = ints;                      // [kNvMaxR]
  int* a_unit = raw_unit + kNvMaxR;          // [kNvMaxQA]
  int* unit_ring = a_unit + kNvMaxQA;        // [kNvUQ]
  int* acc_unit = unit_ring + kNvUQ;         // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_unit + 2);
  int* cnt = reinterpret_cast<int*>(smem + L.cnt_off);
  int* off = reinterpret_cast<int*>(smem + L.off_off);
  int* pre = reinterpret_cast<int*>(smem + L.pre_off);
  const int E = a.E;
  const int tiles = (kEpi == kEpiSwiglu) ? a.inter / 64 : a.rows_per_expert / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(b_full_raw + 8 * s, 1);
      mbar_init(b_empty_raw + 8 * s, 4);
    }
    for (int s = 0; s < QA; ++s) {
      mbar_init(b_full_a + 8 * s, 4);
      mbar_init(b_empty_a + 8 * s, 1);
    }
    for (int s = 0; s < QB; ++s) {
      mbar_init(b_full_b + 8 * s, 1);
      mbar_init(b_empty_b + 8 * s, 1);
    }
    for (int s = 0; s < kNvUQ; ++s) {
      mbar_init(b_unit_full + 8 * s, 1);
      mbar_init(b_unit_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_accf + 8 * b, 2);
      mbar_init(b_acce + 8 * b, 4);
    }
    mbar_init(b_final, 1);
    fence_barrier_init();
  }
  if (warp == 2) {
    tc::tmem_alloc(smem_u32(tmem_holder), static_cast<uint32_t>(L.tmem_cols));
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) slot_begin(a.slot);

  // per-expert unit prefix; units are ordered (expert, tile, token group)
  for (int e = threadIdx.x; e < E; e += kNvThreads) cnt[e] = a.counts[e];
  __syncthreads();
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    // slots of all experts; work units only for the experts in [e_begin, e_end)
    auto units = [&](int e) { return (e >= a.e_begin && e < a.e_end) ? (cnt[e] + L.cap - 1) / L.cap * tiles : 0; };
    int sc = 0, su = 0;
    for (int e = e0; e < e1; ++e) {
      sc += cnt[e];
      su += units(e);
    }
    int ic = sc, iu = su;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xFFFFFFFFu, ic, o), vu = __shfl_up_sync(0xFFFFFFFFu, iu, o);
      if (lane >= o) { ic += vc; iu += vu; }
    }
    int rc = ic - sc, ru = iu - su;
    for (int e = e0; e < e1; ++e) {
      off[e] = rc;
      pre[e] = ru;
      rc += cnt[e];
      ru += units(e);
    }
    if (lane == 31) { off[E] = ic; pre[E] = iu; }
  }
  __syncthreads();
  const int n_units = pre[E];
  const int nk = a.K / kNvKS;

  if (warp == 0) {
    // --------------------------- weight producer ---------------------------------------
    int it = 0, uq = 0;
    int u = blockIdx.x;
    bool ok = true;
    while (ok) {
      const int qs = uq % kNvUQ;
      if (uq >= kNvUQ &&
          !__all_sync(0xFFFFFFFFu, mbar_wait(b_unit_empty + 8 * qs, ((uq / kNvUQ) & 1) ^ 1, a.status)))
        break;
      if (lane == 0) {
        unit_ring[qs] = (u < n_units) ? u : -1;
        mbar_arrive(b_unit_full + 8 * qs);
      }
      __syncwarp();
      ++uq;
      if (u >= n_units) {
        const int s = it % R;
        if (it >= R && !__all_sync(0xFFFFFFFFu, mbar_wait(b_empty_raw + 8 * s, ((it / R) & 1) ^ 1, a.status)))
          break;
        if (lane == 0) {
          raw_unit[s] = -1;
          mbar_arrive(b_full_raw + 8 * s);
        }
        __syncwarp();
        ++it;
        break;
      }
      const NvUnit un = nv_unit_of(u, cnt, off, pre, E, tiles, L.cap);
      const int64_t rbase = static_cast<int64_t>(un.e - a.e_begin) * a.rows_per_expert;   // local expert
      const int64_t y0 = (kEpi == kEpiSwiglu) ? rbase + un.tile * 64 : rbase + un.tile * 128;
      const int64_t y1 = (kEpi == kEpiSwiglu) ? y0 + a.inter : y0 + 64;
      const int64_t tile_g = static_cast<int64_t>(un.e - a.e_begin) * tiles + un.tile;
      const uint8_t* sa = a.a_atoms + tile_g * nk * 512;
      for (int c = 0; c < nk; ++c, ++it) {
        const int s = it % R;
        if (it >= R && !__all_sync(0xFFFFFFFFu, mbar_wait(b_empty_raw + 8 * s, ((it / R) & 1) ^ 1, a.status))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          raw_unit[s] = u;
          const uint32_t dst = sbase + L.raw_off + s * kNvRawBytes;
          mbar_arrive_expect_tx(b_full_raw + 8 * s, static_cast<uint32_t>(kNvRawBytes));
          tma_load_2d(dst, &tmA, c * (kNvKS / 2), static_cast<int32_t>(y0), b_full_raw + 8 * s);
          tma_load_2d(dst + kNvCodes / 2, &tmA, c * (kNvKS / 2), static_cast<int32_t>(y1), b_full_raw + 8 * s);
          bulk_g2s(dst + kNvCodes, sa + c * 512, 512, b_full_raw + 8 * s);
        }
        __syncwarp();
      }
      if (!ok) break;
      int v = 0;
      if (lane == 0) v = static_cast<int>(gridDim.x + atomicAdd(a.unit_next, 1u));
      u = __shfl_sync(0xFFFFFFFFu, v, 0);
    }
    // every copy this warp started has landed before the CTA may exit
    for (int d = 1; d <= R && d <= it; ++d) {
      const int j = it - d;
      mbar_wait(b_full_raw + 8 * (j % R), (j / R) & 1, a.status);
    }
  } else if (warp == 1) {
    // --------------------------- activation producer -----------------------------------
    int ib = 0, uq = 0;
    const uint32_t bbytes = static_cast<uint32_t>(L.b_stage);
    while (true) {
      const int qs = uq % kNvUQ;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(b_unit_full + 8 * qs, (uq / kNvUQ) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&unit_ring[qs]);
      __syncwarp();
      if (lane == 0) mbar_arrive(b_unit_empty + 8 * qs);
      ++uq;
      if (u < 0) break;
      const NvUnit un = nv_unit_of(u, cnt, off, pre, E, tiles, L.cap);
      bool ok = true;
      for (int c = 0; c < nk; ++c, ++ib) {
        const int s = ib % QB;
        if (ib >= QB && !__all_sync(0xFFFFFFFFu, mbar_wait(b_empty_b + 8 * s, ((ib / QB) & 1) ^ 1, a.status))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(b_full_b + 8 * s, bbytes);
          tma_load_2d(sbase + L.b_off + s * L.b_stage, &tmB, c * kNvKS, un.slot0, b_full_b + 8 * s);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
    for (int d = 1; d <= QB && d <= ib; ++d) {
      const int j = ib - d;
      mbar_wait(b_full_b + 8 * (j % QB), (j / QB) & 1, a.status);
    }
  } else if (warp == 2) {
    // --------------------------- MMA issuer --------------------------------------------
    int i = 0, uc = 0;
    bool ok = true;
    while (ok) {
      const int qa0 = i % QA;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(b_full_a + 8 * qa0, (i / QA) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&a_unit[qa0]);
      const int buf = uc & 1;
      if (uc >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(b_acce + 8 * buf, ((uc >> 1) & 1) ^ 1, a.status))) break;
      if (lane == 0) {
        acc_unit[buf] = u;
        mbar_arrive(b_accf + 8 * buf);
        if (u < 0) mbar_arrive(b_accf + 8 * buf);
      }
      __syncwarp();
      if (u < 0) break;
      tc::fence_after_sync();
      const NvUnit un = nv_unit_of(u, cnt, off, pre, E, tiles, L.cap);
      const uint32_t N = static_cast<uint32_t>(max(16, (un.ntok + 15) & ~15));
      const uint32_t idesc = tc::idesc_f16(128u, N);
      const uint32_t d0 = tmem + static_cast<uint32_t>(buf * L.ncols);
      for (int c = 0; c < nk; ++c, ++i) {
        const int qa = i % QA, qb = i % QB;
        if (c > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(b_full_a + 8 * qa, (i / QA) & 1, a.status))) {
          ok = false;
          break;
        }
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(b_full_b + 8 * qb, (i / QB) & 1, a.status))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (lane == 0) {
          const uint32_t sa = sbase + L.a_off + qa * kNvATile;
          const uint32_t sb = sbase + L.b_off + qb * L.b_stage;
#pragma unroll
          for (int j = 0; j < kNvKS / 16; ++j)
            tc::mma_f16(d0, tc::desc_k_sw128(sa + 32 * j), tc::desc_k_sw128(sb + 32 * j), idesc,
                        static_cast<uint32_t>((c | j) != 0));
          tc::commit(b_empty_a + 8 * qa);
          tc::commit(b_empty_b + 8 * qb);
          if (c == nk - 1) tc::commit(b_accf + 8 * buf);
        }
        __syncwarp();
      }
      ++uc;
    }
    if (lane == 0) tc::commit(b_final);
    __syncwarp();
    mbar_wait(b_final, 0, a.status);
  } else if (warp < kWEpi0) {
    // --------------------------- converters --------------------------------------------
    const int cw = warp - kWConv0;
    const int r = cw * 32 + lane;               // weight row of the tile
    const uint32_t swz = static_cast<uint32_t>(r & 7);
    int it = 0;
    while (true) {
      const int s = it % R;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(b_full_raw + 8 * s, (it / R) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&raw_unit[s]);
      const int q = it % QA;
      if (it >= QA && !__all_sync(0xFFFFFFFFu, mbar_wait(b_empty_a + 8 * q, ((it / QA) & 1) ^ 1, a.status))) break;
      if (u < 0) {
        if (cw == 0 && lane == 0) a_unit[q] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(b_full_a + 8 * q);
        break;
      }
      const uint8_t* raw = smem + L.raw_off + s * kNvRawBytes;
      const uint4 c0 = *reinterpret_cast<const uint4*>(raw + r * 32);
      const uint4 c1 = *reinterpret_cast<const uint4*>(raw + r * 32 + 16);
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(raw + kNvCodes + r * 4);
      const uint32_t s01 = e4m3x2_to_f16x2(sw & 0xFFFFu), s23 = e4m3x2_to_f16x2(sw >> 16);
      const uint32_t sc[4] = {bcast_lo(s01), bcast_hi(s01), bcast_lo(s23), bcast_hi(s23)};
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint8_t* arow = smem + L.a_off + q * kNvATile + r * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t h0, h1, h2, h3;
        e2m1x8_to_f16x8(w[j], h0, h1, h2, h3);
        const uint32_t m = sc[j >> 1];
        *reinterpret_cast<uint4*>(arow + ((static_cast<uint32_t>(j) ^ swz) << 4)) =
            make_uint4(hmul2(h0, m), hmul2(h1, m), hmul2(h2, m), hmul2(h3, m));
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        if (cw == 0) a_unit[q] = u;
        mbar_arrive(b_full_a + 8 * q);
        mbar_arrive(b_empty_raw + 8 * s);
      }
      ++it;
    }
  } else {
    // --------------------------- epilogue ----------------------------------------------
    const int q = warp & 3;                    // TMEM lane quadrant this warp may access
    const int row = 32 * q + lane;             // accumulator row = row of the weight tile
    float* xch = reinterpret_cast<float*>(smem + L.xch_off);   // [2][64][16] up values for the gate warps
    int uc = 0;
    while (true) {
      const int buf = uc & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(b_accf + 8 * buf, (uc >> 1) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&acc_unit[buf]);
      if (u < 0) break;
      tc::fence_after_sync();
      const NvUnit un = nv_unit_of(u, cnt, off, pre, E, tiles, L.cap);
      const uint32_t d0 = tmem + static_cast<uint32_t>(buf * L.ncols) + (static_cast<uint32_t>(32 * q) << 16);
      const int N = max(16, (un.ntok + 15) & ~15);
      const float ts = a.tscale[un.e - a.e_begin];
      // per-column factor of the unit's tokens: lane l holds columns l, 32 + l, ... (<= 256)
      float fl[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i = lane + 32 * m;
        float f = 0.f;
        if (i < un.ntok) {
          const int slot = un.slot0 + i;
          f = (kEpi == kEpiSwiglu) ? ldexpf(ts, a.sx[slot]) : ts * a.gw[a.perm[slot]];
        }
        fl[m] = f;
      }
      if (kEpi == kEpiSwiglu) {
        const int64_t col = static_cast<int64_t>(un.tile) * 64 + (row & 63);
        for (int c0 = 0; c0 < N; c0 += 16) {
          float* xb = xch + ((c0 >> 4) & 1) * (64 * 16);
          uint32_t v[16];
          tc::ld_32x32b_x16(d0 + static_cast<uint32_t>(c0), v);
          tc::ld_wait();
          if (q >= 2) {
#pragma unroll
            for (int j = 0; j < 16; ++j) xb[(row - 64) * 16 + j] = __uint_as_float(v[j]);
          }
          nv_epi_bar();
          if (q < 2) {
            const float fsel = pick8(fl, c0 >> 5);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int i = c0 + j;
              const float f = __shfl_sync(0xFFFFFFFFu, fsel, i & 31);
              if (i < un.ntok) {
                const float g = fminf(__uint_as_float(v[j]) * f, a.limit);
                const float uu = fminf(fmaxf(xb[row * 16 + j] * f, -a.limit), a.limit);
                const float hv = g / (1.0f + expf(-g)) * uu;
                a.h_out[(static_cast<int64_t>(un.slot0) + i) * a.inter + col] = __float2half_rn(hv);
              }
            }
          }
        }
      } else {
        float* o0 = a.o_out + static_cast<int64_t>(un.slot0) * a.ldo + static_cast<int64_t>(un.tile) * 128 + row;
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t v[16];
          tc::ld_32x32b_x16(d0 + static_cast<uint32_t>(c0), v);
          tc::ld_wait();
          const float fsel = pick8(fl, c0 >> 5);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int i = c0 + j;
            const float f = __shfl_sync(0xFFFFFFFFu, fsel, i & 31);
            if (i < un.ntok) o0[static_cast<int64_t>(i) * a.ldo] = __uint_as_float(v[j]) * f;
          }
        }
      }
      tc::fence_before_sync();
      nv_epi_bar();
      if (lane == 0) mbar_arrive(b_acce + 8 * buf);
      ++uc;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, static_cast<uint32_t>(L.tmem_cols));
  }
  if (threadIdx.x == 0) slot_end(a.slot);
}

// NVFP4 scales [rows][K/16] -> atoms of 128 rows x 4 bytes (the four 16-blocks of a 64-K
// stage), row r of the tile at byte 4 r.  pair == 0: tiles of 128 consecutive rows;
// pair == I: tile t of expert e is gate rows t*64 .. +63 then up rows I + t*64 .. +63.
__global__ void __launch_bounds__(256) nv_scales_kernel(const uint8_t* __restrict__ scales, int64_t rows,
                                                        int64_t K, int64_t pair, uint8_t* __restrict__ atoms) {
  const int64_t kb = K / kNvKS, total = rows * kb;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / kb, c = idx % kb;
    int64_t tile;
    int within;
    if (pair == 0) {
      tile = r >> 7;
      within = static_cast<int>(r & 127);
    } else {
      const int64_t e = r / (2 * pair), rl = r % (2 * pair);
      const bool up = rl >= pair;
      const int64_t q = up ? rl - pair : rl;
      tile = e * (pair / 64) + q / 64;
      within = static_cast<int>(q % 64) + (up ? 64 : 0);
    }
    const uint32_t w = *reinterpret_cast<const uint32_t*>(scales + r * (K / 16) + 4 * c);
    *reinterpret_cast<uint32_t*>(atoms + (tile * kb + c) * 512 + within * 4) = w;
  }
}

constexpr int kNvSmemLimit = 227 * 1024;

bool nv_layout(int T, int E, NvLayout* L) {
  if (E > kNvMaxExperts) return false;
  L->cap = std::min(kNvMaxCols, std::max(16, (T + 15) / 16 * 16));
  L->ncols = L->cap;
  L->ctas_per_sm = (L->ncols <= 64) ? 2 : 1;
  const int limit = (L->ctas_per_sm == 2) ? 113 * 1024 : kNvSmemLimit;
  L->b_stage = L->ncols * 128;
  L->QA = (L->ctas_per_sm == 2) ? 2 : 3;
  L->QB = (L->ctas_per_sm == 2) ? 3 : 3;
  // fixed part: exchange buffer, per-expert tables, barriers, small ints
  int off = 0;
  const int xch = off;
  off += 2 * 64 * 16 * 4;
  const int c0 = off;
  off += 4 * (E + 1);
  const int o0 = off;
  off += 4 * (E + 1);
  const int p0 = off;
  off += 4 * (E + 1);
  off = static_cast<int>(align_up(off, 16));
  const int b0 = off;
  off += 8 * (2 * kNvMaxR + 2 * kNvMaxQA + 2 * kNvMaxQB + 2 * kNvUQ + 5);
  const int i0 = off;
  off += 4 * (kNvMaxR + kNvMaxQA + kNvUQ + 2 + 2);
  const int fixed = static_cast<int>(align_up(off, 128));
  const int ab = L->QA * kNvATile + L->QB * L->b_stage;
  const int R = (limit - 1024 - fixed - ab) / kNvRawBytes;
  L->R = std::min(R, kNvMaxR);
  if (L->R < 2) return false;
  L->a_off = 0;
  L->b_off = L->a_off + L->QA * kNvATile;
  L->raw_off = L->b_off + L->QB * L->b_stage;
  const int body = static_cast<int>(align_up(L->raw_off + L->R * kNvRawBytes, 128));
  L->xch_off = body + xch;
  L->cnt_off = body + c0;
  L->off_off = body + o0;
  L->pre_off = body + p0;
  L->bar_off = body + b0;
  L->int_off = body + i0;
  L->smem_bytes = body + fixed + 1024;       // + slack for the 1024-byte alignment of the base
  int cols = 32;
  while (cols < 2 * L->ncols) cols *= 2;
  L->tmem_cols = cols;
  return L->smem_bytes <= limit;
}

template <int kEpi, int kCtas>
fp4_status launch_nv_t(const NvArgs& a, const NvLayout& L, const CUtensorMap& mA, const CUtensorMap& mB,
                       cudaStream_t st) {
  auto kern = nv_moe_kernel<kEpi, kCtas>;
  static thread_local bool configured = false;
  if (!configured) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kNvSmemLimit));
    configured = true;
  }
  return launch_pdl(kern, dim3(kCtas * num_sms()), dim3(kNvThreads), static_cast<size_t>(L.smem_bytes), st, true,
                    mA, mB, a, L);
}

}  // namespace

int nv_ntok_cap(int T, int E) {
  NvLayout L;
  return nv_layout(T, E, &L) ? L.cap : 0;
}

bool nv_supported(int T, int E, int H, int I) {
  NvLayout L;
  return H % 128 == 0 && I % 64 == 0 && H % kNvKS == 0 && I % kNvKS == 0 && nv_layout(T, E, &L);
}

fp4_status launch_nv_scales(const uint8_t* scales, int64_t rows, int64_t K, int64_t pair, uint8_t* atoms,
                            cudaStream_t st) {
  const int64_t total = rows * (K / kNvKS);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, num_sms() * 16)));
  nv_scales_kernel<<<grid, 256, 0, st>>>(scales, rows, K, pair, atoms);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch();
  return FP4_OK;
}

fp4_status launch_nv(const NvArgs& a, int T, cudaStream_t st) {
  NvLayout L;
  if (!nv_layout(T, a.E, &L) || L.cap != a.ntok_cap) return FP4_ERR_UNSUPPORTED;
  CUtensorMap mA, mB;
  FP4_TRY(make_tmap_2d_u8(&mA, a.codes, static_cast<uint64_t>(a.K / 2), static_cast<uint64_t>(a.rows_total),
                          static_cast<uint64_t>(a.K / 2), kNvKS / 2, 64, CU_TENSOR_MAP_SWIZZLE_NONE));
  FP4_TRY(make_tmap_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.b_rows, static_cast<uint64_t>(a.K),
                       static_cast<uint64_t>(a.P), static_cast<uint64_t>(a.K) * 2, kNvKS,
                       static_cast<uint32_t>(L.ncols), CU_TENSOR_MAP_SWIZZLE_128B));
  if (a.epi == kEpiSwiglu)
    return L.ctas_per_sm == 2 ? launch_nv_t<kEpiSwiglu, 2>(a, L, mA, mB, st) : launch_nv_t<kEpiSwiglu, 1>(a, L, mA, mB, st);
  return L.ctas_per_sm == 2 ? launch_nv_t<kEpiDown, 2>(a, L, mA, mB, st) : launch_nv_t<kEpiDown, 1>(a, L, mA, mB, st);
}

}  // namespace fp4

// Grouped MXFP4 expert GEMMs on the block-scaled tensor cores (tcgen05.mma
// kind::mxf8f6f4): the 4-bit weights go from HBM to shared memory by TMA and straight
// into the MMA with their UE8M0 block scales; no CUDA core touches a weight.
//
// Format: MXFP4 as "XFP：质量地板驱动的自适应码本量化" (section 路线二) describes it, E2M1
// elements with one power-of-two scale per 32.  The bf16 activations keep their accuracy
// by entering the MMA as the sum of two MXFP8 terms (E4M3 elements, UE8M0 scale per 32):
// x = t1 + t2 with t1 = E4M3(x / s1) s1 and t2 = E4M3((x - t1) / s2) s2, leaving about
// 2^-8 |x| per element.  The two terms of token slot i are B rows 2i and 2i + 1, so the
// product with x_i is D[:, 2i] + D[:, 2i + 1].
//
// A work unit is (expert, tile, token group): one 128-row weight tile times the group's
// activation rows (up to 224 = 112 slots x 2 terms) into one fp32 accumulator in TMEM.
// Each M = 128, K = 32 MMA reads its 4 KB A tile from shared memory in about the time
// of a 128 x 256 product, so the units carry as many columns as TMEM allows.  gate_up
// tiles are 64 gate rows followed by the 64 up rows of the same intermediate indices;
// down tiles are 128 output rows.
//
// Warp roles of a persistent CTA (one per SM; two or three for decode-sized units of <= 64
// or <= 32 columns):
//   warp 0     producer: TMA of the weight tile (two 64-row boxes, FP4 widened to
//              16-byte slots, 128-byte swizzle) and of the activation-term tile, and one
//              bulk copy per scale atom (weights: re-laid once by fp4_mma_scales or per
//              call into the workspace; activations: written as atoms by their producers).
//   warp 1     MMA issuer and TMEM owner: per stage, scales -> TMEM, then 4 MMAs of K = 32
//              into one of two accumulators (double-buffered against the epilogue).
//   warps 2-5  epilogue, one TMEM lane quadrant each: term pairs summed.  gate_up: the up
//              warps hand their rows to the gate warps through shared memory; the gate
//              warps apply the SwiGLU clamp and write h split again into two MXFP8 terms
//              for the down GEMM.  down: rows scaled by the gate weight, written as fp32 in
//              slot order for the combine.
#include <algorithm>

#include "kernels.cuh"
#include "routing.cuh"
#include "tcgen05.cuh"

namespace fp4 {
namespace {

constexpr int kBsThreads = 6 * 32;
constexpr int kBsMaxStages = 8;
constexpr int kKT = 128;                  // K elements per stage (one 128-byte swizzle row of E4M3)
constexpr int kATile = 128 * 128;         // shared bytes of the 128-row FP4 tile (16-byte slots)
constexpr int kSfBytes = 3 * 512;         // scale atoms per stage: A, B rows 0-127, B rows 128-255
constexpr int kSfCols = 16;               // TMEM columns per stage for scales (A 4, B 8)
constexpr int kMaxTokCap = 112;           // tokens per unit: accumulators of 224 columns
constexpr int kMaxExperts = 1024;

struct BsLayout {
  int ntok_cap;      // tokens per work unit
  int ncols;         // columns per accumulator = rows of the B box (16-multiple, <= 224)
  int stage_bytes;
  int stages;
  int tmem_cols;
  int xch_off, cnt_off, off_off, pre_off, gpre_off, bar_off;
  int smem_bytes;
  int ctas_per_sm;   // 2 for narrow units (decode), else 1
};

struct BsUnit {
  int e, tile, slot0, ntok, gid;    // gid: token group number across experts
};

// gpre: token-group prefix over all experts (the numbering the activation atoms use).
__device__ __forceinline__ BsUnit bs_unit_of(int u, const int* cnt, const int* off, const int* pre,
                                            const int* gpre, int E, int tiles, int cap) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid - 1;
  }
  BsUnit un;
  un.e = lo;
  const int n = cnt[lo];
  const int groups = (n + cap - 1) / cap;
  const int local = u - pre[lo];
  un.tile = local / groups;
  const int grp = local - un.tile * groups;
  un.slot0 = off[lo] + grp * cap;
  un.ntok = min(cap, n - grp * cap);
  un.gid = gpre[lo] + grp;
  return un;
}


// byte offset of row r (0..127) in a scale atom: 32 rows x 16 bytes, row r at line r % 32,
// word r / 32 (the four bytes of a word are the four 32-element blocks of one stage)
__device__ __forceinline__ uint32_t sf_row_off(int r) {
  return static_cast<uint32_t>((r & 31) * 16 + (r >> 5) * 4);
}
__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// activation-term rows 0..255 of a token group span two atoms
__device__ __forceinline__ uint32_t sf_row_off2(int r) { return static_cast<uint32_t>((r >> 7) * 512) + sf_row_off(r & 127); }

// E4M3 byte (satfinite, round to nearest even) of y, and its exact value
__device__ __forceinline__ uint32_t e4m3_rn(float y, float& back) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.0f), "f"(y));
  const uint32_t q = pair & 0xFFu;
  uint32_t h2;
  asm("{\n .reg .b16 lo;\n cvt.u16.u32 lo, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}" : "=r"(h2) : "r"(q));
  back = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xFFFFu)));
  return q;
}

// Two at once: E4M3 bytes of y0 (low byte) and y1 (high byte), and their exact values
__device__ __forceinline__ uint32_t e4m3x2_rn(float y0, float y1, float& back0, float& back1) {
  uint16_t pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(y1), "f"(y0));
  uint32_t h2;
  asm("{\n .reg .b16 lo;\n cvt.u16.u32 lo, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}" : "=r"(h2) : "r"(static_cast<uint32_t>(pair)));
  back0 = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xFFFFu)));
  back1 = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 >> 16)));
  return pair;
}

// UE8M0 exponent for a block of E4M3 elements from the bits of its amax (finite, >= 0):
// the least e with amax * 2^-e <= 448 (E4M3's largest finite value), kept in [-126, 127]
// so that 2^e and 2^-e are normal floats.  amax in [2^(B-127), 2^(B-126)) for biased
// exponent B; e = B - 135 puts amax 2^-e in [256, 512), one more when the significand
// exceeds 1.75.
__device__ __forceinline__ int e4m3_block_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int e = static_cast<int>(b >> 23) - 135 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return max(-126, min(127, e));
}
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }

// max |v| over the warp: for non-negative floats the bit patterns order like the values
__device__ __forceinline__ float warp_amax(float v) {
  return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fabsf(v))));
}

// Two-term split of the 32 values held by a warp (one per lane): E4M3 bytes of both
// terms for this lane and the two UE8M0 scale bytes (identical in all lanes).
__device__ __forceinline__ void warp_split2(float v, uint32_t& q1, uint32_t& q2, uint32_t& s1, uint32_t& s2) {
  const int e1 = e4m3_block_exp(warp_amax(v));
  float b1;
  q1 = e4m3_rn(v * exp2i(-e1), b1);
  const float r = v - b1 * exp2i(e1);
  const int e2 = e4m3_block_exp(warp_amax(r));
  float b2;
  q2 = e4m3_rn(r * exp2i(-e2), b2);
  s1 = static_cast<uint32_t>(e1 + 127);
  s2 = static_cast<uint32_t>(e2 + 127);
}

// The two E4M3 terms of one 32-element block of a token row and their UE8M0 scales
struct Split32 {
  uint32_t w1[8], w2[8];
  int e1, e2;
};

// One 32-element block b of token row t (bf16) -> its two-term split
__device__ __forceinline__ void split_compute(const uint16_t* __restrict__ x, int t, int b, int H, Split32& sp) {
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H + 32 * b);
  float v[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 w = src[j];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      v[8 * j + 2 * ii] = __uint_as_float(ws[ii] << 16);
      v[8 * j + 2 * ii + 1] = __uint_as_float(ws[ii] & 0xFFFF0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int ii = 0; ii < 32; ++ii) amax = fmaxf(amax, fabsf(v[ii]));
  const int e1 = e4m3_block_exp(amax);
  const float inv1 = exp2i(-e1), up1 = exp2i(e1);
  uint32_t* w1 = sp.w1;
  uint32_t* w2 = sp.w2;
  float ramax = 0.f;
#pragma unroll
  for (int ii = 0; ii < 32; ii += 2) {
    float b0, b1;
    const uint32_t c = e4m3x2_rn(v[ii] * inv1, v[ii + 1] * inv1, b0, b1);
    if ((ii & 3) == 0) w1[ii >> 2] = 0;
    w1[ii >> 2] |= c << (8 * (ii & 3));
    v[ii] -= b0 * up1;
    v[ii + 1] -= b1 * up1;
    ramax = fmaxf(ramax, fmaxf(fabsf(v[ii]), fabsf(v[ii + 1])));
  }
  const int e2 = e4m3_block_exp(ramax);
  const float inv2 = exp2i(-e2);
#pragma unroll
  for (int ii = 0; ii < 32; ii += 2) {
    float b0, b1;
    const uint32_t c = e4m3x2_rn(v[ii] * inv2, v[ii + 1] * inv2, b0, b1);
    if ((ii & 3) == 0) w2[ii >> 2] = 0;
    w2[ii >> 2] |= c << (8 * (ii & 3));
  }
  sp.e1 = e1;
  sp.e2 = e2;
}

// A block's split into rows 2 slot and 2 slot + 1 of q, and its two UE8M0 scales into the
// token group's atoms (rows 2i, 2i + 1)
__device__ __forceinline__ void split_store(const Split32& sp, int slot, int b, int i, int64_t gid, int H,
                                            uint8_t* __restrict__ q, uint8_t* __restrict__ atoms) {
  const int kb128 = H / 128;
  uint4* d1 = reinterpret_cast<uint4*>(q + (2 * static_cast<int64_t>(slot)) * H + 32 * b);
  uint4* d2 = reinterpret_cast<uint4*>(q + (2 * static_cast<int64_t>(slot) + 1) * H + 32 * b);
  d1[0] = make_uint4(sp.w1[0], sp.w1[1], sp.w1[2], sp.w1[3]);
  d1[1] = make_uint4(sp.w1[4], sp.w1[5], sp.w1[6], sp.w1[7]);
  d2[0] = make_uint4(sp.w2[0], sp.w2[1], sp.w2[2], sp.w2[3]);
  d2[1] = make_uint4(sp.w2[4], sp.w2[5], sp.w2[6], sp.w2[7]);
  uint8_t* at = atoms + (gid * kb128 + (b >> 2)) * 1024 + (b & 3);
  at[sf_row_off2(2 * i)] = static_cast<uint8_t>(sp.e1 + 127);
  at[sf_row_off2(2 * i + 1)] = static_cast<uint8_t>(sp.e2 + 127);
}

// Expert of a slot (largest e with off[e] <= slot), its position in the expert's token
// group and the group's number across experts
__device__ __forceinline__ void slot_place(const int* off, const int* gpre, int E, int cap, int slot, int& i,
                                           int64_t& gid) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= slot) lo = mid; else hi = mid - 1;
  }
  const int local = slot - off[lo];
  const int grp = local / cap;
  i = local - grp * cap;
  gid = static_cast<int64_t>(gpre[lo]) + grp;
}

// x [T][H] bf16 -> slot-ordered two-term MXFP8 rows q [2P][H] E4M3 (rows 2i, 2i + 1 for
// slot i = token perm[i] / k) and their UE8M0 scales as token-group atoms.  One thread
// per 32-element block of a token: the split is computed once and stored into each of the
// token's k slots (inv: pair -> slot).
__global__ void __launch_bounds__(256) split_x_kernel(const uint16_t* __restrict__ x,
                                                      const int32_t* __restrict__ inv,
                                                      const int32_t* __restrict__ counts,
                                                      const int32_t* __restrict__ offsets, int E, int k, int P,
                                                      int H, int cap, uint8_t* __restrict__ q,
                                                      uint8_t* __restrict__ atoms) {
  __shared__ int off_s[kMaxExperts + 1], gpre_s[kMaxExperts + 1];
  pdl_wait();
  // group number of each expert's first group: exclusive scan of ceil(count / cap)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int sg = 0;
    for (int e = e0; e < e1; ++e) sg += (counts[e] + cap - 1) / cap;
    int ig = sg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, ig, o);
      if (lane >= o) ig += v;
    }
    int rg = ig - sg;
    for (int e = e0; e < e1; ++e) {
      gpre_s[e] = rg;
      rg += (counts[e] + cap - 1) / cap;
    }
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) off_s[e] = offsets[e];
  __syncthreads();
  const int nb = H / 32;
  const int64_t total = static_cast<int64_t>(P / k) * nb;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(idx / nb), b = static_cast<int>(idx % nb);
    Split32 sp;
    split_compute(x, t, b, H, sp);
    for (int j = 0; j < k; ++j) {
      const int slot = inv[t * k + j];
      int i;
      int64_t gid;
      slot_place(off_s, gpre_s, E, cap, slot, i, gid);
      split_store(sp, slot, b, i, gid, H, q, atoms);
    }
  }
  pdl_launch_dependents();
}

// Small routing problems (T k <= 1024 slots, E <= 512) in one launch: every CTA forms the
// top-k of the logits, the per-expert counts and the stable slot order in shared memory
// (CTA 0 also stores them for the later kernels: ids, gate weights, counts, offsets,
// perm, inv), then splits its share of the slots' activation rows like split_x_kernel.
__global__ void __launch_bounds__(512) route_split_kernel(
    const float* __restrict__ logits, int T, int E, int k, const uint16_t* __restrict__ x, int H, int cap,
    int32_t* __restrict__ ids, float* __restrict__ gw, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, uint8_t* __restrict__ q, uint8_t* __restrict__ atoms) {
  __shared__ int ids_s[kRouteMaxPairs], perm_s[kRouteMaxPairs];
  __shared__ int cnt[kRouteMaxExperts], off[kRouteMaxExperts + 1], cur[kRouteMaxExperts], gpre[kRouteMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int P = T * k;
  pdl_wait();
  for (int t = warp; t < T; t += nw)
    topk_warp(logits + static_cast<int64_t>(t) * E, E, k, ids_s + t * k,
              blockIdx.x == 0 ? gw + static_cast<int64_t>(t) * k : nullptr);
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    atomicAdd(&cnt[ids_s[p]], 1);
    if (blockIdx.x == 0) ids[p] = ids_s[p];
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scans: first slot and first token group of every expert
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int sc = 0, sg = 0;
    for (int e = e0; e < e1; ++e) {
      sc += cnt[e];
      sg += (cnt[e] + cap - 1) / cap;
    }
    int ic = sc, ig = sg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xFFFFFFFFu, ic, o), vg = __shfl_up_sync(0xFFFFFFFFu, ig, o);
      if (lane >= o) { ic += vc; ig += vg; }
    }
    int rc = ic - sc, rg = ig - sg;
    for (int e = e0; e < e1; ++e) {
      off[e] = rc;
      cur[e] = rc;
      gpre[e] = rg;
      rc += cnt[e];
      rg += (cnt[e] + cap - 1) / cap;
    }
    if (lane == 31) off[E] = ic;
    __syncwarp();
    // stable placement: pairs in ascending order, 32 per round, ranked within the round
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const bool live = p < P;
      const int e = live ? ids_s[p] : -1 - lane;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      const int rank = __popc(peers & lt);
      const int slot = live ? cur[e] + rank : 0;
      __syncwarp();
      if (live && rank == 0) cur[e] += __popc(peers);
      __syncwarp();
      if (live) {
        perm_s[slot] = p;
        if (blockIdx.x == 0) {
          perm[slot] = p;
          inv[p] = slot;
        }
      }
    }
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
      if (e < E) counts[e] = cnt[e];
      offsets[e] = off[e];
    }
  // one thread per (slot, 32-block): at decode sizes the parallelism matters more than the
  // repeated split of a token's blocks
  const int nb = H / 32;
  const int64_t total = static_cast<int64_t>(P) * nb;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int slot = static_cast<int>(idx / nb), b = static_cast<int>(idx % nb);
    Split32 sp;
    split_compute(x, perm_s[slot] / k, b, H, sp);
    int i;
    int64_t gid;
    slot_place(off, gpre, E, cap, slot, i, gid);
    split_store(sp, slot, b, i, gid, H, q, atoms);
  }
  pdl_launch_dependents();
}

// Weight scales [rows][K/32] -> atoms: one thread moves the 4-byte word of one row and
// one 128-K block.  pair == 0: tiles are 128 consecutive rows.  pair == I: rows are the
// gate_up rows of experts (2I rows each) and tile t of expert e is gate rows t*64 .. +63
// followed by up rows I + t*64 .. +63.
__global__ void __launch_bounds__(256) mma_scales_kernel(const uint8_t* __restrict__ scales, int64_t rows,
                                                         int64_t K, int64_t pair, uint8_t* __restrict__ atoms) {
  const int64_t kb = K / 128, total = rows * kb;
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
    const uint32_t w = *reinterpret_cast<const uint32_t*>(scales + r * (K / 32) + 4 * c);
    *reinterpret_cast<uint32_t*>(atoms + (tile * kb + c) * 512 + sf_row_off(within)) = w;
  }
}

template <int kEpi>
__global__ void __launch_bounds__(kBsThreads, 1)
    bs_moe_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const BsArgs a, const BsLayout L) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - sraw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = L.stages;
  const uint32_t bar_full = sbase + L.bar_off;
  const uint32_t bar_empty = bar_full + 8 * kBsMaxStages;
  const uint32_t bar_accf = bar_empty + 8 * kBsMaxStages;    // [2] MMA done + unit id posted
  const uint32_t bar_acce = bar_accf + 16;                    // [2] epilogue done with the buffer
  const uint32_t bar_final = bar_acce + 16;
  const uint32_t tmem_holder = bar_final + 8;
  int* stage_unit = reinterpret_cast<int*>(smem + L.bar_off + 8 * (2 * kBsMaxStages + 5) + 8);
  int* acc_unit = stage_unit + kBsMaxStages;
  int* cnt = reinterpret_cast<int*>(smem + L.cnt_off);
  int* off = reinterpret_cast<int*>(smem + L.off_off);
  int* pre = reinterpret_cast<int*>(smem + L.pre_off);
  int* gpre = reinterpret_cast<int*>(smem + L.gpre_off);
  const int E = a.E;
  const int tiles = (kEpi == kEpiSwiglu) ? a.inter / 64 : a.rows_per_expert / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 2);
      mbar_init(bar_acce + 8 * b, 4);
    }
    mbar_init(bar_final, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, static_cast<uint32_t>(L.tmem_cols));
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + (tmem_holder - sbase));
  // The down GEMM's work units follow from the routing counts, which an earlier kernel
  // (before gate_up) wrote, and its weights depend on nothing: its producer streams the
  // first stages' weights before waiting for gate_up; only h (the B operand) waits.  Every
  // other warp waits here.  gate_up needs the counts of the kernel just before it: it waits
  // first.
  const bool early_w = kEpi == kEpiDown;
  if (!early_w || warp != 0) pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0 && !early_w) slot_begin(a.slot);

  // per-expert unit prefix; units are ordered (expert, tile, token group)
  for (int e = threadIdx.x; e < E; e += kBsThreads) cnt[e] = a.counts[e];
  __syncthreads();
  if (warp == 0) {
    // slots, token groups (all experts) and work units (only the experts in [e_begin, e_end))
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    auto groups = [&](int e) { return (cnt[e] + L.ntok_cap - 1) / L.ntok_cap; };
    auto units = [&](int e) { return (e >= a.e_begin && e < a.e_end) ? groups(e) * tiles : 0; };
    int sc = 0, su = 0, sg = 0;
    for (int e = e0; e < e1; ++e) {
      sc += cnt[e];
      su += units(e);
      sg += groups(e);
    }
    int ic = sc, iu = su, ig = sg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xFFFFFFFFu, ic, o), vu = __shfl_up_sync(0xFFFFFFFFu, iu, o);
      const int vg = __shfl_up_sync(0xFFFFFFFFu, ig, o);
      if (lane >= o) { ic += vc; iu += vu; ig += vg; }
    }
    int rc = ic - sc, ru = iu - su, rg = ig - sg;
    for (int e = e0; e < e1; ++e) {
      off[e] = rc;
      pre[e] = ru;
      gpre[e] = rg;
      rc += cnt[e];
      ru += units(e);
      rg += groups(e);
    }
    if (lane == 31) { off[E] = ic; pre[E] = iu; gpre[E] = ig; }
  }
  __syncthreads();
  const int n_units = pre[E];
  const int nk = a.K / kKT;
  const uint32_t stg = static_cast<uint32_t>(L.stage_bytes);
  const uint32_t b_off = kATile, sf_off = kATile + L.ncols * kKT;   // within a stage

  if (warp == 0) {
    // ------------------------------------ producer ------------------------------------
    int it = 0;
    int u = blockIdx.x;
    bool ok = true;
    // down: weights (A tile + its scale atom) of the first unit's first stages before the
    // dependency wait; their stages get the rest (B tile + atoms) after it
    int pre_n = 0;
    if (early_w) {
      if (u < n_units) {
        const BsUnit un = bs_unit_of(u, cnt, off, pre, gpre, E, tiles, L.ntok_cap);
        const int64_t rbase = static_cast<int64_t>(un.e - a.e_begin) * a.rows_per_expert;
        const int64_t y0 = rbase + un.tile * 128, y1 = y0 + 64;
        const uint8_t* sa = a.a_atoms + (static_cast<int64_t>(un.e - a.e_begin) * tiles + un.tile) * nk * 512;
        const uint32_t sfb = 2 * un.ntok > 128 ? 1024u : 512u;
        pre_n = min(S, nk);
        for (int c = 0; c < pre_n; ++c) {
          const uint32_t st = sbase + c * stg;
          if (lane == 0) {
            stage_unit[c] = u;
            mbar_arrive_expect_tx(bar_full + 8 * c, static_cast<uint32_t>(128 * kKT / 2 + L.ncols * kKT) + 512u + sfb);
            bulk_g2s(st + sf_off, sa + c * 512, 512, bar_full + 8 * c);
            tma_load_2d(st, &tmA, c * kKT, static_cast<int32_t>(y0), bar_full + 8 * c);
            tma_load_2d(st + kATile / 2, &tmA, c * kKT, static_cast<int32_t>(y1), bar_full + 8 * c);
          }
          __syncwarp();
        }
      }
      pdl_wait();
      if (lane == 0) slot_begin(a.slot);
    }
    while (ok) {
      if (u >= n_units) {
        const int s = it % S;
        if (it >= S && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((it / S) & 1) ^ 1, a.status))) break;
        if (lane == 0) {
          stage_unit[s] = -1;
          mbar_arrive(bar_full + 8 * s);
        }
        ++it;
        break;
      }
      const BsUnit un = bs_unit_of(u, cnt, off, pre, gpre, E, tiles, L.ntok_cap);
      const int64_t rbase = static_cast<int64_t>(un.e - a.e_begin) * a.rows_per_expert;   // local expert
      const int64_t y0 = (kEpi == kEpiSwiglu) ? rbase + un.tile * 64 : rbase + un.tile * 128;
      const int64_t y1 = (kEpi == kEpiSwiglu) ? y0 + a.inter : y0 + 64;
      const int brow0 = 2 * un.slot0;
      const int64_t tile_g = static_cast<int64_t>(un.e - a.e_begin) * tiles + un.tile;   // tile across experts
      const uint8_t* sa = a.a_atoms + tile_g * nk * 512;
      const uint8_t* sb = a.b_atoms + static_cast<int64_t>(un.gid) * nk * 1024;
      const bool two_b = 2 * un.ntok > 128;
      for (int c = 0; c < nk; ++c, ++it) {
        const int s = it % S;
        if (it >= S && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((it / S) & 1) ^ 1, a.status))) {
          ok = false;
          break;
        }
        const bool a_done = it < pre_n;     // this stage's weights were issued before the wait
        if (lane == 0) stage_unit[s] = u;
        const uint32_t st = sbase + s * stg;
        const uint32_t sf = st + sf_off;
        if (lane == 0) {
          const uint32_t sfb = two_b ? 1024u : 512u;
          if (!a_done) {
            mbar_arrive_expect_tx(bar_full + 8 * s, static_cast<uint32_t>(128 * kKT / 2 + L.ncols * kKT) + 512u + sfb);
            bulk_g2s(sf, sa + c * 512, 512, bar_full + 8 * s);
            tma_load_2d(st, &tmA, c * kKT, static_cast<int32_t>(y0), bar_full + 8 * s);
            tma_load_2d(st + kATile / 2, &tmA, c * kKT, static_cast<int32_t>(y1), bar_full + 8 * s);
          }
          bulk_g2s(sf + 512, sb + c * 1024, sfb, bar_full + 8 * s);
          tma_load_2d(st + b_off, &tmB, c * kKT, brow0, bar_full + 8 * s);
        }
        __syncwarp();
      }
      if (!ok) break;
      int v = 0;
      if (lane == 0) v = static_cast<int>(gridDim.x + atomicAdd(a.unit_next, 1u));
      u = __shfl_sync(0xFFFFFFFFu, v, 0);
    }
    // every copy this warp started has landed before the CTA may exit
    for (int d = 1; d <= S && d <= it; ++d) {
      const int j = it - d;
      mbar_wait(bar_full + 8 * (j % S), (j / S) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------ MMA issuer ----------------------------------
    const uint32_t sf_t0 = tmem + static_cast<uint32_t>(2 * L.ncols);
    int it = 0, uc = 0;
    bool ok = true;
    while (ok) {
      const int s0 = it % S;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s0, (it / S) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&stage_unit[s0]);
      const int buf = uc & 1;
      if (uc >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_acce + 8 * buf, ((uc >> 1) & 1) ^ 1, a.status))) break;
      if (lane == 0) {
        acc_unit[buf] = u;
        mbar_arrive(bar_accf + 8 * buf);
        if (u < 0) mbar_arrive(bar_accf + 8 * buf);
      }
      __syncwarp();
      if (u < 0) break;
      tc::fence_after_sync();
      const BsUnit un = bs_unit_of(u, cnt, off, pre, gpre, E, tiles, L.ntok_cap);
      const uint32_t N = static_cast<uint32_t>((2 * un.ntok + 15) & ~15);
      const uint32_t idesc = tc::idesc_mxf8f6f4(5u, 0u, 128u, N);
      const uint32_t d0 = tmem + static_cast<uint32_t>(buf * L.ncols);
      for (int c = 0; c < nk; ++c, ++it) {
        const int s = it % S;
        if (c > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s, (it / S) & 1, a.status))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (lane == 0) {
          const uint32_t st = sbase + s * stg;
          const uint32_t sf = st + sf_off;
          const uint32_t t0 = sf_t0 + s * kSfCols;
          tc::cp_sf_32x128b_x4(t0, tc::desc_k_interleave(sf));
          tc::cp_sf_32x128b_x4(t0 + 4, tc::desc_k_interleave(sf + 512));
          if (N > 128) tc::cp_sf_32x128b_x4(t0 + 8, tc::desc_k_interleave(sf + 1024));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc::mma_mxf8f6f4(d0, tc::desc_k_sw128(st + 32 * j), tc::desc_k_sw128(st + b_off + 32 * j), idesc, t0,
                             t0 + 4, static_cast<uint32_t>(j), static_cast<uint32_t>((c | j) != 0));
          tc::commit(bar_empty + 8 * s);
          if (c == nk - 1) tc::commit(bar_accf + 8 * buf);
        }
        __syncwarp();
      }
      ++uc;
    }
    // all MMAs of this thread complete before TMEM is released
    if (lane == 0) tc::commit(bar_final);
    __syncwarp();
    mbar_wait(bar_final, 0, a.status);
  } else {
    // ------------------------------------ epilogue -------------------------------------
    const int q = warp & 3;                    // TMEM lane quadrant this warp may access
    const int row = 32 * q + lane;             // accumulator row = row of the weight tile
    float* xch = reinterpret_cast<float*>(smem + L.xch_off);   // [2][64][8]: up values for the gate warps
    int uc = 0;
    while (true) {
      const int buf = uc & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar_accf + 8 * buf, (uc >> 1) & 1, a.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&acc_unit[buf]);
      if (u < 0) break;
      tc::fence_after_sync();
      const BsUnit un = bs_unit_of(u, cnt, off, pre, gpre, E, tiles, L.ntok_cap);
      const uint32_t d0 =
          tmem + static_cast<uint32_t>(buf * L.ncols) + (static_cast<uint32_t>(32 * q) << 16);
      const int N = (2 * un.ntok + 15) & ~15;
      if (kEpi == kEpiSwiglu) {
        // rows 0-63 gate, 64-127 up of intermediate indices tile*64 + (row & 63)
        const int64_t col = static_cast<int64_t>(un.tile) * 64 + (row & 63);
        uint8_t* hat = a.h_atoms + (static_cast<int64_t>(un.gid) * (a.inter / 128) + (col >> 7)) * 1024 +
                       ((col & 127) >> 5);
        for (int c0 = 0; c0 < N; c0 += 16) {
          float* xb = xch + ((c0 >> 4) & 1) * (64 * 8);
          uint32_t v[16];
          tc::ld_32x32b_x16(d0 + static_cast<uint32_t>(c0), v);
          tc::ld_wait();
          if (q >= 2) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              xb[(row - 64) * 8 + j] = __uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1]);
          }
          epi_bar_sync();
          if (q < 2) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int i = (c0 >> 1) + j;
              const float g = fminf(__uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1]), a.limit);
              const float uu = fminf(fmaxf(xb[row * 8 + j], -a.limit), a.limit);
              const float hv = __fdividef(g, 1.0f + __expf(-g)) * uu;
              uint32_t q1, q2, s1, s2;
              warp_split2(hv, q1, q2, s1, s2);
              if (i < un.ntok) {
                const int64_t r0 = 2 * (static_cast<int64_t>(un.slot0) + i);
                a.hq[r0 * a.inter + col] = static_cast<uint8_t>(q1);
                a.hq[(r0 + 1) * a.inter + col] = static_cast<uint8_t>(q2);
                if (lane == 0) {
                  hat[sf_row_off2(2 * i)] = static_cast<uint8_t>(s1);
                  hat[sf_row_off2(2 * i + 1)] = static_cast<uint8_t>(s2);
                }
              }
            }
          }
        }
      } else {
        // gate weights of the unit's tokens (ntok <= 128): lane l holds slots l, 32+l, 64+l, 96+l
        float wl[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int i = lane + 32 * m;
          wl[m] = (i < un.ntok) ? a.gw[a.perm[un.slot0 + i]] : 0.f;
        }
        float* o0 = a.o_out + static_cast<int64_t>(un.slot0) * a.ldo + static_cast<int64_t>(un.tile) * 128 + row;
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t v[16];
          tc::ld_32x32b_x16(d0 + static_cast<uint32_t>(c0), v);
          tc::ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = (c0 >> 1) + j;
            const float wsel = (i < 32) ? wl[0] : (i < 64) ? wl[1] : (i < 96) ? wl[2] : wl[3];
            const float wgt = __shfl_sync(0xFFFFFFFFu, wsel, i & 31);
            if (i < un.ntok) o0[static_cast<int64_t>(i) * a.ldo] = (__uint_as_float(v[2 * j]) + __uint_as_float(v[2 * j + 1])) * wgt;
          }
        }
      }
      tc::fence_before_sync();
      epi_bar_sync();
      if (lane == 0) mbar_arrive(bar_acce + 8 * buf);
      ++uc;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, static_cast<uint32_t>(L.tmem_cols));
  }
  if (threadIdx.x == 0) slot_end(a.slot);
}

constexpr int kBsSmemLimit = 227 * 1024;

bool bs_layout(int T, int E, BsLayout* L) {
  L->ntok_cap = std::min(kMaxTokCap, (T + 7) / 8 * 8);
  L->ncols = (2 * L->ntok_cap + 15) / 16 * 16;
  L->stage_bytes = static_cast<int>(align_up(static_cast<size_t>(kATile + L->ncols * kKT + kSfBytes), 1024));
  // fixed part (after the stages): exchange buffer, per-expert tables, barriers
  int off = 0;
  const int x0 = off;
  off += 2 * 64 * 8 * 4;
  const int c0 = off;
  off += 4 * (E + 1);
  const int o0 = off;
  off += 4 * (E + 1);
  const int p0 = off;
  off += 4 * (E + 1);
  const int g0 = off;
  off += 4 * (E + 1);
  off = static_cast<int>(align_up(off, 16));
  const int b0 = off;
  off += 8 * (2 * kBsMaxStages + 5) + 8 + 4 * (kBsMaxStages + 2);
  const int fixed = static_cast<int>(align_up(off, 16));
  // narrow units (few tokens per expert) leave the tensor pipe idle between stages: two
  // CTAs per SM, each with half the shared memory and TMEM, keep two pipelines in flight
  L->ctas_per_sm = (L->ncols <= 32) ? 3 : ((L->ncols <= 64) ? 2 : 1);
  const int smem_limit = (L->ctas_per_sm == 3) ? 74 * 1024 : ((L->ctas_per_sm == 2) ? 112 * 1024 : kBsSmemLimit);
  int S = (smem_limit - 1024 - fixed) / L->stage_bytes;
  S = std::min(S, kBsMaxStages);
  // each CTA's allocation (a power of two) must leave room for the others on the SM
  const int tmem_share = (L->ctas_per_sm == 3) ? 128 : 512 / L->ctas_per_sm;
  while (S > 0 && 2 * L->ncols + kSfCols * S > tmem_share) --S;
  if (S < 2) return false;
  L->stages = S;
  const int body = S * L->stage_bytes;
  L->xch_off = body + x0;
  L->cnt_off = body + c0;
  L->off_off = body + o0;
  L->pre_off = body + p0;
  L->gpre_off = body + g0;
  L->bar_off = body + b0;
  L->smem_bytes = body + fixed + 1024;      // + slack for the 1024-byte alignment of the base
  const int need = 2 * L->ncols + kSfCols * S;
  int cols = 32;
  while (cols < need) cols *= 2;
  L->tmem_cols = cols;
  return true;
}

}  // namespace

fp4_status launch_split_x(const uint16_t* x, const int32_t* inv, const int32_t* counts, const int32_t* offsets,
                          int E, int k, int P, int H, int ntok_cap, uint8_t* q, uint8_t* atoms, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(P / k) * (H / 32);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, num_sms() * 16)));
  return launch_pdl(split_x_kernel, dim3(grid), dim3(256), 0, st, true, x, inv, counts, offsets, E, k, P, H,
                    ntok_cap, q, atoms);
}

fp4_status launch_route_split(const float* logits, int T, int E, int k, const uint16_t* x, int H, int ntok_cap,
                              int32_t* ids, float* gw, int32_t* counts, int32_t* offsets, int32_t* perm,
                              int32_t* inv, uint8_t* q, uint8_t* atoms, cudaStream_t st) {
  if (T * k > kRouteMaxPairs || E > kRouteMaxExperts) return FP4_ERR_UNSUPPORTED;
  const int64_t total = static_cast<int64_t>(T) * k * (H / 32);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((total + 511) / 512, num_sms())));
  return launch_pdl(route_split_kernel, dim3(grid), dim3(512), 0, st, true, logits, T, E, k, x, H, ntok_cap, ids, gw,
                    counts, offsets, perm, inv, q, atoms);
}

fp4_status launch_mma_scales(const uint8_t* scales, int64_t rows, int64_t K, int64_t pair, uint8_t* atoms,
                             cudaStream_t st) {
  const int64_t total = rows * (K / 128);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, num_sms() * 16)));
  mma_scales_kernel<<<grid, 256, 0, st>>>(scales, rows, K, pair, atoms);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch();
  return FP4_OK;
}

int bs_ntok_cap(int T, int E) {
  BsLayout L;
  return bs_layout(T, E, &L) ? L.ntok_cap : 0;
}

size_t bs_group_atom_bytes(int P, int E, int ntok_cap, int K) {
  const size_t groups = static_cast<size_t>(P) / ntok_cap + E + 1;   // >= sum over experts of ceil(n_e / cap)
  return groups * (K / 128) * 1024;
}

bool bs_supported(int T, int E, int H, int I) {
  BsLayout L;
  return H % 128 == 0 && I % 128 == 0 && bs_layout(T, E, &L);
}

fp4_status launch_bs(const BsArgs& a, int T, cudaStream_t st) {
  BsLayout L;
  if (!bs_layout(T, a.E, &L) || L.ntok_cap != a.ntok_cap) return FP4_ERR_UNSUPPORTED;
  CUtensorMap mA, mB;
  FP4_TRY(make_tmap_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, a.codes, static_cast<uint64_t>(a.K),
                       static_cast<uint64_t>(a.rows_total), static_cast<uint64_t>(a.K / 2), kKT, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  FP4_TRY(make_tmap_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_q, static_cast<uint64_t>(a.K),
                       static_cast<uint64_t>(2) * a.P, static_cast<uint64_t>(a.K), kKT,
                       static_cast<uint32_t>(L.ncols), CU_TENSOR_MAP_SWIZZLE_128B));
  auto kern = (a.epi == kEpiSwiglu) ? bs_moe_kernel<kEpiSwiglu> : bs_moe_kernel<kEpiDown>;
  static thread_local bool configured[2] = {false, false};
  const int which = (a.epi == kEpiSwiglu) ? 0 : 1;
  if (!configured[which]) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kBsSmemLimit));
    configured[which] = true;
  }
  return launch_pdl(kern, dim3(L.ctas_per_sm * num_sms()), dim3(kBsThreads), static_cast<size_t>(L.smem_bytes), st,
                    true, mA, mB, a, L);
}

}  // namespace fp4

// Grouped W4A16 GEMV on the CUDA cores for decode-sized calls (few tokens per expert, so
// the layer is bound by the weight stream from HBM): NVFP4, CB4, the dense linear layer,
// and MXFP4 when its weights come without the tensor-core scale atoms.
//
// Design (B200): persistent CTAs, two or three per SM, walk work units {expert, 64-row weight
// tile, up to 8 routed tokens}.  One producer warp streams a unit's 4-bit codes with TMA
// (128-byte swizzled boxes, conflict-free for the fragment reads), its scale bytes with
// 4-byte async copies and the f16 activation rows with 1D bulk copies into a shared-
// memory ring guarded by mbarriers.  Eight consumer warps (32 rows x a quarter of the
// stage's K each) dequantise in registers -- E2M1 pairs -> f16x2 with the sm_100
// conversion instruction; NVFP4 E4M3 block scales folded into the f16 operand (exact);
// MXFP4 power-of-two scales applied per 32-block to fp32 partial sums -- and accumulate
// with warp-level f16 MMAs into fp32.  The four K quarters meet in shared memory in a
// fixed order and a fused epilogue writes the SwiGLU-with-clamp activation (gate_up),
// the gate-weighted expert output (down) or y (dense layer).
//
// CB4 ("XFP：质量地板驱动的自适应码本量化", V2 dense + sparse): the 4-bit indices stream
// like E2M1 codes; each row's fp16 codebooks for the stage arrive by one bulk copy; a
// warp looks entries up in registers (low and high byte tables of the 16 entries,
// byte-permute selection) and the CSR outlier term joins in the epilogue.
//
// In kModeRoute the gate_up kernel also finishes the router in its prologue: every CTA
// takes the top-k of the logits, the per-expert counts and the stable permutation into
// shared memory (CTA 0 also stores them for the later kernels), so no separate launch
// sits between the logits and the weight stream.
//
// The per-element unpack-and-scale work is the cost the MXFP4 serving campaign measured
// as a constant overhead per weight element ("The gate that missed by 0.0202 pp",
// section "Serving throughput"); here it runs in registers beside the HBM stream.
#include <algorithm>

#include "kernels.cuh"
#include "routing.cuh"

namespace fp4 {
namespace {

constexpr int kRows = 64;                 // weight rows per unit
constexpr int kTok = 8;                   // tokens per unit (one n8 MMA tile); NVFP4 may use 16
constexpr int kConsumers = 8;             // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kMaxStages = 8;
// CTAs per SM: stages 512 K wide run two per SM (110 KB of shared memory each), 256 K
// wide ones three (73 KB each, at most 72 registers a thread)
constexpr int ctas_per_sm(int kc) { return kc == 256 ? 3 : 2; }
constexpr int smem_budget(int kc) { return kc == 256 ? 73 * 1024 : 110 * 1024; }

struct Layout {
  int kc;            // K elements per stage
  int nchunks;       // K / kc
  int scale_row;     // scale bytes per row per stage
  int codes_off, scales_off, x_off;
  int x_row;         // bytes per token row in the stage (padded)
  int stage_bytes;
  int stages;
  int red_off;       // 4 x [64][tokens per unit + 1] fp32 (one per K quarter)
  int su_off;        // [kMaxStages] int: work unit of each ring stage
  int lut_off;       // 256 fp32 (UE8M0 -> float)
  int cnt_off, off_off, pre_off;   // [E + 1] int each (pre is followed by [E] cursors)
  int perm_off;      // [P] int (kModeRoute)
  int scl_off;       // [scl_n] float: per-slot epilogue factor (2^sexp or gate weight)
  int scl_n;         // slots with a preloaded factor (0: read per unit from global memory)
  int bar_off;
  int smem_bytes;
};

__device__ __forceinline__ void named_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

struct Unit {
  int e, tile, slot0, ntok;
  int ks;            // dense layer split over K: which share of the chunks (else 0)
};

// Exclusive scans by warp 0 over E experts: off = scan(cnt), pre = scan(units per expert),
// where only the experts in [e_lo, e_hi) (those whose weights the call holds) have units.
// In a mixed-format buffer (ex_fmt non-null) only the experts of format `want` have units.
template <int kT>
__device__ void scan_experts(const int* cnt, int* off, int* pre, int E, int tiles, int e_lo, int e_hi,
                             const uint8_t* ex_fmt, int want) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 31) / 32;
  const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
  auto units = [&](int e) {
    const bool mine = e >= e_lo && e < e_hi && (ex_fmt == nullptr || ex_fmt[e - e_lo] == want);
    return mine ? (cnt[e] + kT - 1) / kT * tiles : 0;
  };
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
  if (lane == 31) {
    off[E] = ic;
    pre[E] = iu;
  }
}

// unit u -> {expert, tile, first slot, tokens}; units are ordered by expert, tile, group
template <int kT>
__device__ __forceinline__ Unit unit_of(int u, const int* cnt, const int* off, const int* pre, int E,
                                        int tiles) {
  int lo = 0, hi = E - 1;          // largest e with pre[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid - 1;
  }
  Unit un;
  un.e = lo;
  const int n = cnt[lo];
  const int groups = (n + kT - 1) / kT;
  const int local = u - pre[lo];
  un.tile = local / groups;
  const int grp = local - un.tile * groups;
  un.slot0 = off[lo] + grp * kT;
  un.ntok = min(kT, n - grp * kT);
  un.ks = 0;
  return un;
}

// dense layer: unit u -> {K share u % ksplit, tile, token group}
__device__ __forceinline__ Unit unit_static(int u, int tiles, int T, int ksplit) {
  Unit un;
  un.e = 0;
  un.ks = u % ksplit;
  const int ub = u / ksplit;
  un.tile = ub % tiles;
  un.slot0 = (ub / tiles) * kTok;
  un.ntok = min(kTok, T - un.slot0);
  return un;
}

// row of the expert's matrix that row r (0..63) of a unit reads
template <int kEpi>
__device__ __forceinline__ int64_t tile_row(const DecodeArgs& a, const Unit& un, int r) {
  if (kEpi == kEpiSwiglu) return r < 32 ? un.tile * 32 + r : a.inter + un.tile * 32 + (r - 32);
  return static_cast<int64_t>(un.tile) * kRows + r;
}
// first code row and first scale row of the unit's expert (rows of K/2 code bytes and of
// the per-row scale bytes): uniform buffers stack the local experts; mixed-format buffers
// give each expert's byte offsets
struct RowBase {
  int64_t code, scale;
};
template <int kFmt>
__device__ __forceinline__ RowBase unit_base(const DecodeArgs& a, const Unit& un) {
  const int le = un.e - a.e_begin;
  if (a.row_off == nullptr) {
    const int64_t b = static_cast<int64_t>(le) * a.rows_per_expert;
    return {b, b};
  }
  constexpr int kB = (kFmt == FP4_MXFP4) ? 32 : 16;
  return {a.row_off[le] / (a.K / 2), a.srow_off[le] / (a.K / kB)};
}
template <int kEpi>
__device__ __forceinline__ int64_t unit_row(const DecodeArgs& a, const Unit& un, int r) {
  return static_cast<int64_t>(un.e - a.e_begin) * a.rows_per_expert + tile_row<kEpi>(a, un, r);   // local expert
}

// CB4: eight 4-bit indices (low nibble first) -> four f16x2 registers of codebook
// entries, from byte tables lo[q] / hi[q] holding the low / high bytes of entries
// 4q .. 4q+3.  Byte-permute selects with the low three index bits among entries 0-7 and
// 8-15; a mask made by sign-replicating each index's bit 3 picks between the two.
// PTX prmt in its default mode: a selector nibble with bit 3 set replicates the sign bit
// of the selected byte over the whole result byte (the CUDA intrinsic __byte_perm only
// defines the low three selector bits).
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ void cb4_lookup8(uint32_t w, const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                                            uint32_t (&h)[4]) {
  // bit 3 of every index at a byte's top bit: even nibbles in w << 4, odd ones in w; one
  // sign-replicating byte-permute per half turns them into the select masks (byte i =
  // 0xFF where index i of the half is >= 8)
  const uint32_t ws = w << 4;
  const uint32_t msks[2] = {prmt_sx(ws, w, 0xD9C8u), prmt_sx(ws, w, 0xFBEAu)};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t v = half ? (w >> 16) : w;
    const uint32_t sel = v & 0x7777u;
    const uint32_t msk = msks[half];
    const uint32_t la = __byte_perm(lo[0], lo[1], sel), lb = __byte_perm(lo[2], lo[3], sel);
    const uint32_t ha = __byte_perm(hi[0], hi[1], sel), hb = __byte_perm(hi[2], hi[3], sel);
    const uint32_t L = (la & ~msk) | (lb & msk), H = (ha & ~msk) | (hb & msk);
    h[2 * half] = __byte_perm(L, H, 0x5140);
    h[2 * half + 1] = __byte_perm(L, H, 0x7362);
  }
}

// bf16x2 -> f16x2 of x 2^n with n split as two power-of-two factors f1 f2 (both exact
// multiplications wherever the f16 result is not zero), rounded to nearest: the same bits as
// converting ldexpf(x, n)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float f1, float f2) {
  const __half2 h = __floats2half2_rn((__uint_as_float(w << 16) * f1) * f2, (__uint_as_float(w & 0xFFFF0000u) * f1) * f2);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int kFmt, int kEpi, int kMode, int KC, int kT>
__global__ void __launch_bounds__(kThreads, ctas_per_sm(KC))
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap smap,
                  const DecodeArgs a, const Layout L) {
  // stage geometry (must match make_layout)
  constexpr bool kCb = (kFmt == FP4_CB4 || kFmt == FP4_V2A);      // codebook lookup formats
  constexpr int kB = (kFmt == FP4_MXFP4) ? 32 : 16;
  // scale bytes per row per stage (CB4: fp16 codebooks; V2a: 8-byte group records)
  constexpr int kScaleRow = (kFmt == FP4_CB4) ? KC / 4 : ((kFmt == FP4_V2A) ? KC / 16 : KC / kB);
  constexpr int kScalesOff = kRows * KC / 2;
  constexpr int kLibOff = kScalesOff + kRows * kScaleRow;           // V2a: the expert's library (1 KB)
  constexpr int kXOff = kLibOff + ((kFmt == FP4_V2A) ? kV2aLibBytes : 0);
  constexpr int kXRow = 2 * KC + 64;                 // padded f16 token row
  constexpr int kNq = KC / 128;                      // 32-K regions per warp per stage
  // tokens per unit: one n8 MMA tile, or two (a second tile for tokens 8-15, skipped for
  // units of at most 8 tokens); the dense layer keeps one
  static_assert(kT == 8 || (kT == 16 && kMode != kModeStatic && kFmt == FP4_NVFP4), "tokens per unit");
  constexpr int kNt = kT / 8;
  constexpr int kPitch = kT + 1;                     // fp32 reduction row pitch
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 128-byte swizzled TMA boxes need 1024-byte aligned destinations
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t bar_full = sbase + L.bar_off;
  const uint32_t bar_empty = bar_full + 8 * kMaxStages;
  constexpr int B = (kFmt == FP4_MXFP4) ? 32 : 16;
  const int tiles = (kEpi == kEpiSwiglu) ? a.inter / 32 : a.rows_per_expert / kRows;
  int* cnt = reinterpret_cast<int*>(smem + L.cnt_off);
  int* off = reinterpret_cast<int*>(smem + L.off_off);
  int* pre = reinterpret_cast<int*>(smem + L.pre_off);
  int* perm_s = reinterpret_cast<int*>(smem + L.perm_off);

  // dense layer with bf16 x (no separate conversion launch): the producer streams the weights
  // before waiting on the previous kernel (they do not depend on it) and the raw bf16 rows
  // after it; the consumers convert the rows to f16 as they read them
  const bool fused_x = kMode == kModeStatic && a.x16 == nullptr;
  __shared__ unsigned int exit_count;
  if (threadIdx.x == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(bar_full + 8 * s, fused_x ? 2 : 1);   // fused: the weight bytes, then the x rows
      mbar_init(bar_empty + 8 * s, kConsumers);
    }
    fence_barrier_init();
    exit_count = 0u;
  }
  if (kFmt == FP4_MXFP4)
    for (int i = threadIdx.x; i < 256; i += kThreads)
      reinterpret_cast<float*>(smem + L.lut_off)[i] = ue8m0_to_f32(static_cast<uint32_t>(i));
  if (warp == kConsumers && lane == 0) {
    prefetch_tmap(&tmap);
    if (a.scale_tma) prefetch_tmap(&smap);
  }
  __syncthreads();
  if (!fused_x) pdl_wait();
  pdl_launch_dependents();
  // (fused dense layer: the producer starts the timer after its dependency wait, when the
  // previous launch -- which may share the workspace -- has finished)
  if (threadIdx.x == 0 && !fused_x) slot_begin(a.slot);
  auto finish = [&]() {   // the last warp of the CTA to leave records the CTA's end time
    if (lane == 0 && atomicAdd(&exit_count, 1u) == kConsumers) slot_end(a.slot);
  };

  // ------------------------------- work units ---------------------------------------
  // dense layer: the K chunks may be split over ksplit units (partial sums, reduced by a
  // second kernel in a fixed order); nck chunks per unit
  const int ksplit = (kMode == kModeStatic && a.ksplit > 1) ? a.ksplit : 1;
  const int nck = L.nchunks / ksplit;
  int n_units;
  if (kMode == kModeStatic) {
    n_units = tiles * ((a.T + kTok - 1) / kTok) * ksplit;
  } else {
    const int E = a.E;
    if (kMode == kModeRoute) {
      const int P = a.T * a.topk;
      int* ids_s = reinterpret_cast<int*>(smem);       // scratch in the (still unused) stage ring
      for (int t = warp; t < a.T; t += kConsumers + 1)
        topk_warp(a.logits + static_cast<int64_t>(t) * E, E, a.topk, ids_s + t * a.topk,
                  blockIdx.x == 0 ? a.gw + static_cast<int64_t>(t) * a.topk : nullptr);
      for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = 0;
      __syncthreads();
      for (int p = threadIdx.x; p < P; p += kThreads) {
        atomicAdd(&cnt[ids_s[p]], 1);
        if (blockIdx.x == 0) a.ids[p] = ids_s[p];
      }
      __syncthreads();
      if (warp == 0) {
        scan_experts<kT>(cnt, off, pre, E, tiles, a.e_begin, a.e_end, a.ex_fmt, kFmt);
        __syncwarp();
        // stable placement: pairs in ascending order, 32 per round, ranked within the round
        int* cur = pre + E + 1;                      // [E] cursors
        for (int e = lane; e < E; e += 32) cur[e] = off[e];
        __syncwarp();
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
              a.perm[slot] = p;
              a.inv[p] = slot;
            }
          }
        }
      }
      __syncthreads();
      if (blockIdx.x == 0)
        for (int e = threadIdx.x; e <= E; e += kThreads) {
          if (e < E) a.counts[e] = cnt[e];
          a.offsets[e] = off[e];
        }
    } else {
      for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = a.counts[e];
      __syncthreads();
      if (warp == 0) scan_experts<kT>(cnt, off, pre, E, tiles, a.e_begin, a.e_end, a.ex_fmt, kFmt);
      __syncthreads();
    }
    n_units = pre[E];
  }
  auto get_unit = [&](int u) -> Unit {
    if (kMode == kModeStatic) return unit_static(u, tiles, a.T, ksplit);
    return unit_of<kT>(u, cnt, off, pre, a.E, tiles);
  };
  auto perm_at = [&](int slot) -> int {
    if (kMode == kModeRoute) return perm_s[slot];
    return a.perm[slot];
  };
  constexpr int ncb = KC / 256;                                // 128-byte code boxes per row per stage
  int* stage_unit = reinterpret_cast<int*>(smem + L.su_off);
  // work units: the first is blockIdx.x, later ones come from a counter (zeroed by the router)
  auto next_unit = [&](int u) -> int {
    if (kMode == kModeStatic || a.unit_next == nullptr) return u + static_cast<int>(gridDim.x);
    int v = 0;
    if (lane == 0) v = static_cast<int>(gridDim.x + atomicAdd(a.unit_next, 1u));
    return __shfl_sync(0xFFFFFFFFu, v, 0);
  };

  if (kMode == kModeStatic && warp == kConsumers && fused_x) {
    // ------------------------- producer, dense layer with bf16 x ----------------------
    const bool stma = a.scale_tma != 0;
    constexpr int words = kScaleRow / 4;
    const uint32_t wtx = static_cast<uint32_t>(kRows * (KC / 2) + (stma ? kRows * kScaleRow : 0));
    const int S = L.stages;
    int it = 0;
    bool ok = true, waited = false;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit un = get_unit(u);
      const RowBase rb0 = unit_base<kFmt>(a, un);
      const int64_t y0 = rb0.code + tile_row<kEpi>(a, un, 0), y1 = rb0.code + tile_row<kEpi>(a, un, 32);
      const int64_t sy0 = rb0.scale + tile_row<kEpi>(a, un, 0), sy1 = rb0.scale + tile_row<kEpi>(a, un, 32);
      const int it0 = it;
      int cw = 0;
      const int cb0 = un.ks * nck;               // first chunk of the unit's K share
      for (int cx = 0; cx < nck && ok; ++cx) {
        // weights up to `stages` chunks ahead of the activation rows
        while (cw < nck && cw < cx + S) {
          const int iw = it0 + cw, s = iw % S;
          if (iw >= S && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((iw / S) & 1) ^ 1, a.status))) {
            ok = false;
            break;
          }
          if (lane == 0) stage_unit[s] = u;
          const uint32_t st_base = sbase + s * L.stage_bytes;
          const int k0 = (cb0 + cw) * KC;
          if (!stma) {
            for (int w = lane; w < kRows * words; w += 32) {
              const int r = w / words, cwd = w - r * words;
              cp_async4(st_base + kScalesOff + r * kScaleRow + cwd * 4,
                        a.scales + (rb0.scale + tile_row<kEpi>(a, un, r)) * (a.K / B) + k0 / B + cwd * 4);
            }
            cp_async_arrive(bar_full + 8 * s);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, wtx);
          __syncwarp();
          if (stma && lane == 0) {
            const int32_t sx = k0 / (KC / kScaleRow);
            tma_load_2d(st_base + kScalesOff, &smap, sx, static_cast<int32_t>(sy0), bar_full + 8 * s);
            tma_load_2d(st_base + kScalesOff + 32 * kScaleRow, &smap, sx, static_cast<int32_t>(sy1), bar_full + 8 * s);
          }
          for (int q = lane; q < 2 * ncb; q += 32) {
            const int rb = q & 1, cb = q >> 1;
            tma_load_2d(st_base + (cb * kRows + rb * 32) * 128, &tmap, k0 / 2 + cb * 128,
                        static_cast<int32_t>(rb ? y1 : y0), bar_full + 8 * s);
          }
          ++cw;
        }
        if (!ok) break;
        if (!waited) {
          pdl_wait();                 // x may come from the previous kernel
          waited = true;
          if (lane == 0) {
            if (blockIdx.x == 0) *a.status = 0u;   // this call's status word
            slot_begin(a.slot);
          }
        }
        // the chunk's raw bf16 activation rows into the stage (the consumers convert them)
        const int s = (it0 + cx) % S;
        if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, static_cast<uint32_t>(un.ntok * KC * 2));
        __syncwarp();
        if (lane < un.ntok)
          bulk_g2s(sbase + s * L.stage_bytes + kXOff + lane * kXRow,
                   a.x_bf16 + static_cast<int64_t>(un.slot0 + lane) * a.K + (cb0 + cx) * KC,
                   static_cast<uint32_t>(KC * 2), bar_full + 8 * s);
      }
      it = it0 + nck;
    }
    if (ok) {
      // sentinel stage: no more work for this CTA (both arrivals)
      const int s = it % S;
      if (it < S || __all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((it / S) & 1) ^ 1, a.status))) {
        if (lane == 0) {
          stage_unit[s] = -1;
          mbar_arrive(bar_full + 8 * s);
          mbar_arrive(bar_full + 8 * s);
        }
        ++it;
      }
    }
    if (!waited) {
      pdl_wait();
      if (lane == 0) {
        if (blockIdx.x == 0) *a.status = 0u;
        slot_begin(a.slot);
      }
    }
    for (int d = 1; d <= S && d <= it; ++d) {
      const int j = it - d;
      mbar_wait(bar_full + 8 * (j % S), (j / S) & 1, a.status);
    }
    finish();
    return;
  }

  if (warp == kConsumers) {
    // ------------------------------- producer -------------------------------------
    int it = 0;
    bool ok = true;
    int u = blockIdx.x;
    const bool stma = a.scale_tma != 0;   // the per-row scale bytes arrive as two TMA boxes
    while (true) {
      if (u >= n_units) {
        // sentinel stage: no more work for this CTA
        const int s = it % L.stages;
        if (it >= L.stages &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((it / L.stages) & 1) ^ 1, a.status)))
          break;
        if (lane == 0) {
          stage_unit[s] = -1;
          mbar_arrive(bar_full + 8 * s);
        }
        ++it;
        break;
      }
      const Unit un = get_unit(u);
      const RowBase rb0 = unit_base<kFmt>(a, un);
      const int64_t y0 = rb0.code + tile_row<kEpi>(a, un, 0), y1 = rb0.code + tile_row<kEpi>(a, un, 32);
      const int64_t sy0 = rb0.scale + tile_row<kEpi>(a, un, 0), sy1 = rb0.scale + tile_row<kEpi>(a, un, 32);
      int xr = 0;
      if (lane < un.ntok) xr = (kEpi == kEpiSwiglu) ? perm_at(un.slot0 + lane) / a.topk : un.slot0 + lane;
      const uint32_t tx = static_cast<uint32_t>(kRows * (KC / 2) + un.ntok * KC * 2 +
                                                ((kCb || stma) ? kRows * kScaleRow : 0) +
                                                (kFmt == FP4_V2A ? kV2aLibBytes : 0));
      constexpr int words = kScaleRow / 4;
      for (int c = 0; c < nck; ++c, ++it) {
        const int s = it % L.stages;
        if (it >= L.stages &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(bar_empty + 8 * s, ((it / L.stages) & 1) ^ 1, a.status))) {
          ok = false;
          break;
        }
        if (lane == 0) stage_unit[s] = u;
        const uint32_t st_base = sbase + s * L.stage_bytes;
        const int k0 = (un.ks * nck + c) * KC;
        if (!kCb && !stma) {
          for (int w = lane; w < kRows * words; w += 32) {
            const int r = w / words, cw = w - r * words;
            const uint8_t* src = a.scales + (rb0.scale + tile_row<kEpi>(a, un, r)) * (a.K / B) + k0 / B + cw * 4;
            cp_async4(st_base + kScalesOff + r * kScaleRow + cw * 4, src);
          }
          cp_async_arrive(bar_full + 8 * s);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(bar_full + 8 * s, tx);
        __syncwarp();
        if (stma) {
          // rows 0-31 and 32-63 of the unit (gate_up: the gate and the up block) as two boxes
          if (lane == 0) {
            const int32_t sx = k0 / (KC / kScaleRow);
            tma_load_2d(st_base + kScalesOff, &smap, sx, static_cast<int32_t>(sy0), bar_full + 8 * s);
            tma_load_2d(st_base + kScalesOff + 32 * kScaleRow, &smap, sx, static_cast<int32_t>(sy1), bar_full + 8 * s);
          }
        } else if (kCb)
          for (int r = lane; r < kRows; r += 32)
            bulk_g2s(st_base + kScalesOff + r * kScaleRow,
                     a.scales + (rb0.scale + tile_row<kEpi>(a, un, r)) * (a.K / (KC / kScaleRow)) + k0 / (KC / kScaleRow),
                     static_cast<uint32_t>(kScaleRow), bar_full + 8 * s);
        if (kFmt == FP4_V2A && lane == 0)
          bulk_g2s(st_base + kLibOff, a.lib + static_cast<int64_t>(un.e - a.e_begin) * kV2aLibBytes, kV2aLibBytes,
                   bar_full + 8 * s);
        for (int q = lane; q < 2 * ncb; q += 32) {
          const int rb = q & 1, cb = q >> 1;
          tma_load_2d(st_base + (cb * kRows + rb * 32) * 128, &tmap, k0 / 2 + cb * 128,
                      static_cast<int32_t>(rb ? y1 : y0), bar_full + 8 * s);
        }
        if (lane < un.ntok)
          bulk_g2s(st_base + kXOff + lane * kXRow, a.x16 + static_cast<int64_t>(xr) * a.K + k0,
                   static_cast<uint32_t>(KC * 2), bar_full + 8 * s);
      }
      if (!ok) break;
      u = next_unit(u);
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
  const int rh = warp & 1, kq = warp >> 1;
  const int g = lane >> 2, t = lane & 3;
  const int rbase = 32 * rh + g;                 // rows rbase + 8m, m = 0..3
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  const float* lut_f = reinterpret_cast<const float*>(smem + L.lut_off);
  const int jbase = kq * kNq;                    // this warp's first 32-K region of a stage
  // per-thread offsets within a stage: codes (swizzled 128-byte rows), scales, activations
  const uint32_t c_off = ((jbase >> 3) * kRows + rbase) * 128 + 4 * t;
  uint32_t c_xo[kNq];
#pragma unroll
  for (int jj = 0; jj < kNq; ++jj) c_xo[jj] = static_cast<uint32_t>((((jbase & 7) + jj) ^ g) << 4);
  // NVFP4: byte-permute selectors taking scale byte b of two rows' words into bytes 0, 1
  // (b = t / 2 for even regions, 2 + t / 2 for odd ones)
  const uint32_t nv_sel[2] = {static_cast<uint32_t>((t >> 1) | ((4 + (t >> 1)) << 4)),
                              static_cast<uint32_t>((2 + (t >> 1)) | ((6 + (t >> 1)) << 4))};
  const uint32_t s_off = kScalesOff + rbase * kScaleRow +
                         (kFmt == FP4_MXFP4 ? jbase
                                            : (kFmt == FP4_NVFP4 ? 2 * jbase : (jbase >> 2) * (kFmt == FP4_CB4 ? 32 : 8)));
  const uint32_t x_off = kXOff + g * kXRow + t * 16 + jbase * 64;
  // per-slot epilogue factors, loaded once so no unit's epilogue waits on global memory
  float* scl_s = reinterpret_cast<float*>(smem + L.scl_off);
  if (L.scl_n > 0 && !fused_x) {      // (fused dense layer: written at each unit's start)
    for (int i = threadIdx.x; i < L.scl_n; i += kConsumers * 32) {
      float v;
      if (kEpi == kEpiSwiglu) v = ldexpf(1.0f, a.sexp[perm_at(i) / a.topk]);
      else if (kEpi == kEpiDown) v = a.gw[perm_at(i)];
      else v = ldexpf(1.0f, a.sexp[i]);
      scl_s[i] = v;
    }
    named_bar_sync();
  }
  // fused dense layer: the stages hold raw bf16 rows, converted here to f16 x 2^-s_t with
  // the per-token power of two of x_to_f16_kernel (max|x_t| 2^-s_t in [2^14, 2^15)), which
  // each unit finds first (warp i scans token i of the unit)
  __shared__ int xs_s[kTok];
  if (fused_x) pdl_wait();
  int it = 0;
  while (true) {
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * (it % L.stages), (it / L.stages) & 1, a.status))) {
      finish();
      return;
    }
    const int u = *reinterpret_cast<volatile int*>(&stage_unit[it % L.stages]);
    if (u < 0) break;                              // sentinel: no more work
    const Unit un = get_unit(u);
    const float ts = (kFmt == FP4_NVFP4) ? a.tscale[un.e - a.e_begin] : 1.0f;   // used after the K loop
    float xf1 = 1.0f, xf2 = 1.0f;                  // this thread's token (g): x16 = (x f1) f2
    if (kMode == kModeStatic && fused_x) {
      int sx = 0;
      if (warp < un.ntok) {
        const uint16_t* xr = a.x_bf16 + static_cast<int64_t>(un.slot0 + warp) * a.K;
        float amax = 0.f;
#pragma unroll 4
        for (int h = lane * 8; h < a.K; h += 256) {
          const uint4 v = *reinterpret_cast<const uint4*>(xr + h);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[j] << 16)), fabsf(__uint_as_float(w4[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (amax > 0.f && isfinite(amax)) {
          int e;
          frexpf(amax, &e);
          sx = (e - 1) - 14;
        }
        if (lane == 0) scl_s[un.slot0 + warp] = ldexpf(1.0f, sx);
      }
      if (lane == 0) xs_s[warp] = sx;
      named_bar_sync();
      const int n = -xs_s[g];                      // in [-113, 147] for finite bf16 rows
      const int n1 = min(n, 127);
      xf1 = __uint_as_float(static_cast<uint32_t>(n1 + 127) << 23);
      xf2 = __uint_as_float(static_cast<uint32_t>(n - n1 + 127) << 23);
    }
    float acc[kNt][2][4];
#pragma unroll
    for (int nt = 0; nt < kNt; ++nt)
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][m][q] = 0.f;
    const int nt_used = (un.ntok > 8) ? kNt : 1;     // n8 tiles this unit needs (uniform)
    for (int c = 0; c < nck; ++c, ++it) {
      const int s = it % L.stages;
      if (c > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(bar_full + 8 * s, (it / L.stages) & 1, a.status))) {
        finish();
        return;
      }
      // plain shared-memory loads (ordered after the barrier wait, free to be scheduled)
      const uint8_t* stp = smem + s * L.stage_bytes;
      // scale bytes of this warp's regions, one load per row
      uint32_t sb[4][(kFmt == FP4_MXFP4) ? 1 : 2];
      // CB4: byte tables of the 16 fp16 entries of each of the warp's rows (one group)
      uint32_t tlo[4][4], thi[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint8_t* sp = stp + s_off + m * 8 * kScaleRow;
        if (kCb) {
          uint4 c0, c1;
          if (kFmt == FP4_CB4) {
            c0 = *reinterpret_cast<const uint4*>(sp);
            c1 = *reinterpret_cast<const uint4*>(sp + 16);
          } else {
            // V2a: the group's entries are fp16(mid + scale * library entry), one rounding each
            const uint2 rec = *reinterpret_cast<const uint2*>(sp);
            const uint8_t* lrow = stp + kLibOff + (rec.y & 31u) * 32;
            const uint4 l0 = *reinterpret_cast<const uint4*>(lrow), l1 = *reinterpret_cast<const uint4*>(lrow + 16);
            const uint32_t mid2 = __byte_perm(rec.x, 0u, 0x1010), sc2 = __byte_perm(rec.x, 0u, 0x3232);
            c0 = make_uint4(hfma2(l0.x, sc2, mid2), hfma2(l0.y, sc2, mid2), hfma2(l0.z, sc2, mid2),
                            hfma2(l0.w, sc2, mid2));
            c1 = make_uint4(hfma2(l1.x, sc2, mid2), hfma2(l1.y, sc2, mid2), hfma2(l1.z, sc2, mid2),
                            hfma2(l1.w, sc2, mid2));
          }
          const uint32_t e[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tlo[m][q] = __byte_perm(e[2 * q], e[2 * q + 1], 0x6420);
            thi[m][q] = __byte_perm(e[2 * q], e[2 * q + 1], 0x7531);
          }
          sb[m][0] = 0u;
        } else if (kFmt == FP4_MXFP4) {
          static_assert(kFmt != FP4_MXFP4 || kNq <= 4, "scale word");
          sb[m][0] = (kNq == 4) ? *reinterpret_cast<const uint32_t*>(sp) : *reinterpret_cast<const uint16_t*>(sp);
        } else if (kNq == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(sp);      // 2 kNq = 8 bytes
          sb[m][0] = v.x;
          sb[m][(kFmt == FP4_MXFP4) ? 0 : 1] = v.y;
        } else {
          sb[m][0] = *reinterpret_cast<const uint32_t*>(sp);        // 2 kNq = 4 bytes
          sb[m][(kFmt == FP4_MXFP4) ? 0 : 1] = 0u;
        }
      }
#pragma unroll
      for (int jj = 0; jj < kNq; ++jj) {
        const uint8_t* cp = stp + c_off + c_xo[jj];
        uint32_t w[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) w[m] = *reinterpret_cast<const uint32_t*>(cp + m * 8 * 128);
        uint32_t p[4][4];
        if (kCb) {
#pragma unroll
          for (int m = 0; m < 4; ++m) cb4_lookup8(w[m], tlo[m], thi[m], p[m]);
        } else {
#pragma unroll
          for (int m = 0; m < 4; ++m) e2m1x8_to_f16x8(w[m], p[m][0], p[m][1], p[m][2], p[m][3]);
        }
        uint4 xq[kNt];
#pragma unroll
        for (int nt = 0; nt < kNt; ++nt)
          if (nt < nt_used) xq[nt] = *reinterpret_cast<const uint4*>(stp + x_off + nt * 8 * kXRow + jj * 64);
        if (kMode == kModeStatic && fused_x)
          xq[0] = make_uint4(bf16x2_to_f16x2(xq[0].x, xf1, xf2), bf16x2_to_f16x2(xq[0].y, xf1, xf2),
                             bf16x2_to_f16x2(xq[0].z, xf1, xf2), bf16x2_to_f16x2(xq[0].w, xf1, xf2));
        if (kCb) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_16816(acc[0][mt], p[2 * mt][0], p[2 * mt + 1][0], p[2 * mt][1], p[2 * mt + 1][1], xq[0].x, xq[0].y);
            mma_16816(acc[0][mt], p[2 * mt][2], p[2 * mt + 1][2], p[2 * mt][3], p[2 * mt + 1][3], xq[0].z, xq[0].w);
          }
        } else if (kFmt == FP4_NVFP4) {
          // this thread's 8 K positions lie in block 2 jj + (t >> 1): byte (2 jj + (t >> 1)) & 3 of
          // word jj / 2 of the row's run; one byte-permute gathers it for two rows at once
          const int wi = (kFmt == FP4_NVFP4) ? (jj >> 1) : 0;
          const uint32_t sel = nv_sel[jj & 1];
          const uint32_t s01 = e4m3x2_to_f16x2(__byte_perm(sb[0][wi], sb[1][wi], sel));
          const uint32_t s23 = e4m3x2_to_f16x2(__byte_perm(sb[2][wi], sb[3][wi], sel));
          const uint32_t sc[4] = {__byte_perm(s01, 0, 0x1010), __byte_perm(s01, 0, 0x3232),
                                  __byte_perm(s23, 0, 0x1010), __byte_perm(s23, 0, 0x3232)};
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int q = 0; q < 4; ++q) p[m][q] = hmul2(p[m][q], sc[m]);
#pragma unroll
          for (int nt = 0; nt < kNt; ++nt) {
            if (nt >= nt_used) break;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              mma_16816(acc[nt][mt], p[2 * mt][0], p[2 * mt + 1][0], p[2 * mt][1], p[2 * mt + 1][1], xq[nt].x,
                        xq[nt].y);
              mma_16816(acc[nt][mt], p[2 * mt][2], p[2 * mt + 1][2], p[2 * mt][3], p[2 * mt + 1][3], xq[nt].z,
                        xq[nt].w);
            }
          }
        } else {
          float f[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) f[m] = lut_f[(sb[m][0] >> (8 * jj)) & 0xFFu];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            float part[4];
            mma_16816_z(part, p[2 * mt][0], p[2 * mt + 1][0], p[2 * mt][1], p[2 * mt + 1][1], xq[0].x, xq[0].y);
            mma_16816(part, p[2 * mt][2], p[2 * mt + 1][2], p[2 * mt][3], p[2 * mt + 1][3], xq[0].z, xq[0].w);
            acc[0][mt][0] = fmaf(f[2 * mt], part[0], acc[0][mt][0]);
            acc[0][mt][1] = fmaf(f[2 * mt], part[1], acc[0][mt][1]);
            acc[0][mt][2] = fmaf(f[2 * mt + 1], part[2], acc[0][mt][2]);
            acc[0][mt][3] = fmaf(f[2 * mt + 1], part[3], acc[0][mt][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }
    // ---- the four K quarters meet in shared memory; summed in a fixed order ----
    named_bar_sync();                       // the previous unit's epilogue is done with red
    {
      float* b = red + kq * kRows * kPitch;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int r = rbase + 16 * mt, c = 8 * nt + 2 * t;
          b[r * kPitch + c] = acc[nt][mt][0];
          b[r * kPitch + c + 1] = acc[nt][mt][1];
          b[(r + 8) * kPitch + c] = acc[nt][mt][2];
          b[(r + 8) * kPitch + c + 1] = acc[nt][mt][3];
        }
    }
    named_bar_sync();
    auto val = [&](int r, int i) {
      const int o = r * kPitch + i, q = kRows * kPitch;
      return ((red[o] + red[q + o]) + red[2 * q + o]) + red[3 * q + o];
    };
    // ---- fused epilogue ----
    // CB4 sparse term of row r against an activation row (same scaling as the MMA input)
    // (four outliers at a time: their columns and values, then the activations, are loaded
    // together; the products are added in ascending position order)
    auto sparse = [&](int r, const __half* xrow) -> float {
      if (!kCb || a.sp_rowptr == nullptr) return 0.f;
      const int64_t R = unit_row<kEpi>(a, un, r);
      const int j1 = a.sp_rowptr[R + 1];
      float acc_s = 0.f;
      for (int j = a.sp_rowptr[R]; j < j1; j += 4) {
        int c[4];
        float v[4], xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          c[q] = (j + q < j1) ? a.sp_col[j + q] : 0;
          v[q] = (j + q < j1) ? __half2float(__ushort_as_half(a.sp_val[j + q])) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = __half2float(xrow[c[q]]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (j + q < j1) acc_s = fmaf(v[q], xv[q], acc_s);
      }
      return acc_s;
    };
    if (kEpi == kEpiSwiglu) {
      for (int idx = threadIdx.x; idx < 32 * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 31, i = idx >> 5;
        const float sc = (L.scl_n > 0) ? ts * scl_s[un.slot0 + i]
                                       : ldexpf(ts, a.sexp[perm_at(un.slot0 + i) / a.topk]);
        const __half* xrow =
            kCb ? a.x16 + static_cast<int64_t>(perm_at(un.slot0 + i) / a.topk) * a.K : nullptr;
        const float gv = fminf((val(r, i) + sparse(r, xrow)) * sc, a.limit);
        const float uv = fminf(fmaxf((val(32 + r, i) + sparse(32 + r, xrow)) * sc, -a.limit), a.limit);
        const float hv = gv / (1.0f + expf(-gv)) * uv;
        a.h_out[static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * 32 + r] = __float2half_rn(hv);
      }
    } else if (kEpi == kEpiDown) {
      for (int idx = threadIdx.x; idx < kRows * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 63, i = idx >> 6;
        const float wgt = (L.scl_n > 0) ? scl_s[un.slot0 + i] : a.gw[perm_at(un.slot0 + i)];
        const float v = val(r, i) + sparse(r, a.x16 + static_cast<int64_t>(un.slot0 + i) * a.K);
        a.o_out[static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * kRows + r] = v * ts * wgt;
      }
    } else {
      for (int idx = threadIdx.x; idx < kRows * un.ntok; idx += kConsumers * 32) {
        const int r = idx & 63, i = idx >> 6;
        const float v = (L.scl_n > 0) ? (val(r, i) * ts) * scl_s[un.slot0 + i]
                                      : ldexpf(val(r, i) * ts, a.sexp[un.slot0 + i]);
        const int64_t o = static_cast<int64_t>(un.slot0 + i) * a.ldo + un.tile * kRows + r;
        if (ksplit > 1) a.part[static_cast<int64_t>(un.ks) * a.T * a.ldo + o] = v;    // fp32 partial
        else a.y_out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      }
    }
  }
  finish();
}

Layout make_layout(int fmt, int K, int E, int P, int P_scl, int tok) {
  Layout L{};
  const int B = (fmt == FP4_MXFP4) ? 32 : 16;
  // CB4 stages carry 4 codebook bytes per 16 indices: the smaller stage keeps 5 in flight
  const bool cb = (fmt == FP4_CB4 || fmt == FP4_V2A);
  const int kc = (!cb && K % 512 == 0) ? 512 : ((K % 256 == 0) ? 256 : 0);
  if (kc == 0) return L;
  L.kc = kc;
  L.nchunks = K / kc;
  L.scale_row = (fmt == FP4_CB4) ? kc / 4 : ((fmt == FP4_V2A) ? kc / 16 : kc / B);
  L.codes_off = 0;
  L.scales_off = kRows * kc / 2;
  L.x_off = L.scales_off + kRows * L.scale_row + ((fmt == FP4_V2A) ? kV2aLibBytes : 0);
  L.x_row = 2 * kc + 64;
  L.stage_bytes = static_cast<int>(align_up(L.x_off + tok * L.x_row, 1024));
  const int Eb = static_cast<int>(align_up(sizeof(int) * (E + 1), 16));
  const int Cb = static_cast<int>(align_up(sizeof(int) * E, 16));
  const int Pb = static_cast<int>(align_up(sizeof(int) * P, 16));
  const int Sb = static_cast<int>(align_up(sizeof(float) * P_scl, 16));
  const int fixed =
      4 * kRows * (tok + 1) * 4 + 4 * kMaxStages + 1024 + 3 * Eb + Cb + Pb + Sb + 16 * kMaxStages + 1024;
  L.stages = std::min(kMaxStages, (smem_budget(kc) - fixed) / L.stage_bytes);
  if (L.stages < 2 || L.stages * L.stage_bytes < static_cast<int>(sizeof(int)) * P) return Layout{};
  L.red_off = L.stages * L.stage_bytes;
  L.su_off = L.red_off + 4 * kRows * (tok + 1) * 4;
  L.lut_off = L.su_off + 4 * kMaxStages;
  L.cnt_off = L.lut_off + 1024;
  L.off_off = L.cnt_off + Eb;
  L.pre_off = L.off_off + Eb;
  L.perm_off = L.pre_off + Eb + Cb;
  L.scl_off = L.perm_off + Pb;
  L.scl_n = P_scl;
  L.bar_off = L.scl_off + Sb;
  L.smem_bytes = L.bar_off + 16 * kMaxStages + 1024;   // + alignment slack
  return L;
}

template <int kFmt, int kEpi, int kMode, int KC, int kT>
fp4_status launch_kc(const DecodeArgs& a, const Layout& L, const CUtensorMap& map, const CUtensorMap& smap, int grid,
                     cudaStream_t st, bool pdl) {
  auto kern = decode_kernel<kFmt, kEpi, kMode, KC, kT>;
  static thread_local int configured = 0;
  if (configured < L.smem_bytes) {
    FP4_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.smem_bytes));
    configured = L.smem_bytes;
  }
  return launch_pdl(kern, dim3(grid), dim3(kThreads), static_cast<size_t>(L.smem_bytes), st, pdl, map, smap, a, L);
}

template <int kFmt, int kEpi, int kMode>
fp4_status launch_one(const DecodeArgs& a, const Layout& L, const CUtensorMap& map, const CUtensorMap& smap,
                      int grid, cudaStream_t st, bool pdl, int tok) {
  if constexpr (kFmt == FP4_NVFP4 && kMode != kModeStatic) {
    if (tok == 16) {
      if (L.kc == 512) return launch_kc<kFmt, kEpi, kMode, 512, 16>(a, L, map, smap, grid, st, pdl);
      return launch_kc<kFmt, kEpi, kMode, 256, 16>(a, L, map, smap, grid, st, pdl);
    }
  }
  if constexpr (kFmt != FP4_CB4 && kFmt != FP4_V2A) {
    if (L.kc == 512) return launch_kc<kFmt, kEpi, kMode, 512, kTok>(a, L, map, smap, grid, st, pdl);
  }
  return launch_kc<kFmt, kEpi, kMode, 256, kTok>(a, L, map, smap, grid, st, pdl);
}

template <int kFmt>
fp4_status dispatch(const DecodeArgs& a, const Layout& L, const CUtensorMap& map, const CUtensorMap& smap, int grid,
                    cudaStream_t st, bool pdl, int tok) {
  if (a.epi == kEpiSwiglu && a.mode == kModeRoute)
    return launch_one<kFmt, kEpiSwiglu, kModeRoute>(a, L, map, smap, grid, st, pdl, tok);
  if (a.epi == kEpiSwiglu) return launch_one<kFmt, kEpiSwiglu, kModeList>(a, L, map, smap, grid, st, pdl, tok);
  if (a.epi == kEpiDown) return launch_one<kFmt, kEpiDown, kModeList>(a, L, map, smap, grid, st, pdl, tok);
  if constexpr (kFmt == FP4_CB4 || kFmt == FP4_V2A) return FP4_ERR_UNSUPPORTED;   // (no dense layer)
  else return launch_one<kFmt, kEpiLinear, kModeStatic>(a, L, map, smap, grid, st, pdl, kTok);
}

}  // namespace

int linear_ksplit(int fmt, int64_t K, int64_t T, int64_t N, size_t part_bytes) {
  if (K > INT32_MAX) return 1;
  const Layout L = make_layout(fmt, static_cast<int>(K), 1, 0, 0, kTok);
  if (L.kc == 0) return 1;
  const int64_t base = (N / kRows) * ((T + kTok - 1) / kTok);
  const int64_t slots = static_cast<int64_t>(ctas_per_sm(L.kc)) * num_sms();
  int ks = 1;
  while (L.nchunks % (2 * ks) == 0 && base * 2 * ks <= slots &&
         static_cast<uint64_t>(2 * ks) * static_cast<uint64_t>(T) * static_cast<uint64_t>(N) * 4u <= part_bytes)
    ks *= 2;
  return ks;
}

// y = bf16 of the K shares' fp32 partial sums, added in share order (deterministic)
__global__ void __launch_bounds__(256) linear_reduce_kernel(const float* __restrict__ part, int ksplit, int64_t n,
                                                            uint16_t* __restrict__ y) {
  // the next kernel on the stream may start now: what it reads before its own dependency
  // wait (a layer's weights) does not depend on this one
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x * 4) {
    float4 s = *reinterpret_cast<const float4*>(part + i);
    for (int ks = 1; ks < ksplit; ++ks) {
      const float4 v = *reinterpret_cast<const float4*>(part + ks * n + i);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(s.x)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.y))) << 16);
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(s.z)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.w))) << 16);
    *reinterpret_cast<uint2*>(y + i) = make_uint2(lo, hi);
  }
}

fp4_status launch_linear_reduce(const float* part, int ksplit, int64_t n_elems, uint16_t* y, cudaStream_t st) {
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n_elems / 4 + 255) / 256, num_sms() * 4)));
  return launch_pdl(linear_reduce_kernel, dim3(grid), dim3(256), 0, st, true, part, ksplit, n_elems, y);
}

fp4_status launch_decode(const DecodeArgs& a, cudaStream_t st, bool pdl) {
  const int E = (a.mode == kModeStatic) ? 1 : a.E;
  const int P_all = (a.mode == kModeStatic) ? a.T : a.T * a.topk;
  const int P = (a.mode == kModeRoute) ? P_all : 0;
  // NVFP4 with at least 32 tokens and as many routed pairs as 2 x the experts: units of up
  // to 16 tokens, so that experts drawing many tokens dequantise each weight tile once per
  // 16 of them (measured: 773 -> 722 us on 256 experts x 64 tokens; with 16 tokens the
  // shallower ring of the 16-row stages cost more than it saved)
  const int tok = (a.mode != kModeStatic && a.fmt == FP4_NVFP4 && a.T >= 32 &&
                   static_cast<int64_t>(a.T) * a.topk >= 2 * static_cast<int64_t>(a.E)) ? 16 : kTok;
  const Layout L = make_layout(a.fmt, a.K, E, P, P_all <= kRouteMaxPairs ? P_all : 0, tok);
  if (L.kc == 0) return FP4_ERR_UNSUPPORTED;
  CUtensorMap map;
  FP4_TRY(make_tmap_2d_u8(&map, a.codes, static_cast<uint64_t>(a.K / 2), static_cast<uint64_t>(a.rows_total),
                          static_cast<uint64_t>(a.K / 2), 128, 32, CU_TENSOR_MAP_SWIZZLE_128B));
  int grid = ctas_per_sm(L.kc) * num_sms();
  if (a.mode == kModeStatic)
    grid = std::min(grid, a.static_tiles * ((a.T + kTok - 1) / kTok) * std::max(1, a.ksplit));
  // the per-row scale bytes (E2M1 block scales, CB4 codebooks, V2a group records) by TMA
  // when a stage's share of a row and the row stride are multiples of 16 bytes
  DecodeArgs b = a;
  const int64_t k_per_byte = L.kc / L.scale_row;                     // K elements per scale byte
  const int64_t srow = a.K / k_per_byte;                             // scale bytes per row
  b.scale_tma = (L.scale_row % 16 == 0 && srow % 16 == 0) ? 1 : 0;
  CUtensorMap smap = map;
  if (b.scale_tma)
    FP4_TRY(make_tmap_2d_u8(&smap, a.scales, static_cast<uint64_t>(srow),
                            static_cast<uint64_t>(a.scale_rows_total > 0 ? a.scale_rows_total : a.rows_total),
                            static_cast<uint64_t>(srow), static_cast<uint32_t>(L.scale_row), 32,
                            CU_TENSOR_MAP_SWIZZLE_NONE));
  if (a.fmt == FP4_CB4) return dispatch<FP4_CB4>(b, L, map, smap, grid, st, pdl, kTok);
  if (a.fmt == FP4_V2A) return dispatch<FP4_V2A>(b, L, map, smap, grid, st, pdl, kTok);
  return (a.fmt == FP4_NVFP4) ? dispatch<FP4_NVFP4>(b, L, map, smap, grid, st, pdl, tok)
                              : dispatch<FP4_MXFP4>(b, L, map, smap, grid, st, pdl, kTok);
}

// y[t, n] = bf16( sum_{j = 0..k-1} o[inv[t k + j], n] ), fixed j order (deterministic).
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv,
                                                      int T, int k, int H, uint16_t* __restrict__ y) {
  pdl_launch_dependents();    // (the next layer's router weights do not depend on this kernel)
  pdl_wait();
  const int64_t n4 = static_cast<int64_t>(T) * (H / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int tt = static_cast<int>(i / (H / 4));
    const int h = static_cast<int>(i % (H / 4)) * 4;
    // the k slot rows are fetched together (eight at a time) and summed in j order
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += 8) {
      int r[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) r[j] = (j0 + j < k) ? inv[tt * k + j0 + j] : -1;
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (r[j] >= 0) v[j] = *reinterpret_cast<const float4*>(o + static_cast<int64_t>(r[j]) * H + h);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (r[j] >= 0) { s.x += v[j].x; s.y += v[j].y; s.z += v[j].z; s.w += v[j].w; }
    }
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(s.x)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.y))) << 16);
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(s.z)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(s.w))) << 16);
    *reinterpret_cast<uint2*>(y + static_cast<int64_t>(tt) * H + h) = make_uint2(lo, hi);
  }
}

// Expert-parallel partial sum: only the slots of this call's experts contribute, fp32 out.
__global__ void __launch_bounds__(256) combine_partial_kernel(const float* __restrict__ o,
                                                              const int32_t* __restrict__ inv,
                                                              const int32_t* __restrict__ ids, int T, int k, int H,
                                                              int e_begin, int e_end, float* __restrict__ y) {
  pdl_launch_dependents();   // successors read nothing of this kernel before their own wait
  pdl_wait();
  const int64_t n4 = static_cast<int64_t>(T) * (H / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int tt = static_cast<int>(i / (H / 4));
    const int h = static_cast<int>(i % (H / 4)) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += 8) {
      int r[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        r[j] = -1;
        if (j0 + j < k) {
          const int e = ids[tt * k + j0 + j];
          if (e >= e_begin && e < e_end) r[j] = inv[tt * k + j0 + j];
        }
      }
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (r[j] >= 0) v[j] = *reinterpret_cast<const float4*>(o + static_cast<int64_t>(r[j]) * H + h);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (r[j] >= 0) { s.x += v[j].x; s.y += v[j].y; s.z += v[j].z; s.w += v[j].w; }
    }
    *reinterpret_cast<float4*>(y + static_cast<int64_t>(tt) * H + h) = s;
  }
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ in, int64_t n,
                                                          uint16_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
}

fp4_status launch_f32_to_bf16(const float* in, int64_t n, uint16_t* out, cudaStream_t st) {
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, num_sms() * 8)));
  f32_to_bf16_kernel<<<grid, 256, 0, st>>>(in, n, out);
  FP4_TRY_CUDA(cudaGetLastError());
  note_launch();
  return FP4_OK;
}

}  // namespace fp4

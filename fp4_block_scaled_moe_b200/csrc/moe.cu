// moe_fp4_forward and fp4_linear: argument checks, workspace layout, launch sequence.
//
// Layer definition: router top-k ("The gate that missed by 0.0202 pp", section "A file
// is a census; a decode step is a sample"), experts with the SwiGLU gate and its clamp
// ("GLM-5.3-Flash-MXFP4" model card, section "Verification compute and EAGLE"), and
// the gate-weighted sum over the k selected experts.
#include <cmath>

#include "kernels.cuh"

namespace fp4 {
namespace {

constexpr size_t kAlign = 256;

enum Variant { kVarGemv = 1, kVarTensor = 2 };

// Which expert-GEMM kernels a call runs (the arguments are already validated).
// Experts whose weights the call holds: [expert_begin, expert_begin + local_experts), or
// all E when local_experts is 0.
int64_t local_count(const fp4_moe_weights* w) {
  return w->local_experts == 0 ? w->num_experts : w->local_experts;
}

bool tensor_supported(const fp4_moe_weights* w, int32_t T) {
  if (w->fmt == FP4_MXFP4) return bs_supported(T, w->num_experts, w->hidden, w->inter);
  if (w->fmt == FP4_NVFP4) return nv_supported(T, w->num_experts, w->hidden, w->inter);
  return false;
}

int moe_variant(const fp4_moe_weights* w, int32_t T, int32_t k) {
  if (w->expert_format != nullptr) return kVarGemv;      // mixed-format buffers: CUDA-core kernels
  const bool tc_ok = tensor_supported(w, T);
  if (w->kernel_variant == kVarTensor) return kVarTensor;
  if (w->kernel_variant == kVarGemv) return kVarGemv;
  // MXFP4: tensor cores when the scale atoms come with the weights, or when the call has
  // enough tokens per expert to amortise re-laying them in the workspace.
  const bool prepared = w->gu_mma_scales != nullptr && w->dn_mma_scales != nullptr;
  const bool many = static_cast<int64_t>(T) * k >= 4 * static_cast<int64_t>(w->num_experts);
  // NVFP4 widens its weights on chip before the tensor cores; measured on the NVFP4 decode
  // experts (64 experts, hidden 6144), the GEMV with 16-token units stays ahead up to 32
  // routed pairs per expert (1070 against 1743 us) and falls behind from 64 (1968 against
  // 1858 us)
  const bool nv_many = static_cast<int64_t>(T) * k >= 64 * static_cast<int64_t>(w->num_experts);
  if (w->fmt == FP4_NVFP4) return (tc_ok && nv_many) ? kVarTensor : kVarGemv;
  return (tc_ok && (prepared || many)) ? kVarTensor : kVarGemv;
}

struct MoeWs {
  size_t status, logits, ids, gw, counts, offsets, perm, inv, sexp, x16, h, o, xq, xs, hq, hs, agu, adn, total;
};

// NVFP4 on the tensor cores: f16 activation rows in slot order and their exponents,
// h as f16, and the weights' scale atoms unless the caller has them.
bool moe_ws_layout_nv(const fp4_moe_weights* w, int32_t T, int32_t k, MoeWs* L) {
  const int64_t E = w->num_experts, H = w->hidden, I = w->inter;
  const int64_t P = static_cast<int64_t>(T) * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  *L = MoeWs{};
  L->status = take(sizeof(WsControl));
  L->logits = take(sizeof(float) * T * E);
  L->ids = take(sizeof(int32_t) * P);
  L->gw = take(sizeof(float) * P);
  L->counts = take(sizeof(int32_t) * E);
  L->offsets = take(sizeof(int32_t) * (E + 1));
  L->perm = take(sizeof(int32_t) * P);
  L->inv = take(sizeof(int32_t) * P);
  L->sexp = take(sizeof(int32_t) * P);                 // per-slot exponents of xs
  L->xs = take(sizeof(uint16_t) * P * H);
  L->h = take(sizeof(uint16_t) * P * I);
  L->o = take(sizeof(float) * P * H);
  const int64_t El = local_count(w);
  L->agu = take(w->gu_mma_scales == nullptr ? El * 2 * I * (H / 16) : 0);
  L->adn = take(w->dn_mma_scales == nullptr ? El * H * (I / 16) : 0);
  L->total = off;
  return true;
}

bool moe_ws_layout(const fp4_moe_weights* w, int32_t T, int32_t k, MoeWs* L) {
  const int64_t E = w->num_experts, H = w->hidden, I = w->inter;
  const bool tensor = moe_variant(w, T, k) == kVarTensor;
  if (tensor && w->fmt == FP4_NVFP4) return moe_ws_layout_nv(w, T, k, L);
  const int64_t P = static_cast<int64_t>(T) * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  L->status = take(sizeof(WsControl));
  L->logits = take(sizeof(float) * T * E);
  L->ids = take(sizeof(int32_t) * P);
  L->gw = take(sizeof(float) * P);
  L->counts = take(sizeof(int32_t) * E);
  L->offsets = take(sizeof(int32_t) * (E + 1));
  L->perm = take(sizeof(int32_t) * P);
  L->inv = take(sizeof(int32_t) * P);
  L->sexp = take(sizeof(int32_t) * T);
  L->x16 = take(tensor ? 0 : sizeof(uint16_t) * T * H);
  L->h = take(tensor ? 0 : sizeof(uint16_t) * P * I);
  L->o = take(sizeof(float) * P * H);
  // tensor-core variant: x and h as two MXFP8 terms per slot (rows 2i, 2i + 1), their
  // scale atoms per token group, and the weights' scale atoms unless the caller has them
  const int cap = tensor ? bs_ntok_cap(T, static_cast<int>(E)) : 1;
  L->xq = take(tensor ? 2 * P * H : 0);
  L->xs = take(tensor ? bs_group_atom_bytes(static_cast<int>(P), static_cast<int>(E), cap, static_cast<int>(H)) : 0);
  L->hq = take(tensor ? 2 * P * I : 0);
  L->hs = take(tensor ? bs_group_atom_bytes(static_cast<int>(P), static_cast<int>(E), cap, static_cast<int>(I)) : 0);
  const int64_t El = local_count(w);
  L->agu = take(tensor && w->gu_mma_scales == nullptr ? El * 2 * I * (H / 32) : 0);
  L->adn = take(tensor && w->dn_mma_scales == nullptr ? El * H * (I / 32) : 0);
  L->total = off;
  return true;
}

fp4_status check_moe(const fp4_moe_weights* w, int32_t T, int32_t k) {
  if (w == nullptr) return FP4_ERR_INVALID_ARG;
  if (w->fmt != FP4_MXFP4 && w->fmt != FP4_NVFP4 && w->fmt != FP4_CB4 && w->fmt != FP4_V2A)
    return FP4_ERR_INVALID_ARG;
  int64_t n;
  FP4_TRY(checked_count({w->num_experts, w->hidden, w->inter, T}, &n));
  if (k <= 0) return FP4_ERR_EMPTY_SHAPE;
  const int64_t E = w->num_experts, H = w->hidden, I = w->inter;
  // byte sizes of the largest tensors must not overflow
  int64_t tmp;
  FP4_TRY(checked_count({E, 2 * I, H}, &tmp));
  int64_t P;
  if (!mul_ok(T, k, &P) || P >= (int64_t(1) << 31)) return FP4_ERR_SHAPE_OVERFLOW;
  if (!mul_ok(P, H * 4, &tmp) || !mul_ok(static_cast<int64_t>(T) * E, 4, &tmp)) return FP4_ERR_SHAPE_OVERFLOW;
  if (E * 2 * I >= (int64_t(1) << 31) || E * H >= (int64_t(1) << 31)) return FP4_ERR_SHAPE_OVERFLOW;
  if (k > E || k > 32 || E > 1024) return FP4_ERR_INVALID_ARG;
  if (w->local_experts < 0 || w->expert_begin < 0 || (w->local_experts == 0 && w->expert_begin != 0) ||
      static_cast<int64_t>(w->expert_begin) + w->local_experts > E)
    return FP4_ERR_INVALID_ARG;
  const int B = (w->fmt == FP4_MXFP4) ? 32 : (w->fmt == FP4_NVFP4 ? 16 : 128);   // CB4 / V2a: 128-groups
  if (H % B != 0 || I % B != 0) return FP4_ERR_ALIGNMENT;
  if (H % 256 != 0 || I % 256 != 0) return FP4_ERR_UNSUPPORTED;
  if (!(w->swiglu_limit > 0.f) || !(w->swiglu_limit <= 128.f)) return FP4_ERR_INVALID_ARG;
  if (w->fmt == FP4_CB4 || w->fmt == FP4_V2A) {
    if (!w->gu_codes || !w->gu_cb || !w->dn_codes || !w->dn_cb || !w->gu_rowptr || !w->dn_rowptr)
      return FP4_ERR_INVALID_ARG;
    if (w->fmt == FP4_V2A && (!w->gu_scales || !w->dn_scales)) return FP4_ERR_INVALID_ARG;
    if (w->fmt == FP4_V2A && (!aligned16(w->gu_scales) || !aligned16(w->dn_scales))) return FP4_ERR_ALIGNMENT;
    if (!aligned16(w->gu_codes) || !aligned16(w->gu_cb) || !aligned16(w->dn_codes) || !aligned16(w->dn_cb))
      return FP4_ERR_ALIGNMENT;
    if (w->kernel_variant == kVarTensor) return FP4_ERR_UNSUPPORTED;
    if (w->kernel_variant < 0 || w->kernel_variant > 2) return FP4_ERR_INVALID_ARG;
    return FP4_OK;
  }
  if (!w->gu_codes || !w->gu_scales || !w->dn_codes || !w->dn_scales) return FP4_ERR_INVALID_ARG;
  if (w->fmt == FP4_NVFP4 && (!w->gu_tscale || !w->dn_tscale)) return FP4_ERR_INVALID_ARG;
  if (w->expert_format != nullptr) {
    if (w->fmt != FP4_MXFP4) return FP4_ERR_UNSUPPORTED;
    if (!w->gu_offset || !w->gu_scale_offset || !w->dn_offset || !w->dn_scale_offset) return FP4_ERR_INVALID_ARG;
    if (w->gu_bytes <= 0 || w->dn_bytes <= 0 || w->gu_scale_bytes <= 0 || w->dn_scale_bytes <= 0)
      return FP4_ERR_EMPTY_SHAPE;
    if (w->gu_bytes % (H / 2) || w->dn_bytes % (I / 2) || w->gu_scale_bytes % (H / 32) || w->dn_scale_bytes % (I / 32))
      return FP4_ERR_ALIGNMENT;
    if (w->kernel_variant == kVarTensor) return FP4_ERR_UNSUPPORTED;
  }
  if (w->kernel_variant < 0 || w->kernel_variant > 2) return FP4_ERR_INVALID_ARG;
  if (w->kernel_variant == kVarTensor && !tensor_supported(w, T)) return FP4_ERR_UNSUPPORTED;
  if (!aligned16(w->gu_codes) || !aligned16(w->gu_scales) || !aligned16(w->dn_codes) || !aligned16(w->dn_scales))
    return FP4_ERR_ALIGNMENT;
  if (!aligned16(w->gu_mma_scales) || !aligned16(w->dn_mma_scales)) return FP4_ERR_ALIGNMENT;
  return FP4_OK;
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" size_t moe_fp4_workspace_size(const fp4_moe_weights* w, int32_t T, int32_t k) {
  if (check_moe(w, T, k) != FP4_OK) return 0;
  MoeWs L;
  moe_ws_layout(w, T, k, &L);
  return L.total;
}

extern "C" int32_t moe_fp4_expert_kernels(const fp4_moe_weights* w, int32_t T, int32_t k) {
  if (check_moe(w, T, k) != FP4_OK) return 0;
  return moe_variant(w, T, k);
}

namespace fp4 {
namespace {

// The layer's last step: y = bf16(sum_j o) (full expert set), or the fp32 sum over the
// slots of the call's experts (expert-parallel partial sum).
fp4_status launch_combine(const float* o, const int32_t* inv, const int32_t* ids, int T, int k, int H, int e0,
                          int e1, void* y_bf16, float* y_partial, cudaStream_t st) {
  const int64_t n4 = static_cast<int64_t>(T) * (H / 4);
  const int grid = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, num_sms() * 8));
  if (y_partial != nullptr)
    return launch_pdl(combine_partial_kernel, dim3(grid), dim3(256), 0, st, true, o, inv, ids, T, k, H, e0, e1,
                      y_partial);
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, st, true, o, inv, T, k, H,
                    static_cast<uint16_t*>(y_bf16));
}

fp4_status moe_forward_impl(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                            const float* router_bias, int32_t T, int32_t k, void* y_bf16, float* y_partial,
                            const fp4_route_out* route, void* workspace, size_t ws_bytes, void* stream) {
  FP4_TRY(check_moe(w, T, k));
  void* y_out = y_partial ? static_cast<void*>(y_partial) : y_bf16;
  if (!x_bf16 || !router_w || !y_out) return FP4_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(router_w) || !aligned16(y_out)) return FP4_ERR_ALIGNMENT;
  MoeWs L;
  moe_ws_layout(w, T, k, &L);
  if (workspace == nullptr || ws_bytes < L.total) return FP4_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return FP4_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = w->num_experts, H = w->hidden, I = w->inter;
  const int P = T * k;
  const int El = static_cast<int>(local_count(w));
  const int e0 = w->expert_begin, e1 = w->expert_begin + El;

  auto pick = [](auto* user, void* fallback) { return user ? user : reinterpret_cast<decltype(user)>(fallback); };
  const fp4_route_out none = {};
  const fp4_route_out& ro = route ? *route : none;
  RouteArgs ra{};
  ra.x = x_bf16; ra.router_w = router_w; ra.router_bias = router_bias;
  ra.T = T; ra.H = H; ra.E = E; ra.k = k;
  ra.logits_in = nullptr;
  ra.logits = pick(ro.logits, ws + L.logits);
  ra.ids = pick(ro.topk_ids, ws + L.ids);
  ra.gw = pick(ro.topk_w, ws + L.gw);
  ra.counts = pick(ro.counts, ws + L.counts);
  ra.offsets = pick(ro.offsets, ws + L.offsets);
  ra.perm = pick(ro.perm, ws + L.perm);
  ra.inv = pick(ro.inv, ws + L.inv);
  ra.x16 = reinterpret_cast<__half*>(ws + L.x16);
  ra.sexp = reinterpret_cast<int*>(ws + L.sexp);
  ra.ctrl = reinterpret_cast<WsControl*>(ws + L.status);
  if (moe_variant(w, T, k) == kVarTensor && w->fmt == FP4_NVFP4) {
    // router (logits, top-k, permutation), then the slot-ordered f16 activation rows
    ra.x16 = nullptr;
    ra.logits_only = false;
    ra.pdl_first = true;
    FP4_TRY(launch_route(ra, st));
    __half* xs = reinterpret_cast<__half*>(ws + L.xs);
    int* sx = reinterpret_cast<int*>(ws + L.sexp);
    FP4_TRY(launch_gather_x16(static_cast<const uint16_t*>(x_bf16), ra.perm, k, P, H, xs, sx, st));
    const uint8_t* agu = w->gu_mma_scales;
    const uint8_t* adn = w->dn_mma_scales;
    if (agu == nullptr) {
      FP4_TRY(launch_nv_scales(w->gu_scales, static_cast<int64_t>(El) * 2 * I, H, I, ws + L.agu, st));
      agu = ws + L.agu;
    }
    if (adn == nullptr) {
      FP4_TRY(launch_nv_scales(w->dn_scales, static_cast<int64_t>(El) * H, I, 0, ws + L.adn, st));
      adn = ws + L.adn;
    }
    NvArgs g{};
    g.epi = kEpiSwiglu;
    g.codes = w->gu_codes;
    g.a_atoms = agu;
    g.tscale = w->gu_tscale;
    g.rows_total = static_cast<int64_t>(El) * 2 * I;
    g.K = H;
    g.rows_per_expert = 2 * I;
    g.inter = I;
    g.E = E;
    g.e_begin = e0;
    g.e_end = e1;
    g.P = P;
    g.ntok_cap = nv_ntok_cap(T, E);
    g.counts = ra.counts;
    g.b_rows = xs;
    g.sx = sx;
    g.limit = w->swiglu_limit;
    g.h_out = reinterpret_cast<__half*>(ws + L.h);
    g.status = &ra.ctrl->status;
    g.slot = &ra.ctrl->slot[0];
    g.unit_next = &ra.ctrl->unit_next[0];
    FP4_TRY(launch_nv(g, T, st));
    NvArgs d = g;
    d.epi = kEpiDown;
    d.codes = w->dn_codes;
    d.a_atoms = adn;
    d.tscale = w->dn_tscale;
    d.rows_total = static_cast<int64_t>(El) * H;
    d.K = I;
    d.rows_per_expert = H;
    d.b_rows = g.h_out;
    d.sx = nullptr;
    d.h_out = nullptr;
    d.gw = ra.gw;
    d.perm = ra.perm;
    d.o_out = reinterpret_cast<float*>(ws + L.o);
    d.ldo = H;
    d.slot = &ra.ctrl->slot[1];
    d.unit_next = &ra.ctrl->unit_next[1];
    FP4_TRY(launch_nv(d, T, st));
    return launch_combine(d.o_out, ra.inv, ra.ids, T, k, H, e0, e1, y_bf16, y_partial, st);
  }
  if (moe_variant(w, T, k) == kVarTensor) {
    // small routing problems: top-k, permutation and the activation split share a launch
    const bool fused_split = P <= kRouteMaxPairs && E <= kRouteMaxExperts;
    ra.x16 = nullptr;
    ra.logits_only = fused_split;
    ra.pdl_first = true;
    FP4_TRY(launch_route(ra, st));
    uint8_t* xq = ws + L.xq;
    uint8_t* xs = ws + L.xs;
    const int cap = bs_ntok_cap(T, E);
    const uint8_t* agu = w->gu_mma_scales;
    const uint8_t* adn = w->dn_mma_scales;
    if (agu == nullptr) {
      FP4_TRY(launch_mma_scales(w->gu_scales, static_cast<int64_t>(El) * 2 * I, H, I, ws + L.agu, st));
      agu = ws + L.agu;
    }
    if (adn == nullptr) {
      FP4_TRY(launch_mma_scales(w->dn_scales, static_cast<int64_t>(El) * H, I, 0, ws + L.adn, st));
      adn = ws + L.adn;
    }
    if (fused_split)
      FP4_TRY(launch_route_split(ra.logits, T, E, k, static_cast<const uint16_t*>(x_bf16), H, cap, ra.ids, ra.gw,
                                 ra.counts, ra.offsets, ra.perm, ra.inv, xq, xs, st));
    else
      FP4_TRY(launch_split_x(static_cast<const uint16_t*>(x_bf16), ra.inv, ra.counts, ra.offsets, E, k, P, H, cap,
                             xq, xs, st));
    BsArgs g{};
    g.epi = kEpiSwiglu;
    g.codes = w->gu_codes;
    g.a_atoms = agu;
    g.ntok_cap = cap;
    g.rows_total = static_cast<int64_t>(El) * 2 * I;
    g.K = H;
    g.rows_per_expert = 2 * I;
    g.inter = I;
    g.E = E;
    g.e_begin = e0;
    g.e_end = e1;
    g.P = P;
    g.counts = ra.counts;
    g.b_q = xq;
    g.b_atoms = xs;
    g.limit = w->swiglu_limit;
    g.hq = ws + L.hq;
    g.h_atoms = ws + L.hs;
    g.status = &ra.ctrl->status;
    g.slot = &ra.ctrl->slot[0];
    g.unit_next = &ra.ctrl->unit_next[0];
    FP4_TRY(launch_bs(g, T, st));
    BsArgs d = g;
    d.epi = kEpiDown;
    d.codes = w->dn_codes;
    d.a_atoms = adn;
    d.rows_total = static_cast<int64_t>(El) * H;
    d.K = I;
    d.rows_per_expert = H;
    d.b_q = g.hq;
    d.b_atoms = g.h_atoms;
    d.gw = ra.gw;
    d.perm = ra.perm;
    d.o_out = reinterpret_cast<float*>(ws + L.o);
    d.ldo = H;
    d.slot = &ra.ctrl->slot[1];
    d.unit_next = &ra.ctrl->unit_next[1];
    FP4_TRY(launch_bs(d, T, st));
    return launch_combine(d.o_out, ra.inv, ra.ids, T, k, H, e0, e1, y_bf16, y_partial, st);
  }

  // small routing problems finish inside the gate_up kernel's prologue
  const bool fused = P <= kRouteMaxPairs && E <= kRouteMaxExperts;
  ra.logits_only = fused;
  ra.pdl_first = true;
  FP4_TRY(launch_route(ra, st));

  DecodeArgs g{};
  g.fmt = w->fmt;
  g.epi = kEpiSwiglu;
  g.mode = fused ? kModeRoute : kModeList;
  g.codes = w->gu_codes;
  g.scales = (w->fmt == FP4_CB4) ? reinterpret_cast<const uint8_t*>(w->gu_cb) : w->gu_scales;
  g.lib = (w->fmt == FP4_V2A) ? reinterpret_cast<const uint8_t*>(w->gu_cb) : nullptr;
  g.tscale = w->gu_tscale;
  if (w->fmt == FP4_CB4 || w->fmt == FP4_V2A) {
    g.sp_rowptr = w->gu_rowptr;
    g.sp_col = w->gu_col;
    g.sp_val = w->gu_val;
  }
  const bool mixed = w->expert_format != nullptr;
  g.rows_total = mixed ? w->gu_bytes / (H / 2) : static_cast<int64_t>(El) * 2 * I;
  g.K = H;
  g.rows_per_expert = 2 * I;
  g.inter = I;
  g.E = E;
  g.e_begin = e0;
  g.e_end = e1;
  g.ex_fmt = w->expert_format;
  g.row_off = w->gu_offset;
  g.srow_off = w->gu_scale_offset;
  g.scale_rows_total = mixed ? w->gu_scale_bytes / (H / 32) : 0;
  g.T = T;
  g.topk = k;
  g.logits = ra.logits;
  g.ids = ra.ids;
  g.gw = ra.gw;
  g.counts = ra.counts;
  g.offsets = ra.offsets;
  g.perm = ra.perm;
  g.inv = ra.inv;
  g.x16 = ra.x16;
  g.sexp = ra.sexp;
  g.limit = w->swiglu_limit;
  g.h_out = reinterpret_cast<__half*>(ws + L.h);
  g.ldo = I;
  g.status = &ra.ctrl->status;
  g.slot = &ra.ctrl->slot[0];
  g.unit_next = &ra.ctrl->unit_next[0];
  FP4_TRY(launch_decode(g, st, true));
  Dense16Args dg{};
  if (mixed) {                     // the bf16 experts of the mixed buffer, same units and epilogue
    dg.epi = kEpiSwiglu;
    dg.weights = w->gu_codes;
    dg.offset = w->gu_offset;
    dg.ex_fmt = w->expert_format;
    dg.e_begin = e0;
    dg.e_end = e1;
    dg.E = E;
    dg.K = H;
    dg.rows_per_expert = 2 * I;
    dg.inter = I;
    dg.topk = k;
    dg.counts = ra.counts;
    dg.perm = ra.perm;
    dg.x16 = ra.x16;
    dg.sexp = ra.sexp;
    dg.limit = w->swiglu_limit;
    dg.h_out = g.h_out;
    FP4_TRY(launch_dense16(dg, st));
  }

  DecodeArgs d = g;
  d.epi = kEpiDown;
  d.mode = kModeList;
  d.codes = w->dn_codes;
  d.scales = (w->fmt == FP4_CB4) ? reinterpret_cast<const uint8_t*>(w->dn_cb) : w->dn_scales;
  d.lib = (w->fmt == FP4_V2A) ? reinterpret_cast<const uint8_t*>(w->dn_cb) : nullptr;
  d.tscale = w->dn_tscale;
  if (w->fmt == FP4_CB4 || w->fmt == FP4_V2A) {
    d.sp_rowptr = w->dn_rowptr;
    d.sp_col = w->dn_col;
    d.sp_val = w->dn_val;
  }
  d.rows_total = mixed ? w->dn_bytes / (I / 2) : static_cast<int64_t>(El) * H;
  d.K = I;
  d.rows_per_expert = H;
  d.row_off = w->dn_offset;
  d.srow_off = w->dn_scale_offset;
  d.scale_rows_total = mixed ? w->dn_scale_bytes / (I / 32) : 0;
  d.x16 = g.h_out;
  d.sexp = nullptr;
  d.o_out = reinterpret_cast<float*>(ws + L.o);
  d.slot = &ra.ctrl->slot[1];
  d.unit_next = &ra.ctrl->unit_next[1];
  d.ldo = H;
  FP4_TRY(launch_decode(d, st, true));
  if (mixed) {
    Dense16Args dd = dg;
    dd.epi = kEpiDown;
    dd.weights = w->dn_codes;
    dd.offset = w->dn_offset;
    dd.K = I;
    dd.rows_per_expert = H;
    dd.x16 = g.h_out;
    dd.sexp = nullptr;
    dd.h_out = nullptr;
    dd.gw = ra.gw;
    dd.o_out = d.o_out;
    dd.ldo = H;
    FP4_TRY(launch_dense16(dd, st));
  }
  return launch_combine(d.o_out, ra.inv, ra.ids, T, k, H, e0, e1, y_bf16, y_partial, st);
}

}  // namespace
}  // namespace fp4

extern "C" fp4_status moe_fp4_forward(const fp4_moe_weights* w, const void* x_bf16, const float* router_w,
                                      const float* router_bias, int32_t T, int32_t k, void* y_bf16,
                                      const fp4_route_out* route, void* workspace, size_t ws_bytes,
                                      void* stream) {
  if (w != nullptr && w->local_experts != 0 && w->local_experts != w->num_experts)
    return FP4_ERR_INVALID_ARG;        // a part of the experts gives a partial sum: moe_fp4_forward_partial
  if (y_bf16 == nullptr) return FP4_ERR_INVALID_ARG;
  return moe_forward_impl(w, x_bf16, router_w, router_bias, T, k, y_bf16, nullptr, route, workspace, ws_bytes,
                          stream);
}

extern "C" fp4_status moe_fp4_forward_partial(const fp4_moe_weights* w, const void* x_bf16,
                                              const float* router_w, const float* router_bias, int32_t T,
                                              int32_t k, float* y_partial, const fp4_route_out* route,
                                              void* workspace, size_t ws_bytes, void* stream) {
  if (y_partial == nullptr) return FP4_ERR_INVALID_ARG;
  return moe_forward_impl(w, x_bf16, router_w, router_bias, T, k, nullptr, y_partial, route, workspace, ws_bytes,
                          stream);
}

extern "C" fp4_status fp4_f32_to_bf16(const float* in, int64_t n, void* out, void* stream) {
  if (n <= 0) return FP4_ERR_EMPTY_SHAPE;
  if (in == nullptr || out == nullptr) return FP4_ERR_INVALID_ARG;
  return launch_f32_to_bf16(in, n, static_cast<uint16_t*>(out), static_cast<cudaStream_t>(stream));
}

// fp32 partial sums of a dense layer split over K (few tokens, few output tiles)
constexpr size_t kLinearPartBytes = size_t(1) << 20;

extern "C" size_t fp4_linear_workspace_size(int32_t T, int64_t K) {
  if (T <= 0 || K <= 0) return 0;
  return align_up(sizeof(WsControl), kAlign) + align_up(sizeof(int32_t) * T, kAlign) +
         align_up(sizeof(uint16_t) * static_cast<size_t>(T) * static_cast<size_t>(K), kAlign) + kLinearPartBytes;
}

extern "C" fp4_status fp4_linear(fp4_format fmt, const void* x_bf16, int32_t T, int64_t K,
                                 const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                                 int64_t N, void* y_bf16, void* workspace, size_t ws_bytes, void* stream) {
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4)
    return (fmt == FP4_CB4 || fmt == FP4_V2A) ? FP4_ERR_UNSUPPORTED : FP4_ERR_INVALID_ARG;
  int64_t n;
  FP4_TRY(checked_count({T, K, N}, &n));
  int64_t tmp;
  FP4_TRY(checked_count({N, K}, &tmp));
  if (N >= (int64_t(1) << 31) || K >= (int64_t(1) << 30) || !mul_ok(T, K * 2, &tmp)) return FP4_ERR_SHAPE_OVERFLOW;
  const int B = (fmt == FP4_MXFP4) ? 32 : 16;
  if (K % B != 0) return FP4_ERR_ALIGNMENT;
  if (K % 256 != 0 || N % 64 != 0) return FP4_ERR_UNSUPPORTED;
  if (!x_bf16 || !codes || !scales || !y_bf16 || (fmt == FP4_NVFP4 && !tensor_scale)) return FP4_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales) || !aligned16(y_bf16)) return FP4_ERR_ALIGNMENT;
  const size_t need = fp4_linear_workspace_size(T, K);
  if (workspace == nullptr || ws_bytes < need) return FP4_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return FP4_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsControl* ctrl = reinterpret_cast<WsControl*>(ws);
  const size_t ctrl_bytes = align_up(sizeof(WsControl), kAlign);
  int* sexp = reinterpret_cast<int*>(ws + ctrl_bytes);
  __half* x16 = reinterpret_cast<__half*>(ws + ctrl_bytes + align_up(sizeof(int32_t) * T, kAlign));
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(x16) +
                                         align_up(sizeof(uint16_t) * static_cast<size_t>(T) * static_cast<size_t>(K), kAlign));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // up to kLinearFusedTokens tokens the GEMV converts x itself in one launch (each work unit
  // scans its 8 token rows for their scale first); beyond, x_to_f16_kernel converts it once
  constexpr int64_t kLinearFusedTokens = 64;
  const bool fused = T <= kLinearFusedTokens;
  if (!fused)
    FP4_TRY(launch_pdl(x_to_f16_kernel, dim3((T + 7) / 8), dim3(256), 0, st, true,
                       static_cast<const uint16_t*>(x_bf16), static_cast<int>(T), static_cast<int>(K), x16, sexp,
                       ctrl));
  DecodeArgs a{};
  a.fmt = fmt;
  a.epi = kEpiLinear;
  a.mode = kModeStatic;
  a.T = T;
  a.codes = codes;
  a.scales = scales;
  a.tscale = tensor_scale;
  a.rows_total = N;
  a.K = static_cast<int>(K);
  a.rows_per_expert = static_cast<int>(N);
  a.static_tiles = static_cast<int>(N / 64);
  a.e_begin = 0;
  a.e_end = 1;
  a.x16 = fused ? nullptr : x16;
  a.x_bf16 = static_cast<const uint16_t*>(x_bf16);
  a.sexp = fused ? nullptr : sexp;
  a.y_out = static_cast<uint16_t*>(y_bf16);
  a.ldo = static_cast<int>(N);
  a.status = &ctrl->status;
  a.slot = &ctrl->slot[0];
  // too few 64-row tiles x token groups to fill the GPU: split K, partials reduced after
  a.ksplit = linear_ksplit(fmt, K, T, N, kLinearPartBytes);
  a.part = part;
  FP4_TRY(launch_decode(a, st, true));
  if (a.ksplit > 1) FP4_TRY(launch_linear_reduce(part, a.ksplit, T * N, static_cast<uint16_t*>(y_bf16), st));
  return FP4_OK;
}

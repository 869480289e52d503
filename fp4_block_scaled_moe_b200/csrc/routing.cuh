// Router device routines shared by the routing kernels and by the grouped kernels
// fused routing prologue.
#pragma once

#include "common.cuh"

namespace fp4 {

constexpr int kMaxE = 1024;

// Order key: larger logit first; -0 equals +0; NaN below every number.
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 0u;
  v = v + 0.0f;                                    // -0 -> +0
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// The logit of an order key (inverse of order_key for every number; a NaN key reads as a NaN)
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of one token's logits by one warp (E <= 1024, k <= 32): descending logit, ties to
// the lower expert.  Writes ids[0..k) and, when gw != null, the softmax over the k logits.
template <int kPer>
__device__ __forceinline__ void topk_warp_n(const float* __restrict__ lg, int E, int k, int32_t* __restrict__ ids,
                                            float* __restrict__ gw) {
  const int lane = threadIdx.x & 31;
  uint32_t key[kPer];
  const int per = (E + 31) / 32;
  uint32_t taken = 0;   // bit j: my entry j already selected (or absent)
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = j * 32 + lane;
    const bool have = j < per && e < E;
    key[j] = have ? order_key(lg[e]) : 0u;
    if (!have) taken |= 1u << j;
  }
  float m = 0.f, sum = 0.f, my_logit = 0.f;
  int my_id = 0;
  for (int r = 0; r < k; ++r) {
    uint32_t best = 0;
    int best_e = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (!(taken >> j & 1u)) {
        const int e = j * 32 + lane;
        if (key[j] > best || (key[j] == best && e < best_e)) { best = key[j]; best_e = e; }
      }
    }
    // the warp's largest key, then the lowest expert holding it (two warp reductions)
    const uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, best);
    best_e = __reduce_min_sync(0xFFFFFFFFu, best == wmax ? best_e : 0x7FFFFFFF);
    best = wmax;
    if ((best_e & 31) == lane) taken |= 1u << (best_e >> 5);
    const float l = key_value(best);                 // the logit itself (-0 read as +0)
    if (r == 0) m = l;
    const float z = expf(l - m);
    sum += z;
    if (lane == r) { my_logit = l; my_id = best_e; }
  }
  if (lane < k) {
    ids[lane] = my_id;
    if (gw != nullptr) gw[lane] = expf(my_logit - m) / sum;
  }
}

__device__ __forceinline__ void topk_warp(const float* __restrict__ lg, int E, int k, int32_t* __restrict__ ids,
                                          float* __restrict__ gw) {
  if (E <= 64) topk_warp_n<2>(lg, E, k, ids, gw);
  else if (E <= 256) topk_warp_n<8>(lg, E, k, ids, gw);
  else topk_warp_n<kMaxE / 32>(lg, E, k, ids, gw);
}

}  // namespace fp4

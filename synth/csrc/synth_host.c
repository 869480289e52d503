/* Host twin of synth/draws.py in C, for drawing large weight slices quickly.
 * Same recipe as synth/draws.py and synth/csrc/synth_gen.cu: Philox4x32-10 words
 * (Salmon et al., SC'11) and Bailey's polar Student-t(4) step, each float operation
 * correctly rounded in the same order (build with -ffp-contract=off, SSE floats).
 * Input generation only. */
#include <math.h>
#include <stdint.h>

static void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

static float signed_uniform(uint32_t r) { return (float)((int32_t)(r >> 8) - (1 << 23)) * 0x1p-23f; }
static float unit_uniform(uint32_t r) { return (float)(r >> 8) * 0x1p-24f; }

__attribute__((visibility("default"))) void synth_t4_host(float* out, int64_t start, int64_t count, uint32_t seed,
                                                         uint32_t tid, float scale, int with_outliers, float frac,
                                                         float lo_s, float span_s, float sigma) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    const uint64_t idx = (uint64_t)(start + i);
    const uint32_t lo = (uint32_t)idx, hi = (uint32_t)(idx >> 32);
    float t = 0.0f;
    int done = 0;
    for (uint32_t attempt = 0; attempt < 8 && !done; ++attempt) {
      uint32_t c[4] = {lo, hi, attempt, 0u};
      philox4x32_10(c, seed, tid);
      for (int p = 0; p < 2 && !done; ++p) {
        const float u = signed_uniform(c[2 * p]), v = signed_uniform(c[2 * p + 1]);
        const float uu = u * u, vv = v * v;
        const float w = uu + vv;
        if (w > 0.0f && w <= 1.0f) {
          float s = sqrtf(w);
          s = 1.0f / s;
          s = s - 1.0f;
          s = s * 4.0f;
          s = s / w;
          s = sqrtf(s);
          t = u * s;
          done = 1;
        }
      }
    }
    float wv = t * scale;
    if (with_outliers) {
      uint32_t c[4] = {lo, hi, 0xFFFFFFFFu, 0u};
      philox4x32_10(c, seed, tid);
      if (unit_uniform(c[0]) < frac) {
        float m = span_s * unit_uniform(c[1]);
        m = lo_s + m;
        m = m * sigma;
        wv = (c[2] & 1u) ? -m : m;
      }
    }
    out[i] = wv;
  }
}

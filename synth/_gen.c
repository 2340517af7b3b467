/* Fast host-side twin of synth.normal(): the same counter-based draw, written
 * in C so that generating a few hundred MB of seeded inputs on the CPU takes
 * seconds. Integer hashing, one exact int->float conversion, one fp32
 * multiply, one round-to-nearest-even to bf16 -- identical bits to the torch
 * implementation on any device (a test checks this). */
#include <stdint.h>
#include <string.h>

static inline uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352du;
  x ^= x >> 15;
  x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7fffu + ((u >> 16) & 1u); /* finite inputs only */
  return (uint16_t)(u >> 16);
}

/* out_kind: 0 = fp32, 1 = bf16. kj[4], khi: per-tensor keys from synth._keys. */
void synth_normal(void* out, int out_kind, int64_t n, int64_t offset, const uint32_t* kj, uint32_t khi,
                  float c) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint64_t idx = (uint64_t)(offset + i);
    uint32_t lo = (uint32_t)idx;
    uint32_t hi = mix32((uint32_t)(idx >> 32) ^ khi);
    int64_t s = 0;
    for (int j = 0; j < 4; ++j) {
      uint32_t w = mix32(mix32(lo ^ kj[j]) ^ hi);
      s += (w & 0xffffu) + (w >> 16);
    }
    float v = (float)(s - 262140) * c;
    if (out_kind == 0)
      ((float*)out)[i] = v;
    else
      ((uint16_t*)out)[i] = f32_to_bf16_rne(v);
  }
}

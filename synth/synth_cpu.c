/*
 * synth_cpu.c -- seeded synthetic inputs, host side.
 *
 * This is the input generator shared by the CUDA path's tests/benchmark and by
 * the oracle. It holds none of the MoE layer's arithmetic: it only turns
 * (seed, index) into a float. The device twin (synth_gpu.cu) implements the
 * same published generator independently, so either side can materialise any
 * slice of a tensor (one expert of a 256-expert layer, say) on its own.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; constants as published by Vigna in the
 * public-domain reference implementation) used as a counter-based hash:
 *   h(seed, c) = mix(seed + (c + 1) * 0x9E3779B97F4A7C15)
 * Normal deviates: Irwin-Hall sum of twelve 24-bit uniforms (two per hash,
 * bits 40..63 and 16..39 of six consecutive hashes), centred, as an exact
 * integer z in (-6*2^24, 6*2^24); value = RN32(RN32(z) * RN32(sigma * 2^-24)).
 * Variance of the sum of twelve U(0,1) is 1, so the value has std ~ sigma.
 */
#include <stdint.h>

static inline uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t synth_hash(uint64_t seed, uint64_t ctr) {
  return sm64_mix(seed + (ctr + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

static inline float synth_normal_one(uint64_t seed, uint64_t i, float c) {
  int64_t s = 0;
  for (int m = 0; m < 6; ++m) {
    uint64_t h = synth_hash(seed, 6ULL * i + (uint64_t)m);
    s += (int64_t)(h >> 40) + (int64_t)((h >> 16) & 0xFFFFFFULL);
  }
  int32_t z = (int32_t)(s - 6LL * 16777216LL);
  return (float)z * c;
}

/* out[i] = normal(seed, offset + i) * sigma for i in [0, n). */
void synth_normal_f32(float* out, uint64_t n, uint64_t seed, uint64_t offset,
                      float sigma, int nthreads) {
  const float c = sigma * 0x1p-24f;
  (void)nthreads;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
  for (int64_t i = 0; i < (int64_t)n; ++i)
    out[i] = synth_normal_one(seed, offset + (uint64_t)i, c);
}

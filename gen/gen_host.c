/* Host side of the seeded synthetic input generator (definition in
 * gen/__init__.py).  Multi-threaded fill of large host buffers; bit-identical
 * to the numpy and CUDA versions.  Holds none of the MoE method's arithmetic. */
#include <stdint.h>

static uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static float gen_value(uint64_t key, uint64_t i, float sigma) {
  const uint64_t r0 = splitmix64(key ^ (2ull * i));
  const uint64_t r1 = splitmix64(key ^ (2ull * i + 1ull));
  int s = 0;
  for (int j = 0; j < 6; ++j) {
    s += (int)((r0 >> (10 * j)) & 1023ull);
    s += (int)((r1 >> (10 * j)) & 1023ull);
  }
  const float z = (float)(s - 6138) / 1024.0f;
  return z * sigma;
}

__attribute__((visibility("default"))) void moegen_host_fill_f32(float* out, uint64_t seed, uint64_t tid,
                                                                  uint64_t start, uint64_t count, float sigma) {
  const uint64_t key = splitmix64(seed ^ (tid << 40));
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)count; ++i) out[i] = gen_value(key, start + (uint64_t)i, sigma);
}

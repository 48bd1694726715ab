// Device side of the seeded synthetic input generator (see gen/__init__.py for
// the definition).  Built into gen/libmoegen.so; used by the tests and the
// benchmark to fill large device buffers without a host round trip.  It is not
// part of the MoE library and holds none of the method's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float gen_value(uint64_t seed, uint64_t tid, uint64_t i, float sigma) {
  const uint64_t base = splitmix64(seed ^ (tid << 40));
  const uint64_t r0 = splitmix64(base ^ (2ull * i));
  const uint64_t r1 = splitmix64(base ^ (2ull * i + 1ull));
  int s = 0;
#pragma unroll
  for (int j = 0; j < 6; ++j) {
    s += (int)((r0 >> (10 * j)) & 1023ull);
    s += (int)((r1 >> (10 * j)) & 1023ull);
  }
  const float z = (float)(s - 6138) / 1024.0f;  // exact
  return __fmul_rn(z, sigma);                   // one IEEE multiply, never contracted
}

__global__ void fill_f32_kernel(float* out, uint64_t seed, uint64_t tid, uint64_t start,
                                uint64_t count, float sigma) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < count;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = gen_value(seed, tid, start + i, sigma);
}

__global__ void fill_bf16_kernel(__nv_bfloat16* out, uint64_t seed, uint64_t tid, uint64_t start,
                                 uint64_t count, float sigma) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < count;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(gen_value(seed, tid, start + i, sigma));
}

int grid_for(uint64_t count) {
  uint64_t g = (count + 255) / 256;
  if (g > 148ull * 32) g = 148ull * 32;
  if (g == 0) g = 1;
  return (int)g;
}

}  // namespace

#define MOEGEN_API __attribute__((visibility("default")))

extern "C" {

// Fill out[0..count) with fp32 values of elements [start, start+count) of tensor tid.
MOEGEN_API int moegen_fill_f32(float* out, uint64_t seed, uint64_t tid, uint64_t start, uint64_t count,
                    float sigma, cudaStream_t stream) {
  if (count == 0) return 0;
  fill_f32_kernel<<<grid_for(count), 256, 0, stream>>>(out, seed, tid, start, count, sigma);
  return (int)cudaGetLastError();
}

// Same as moegen_fill_f32, rounded to bf16 (round-to-nearest-even).
MOEGEN_API int moegen_fill_bf16(void* out, uint64_t seed, uint64_t tid, uint64_t start, uint64_t count,
                     float sigma, cudaStream_t stream) {
  if (count == 0) return 0;
  fill_bf16_kernel<<<grid_for(count), 256, 0, stream>>>((__nv_bfloat16*)out, seed, tid, start,
                                                        count, sigma);
  return (int)cudaGetLastError();
}

}  // extern "C"

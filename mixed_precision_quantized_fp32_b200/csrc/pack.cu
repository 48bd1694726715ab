// moe_pack kernels: group-wise quantization of fp32 expert weights into the
// packed layer buffer (the expert-packing step of the MoE mixed-precision
// quantization page, sec. 2.3 / 3.5; per-projection bit widths as on the
// AlphaQ page, sec. 4.2).  Every float operation that decides a code is one
// IEEE fp32 operation (explicit __fdiv_rn / __fmul_rn, rintf), so the codes
// are reproducible bit for bit.
#include <cuda_fp8.h>
#include <cuda_fp4.h>

#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

struct FmtArg {
  uint8_t v[3 * kMaxE];
};

// Header writer: one block.  Layout offsets are recomputed on the device from
// (E, H, F, fmt) with the same rule as the host size query.
__global__ void pack_header_kernel(uint8_t* out, int E, int H, int F, FmtArg fmt, int e0, int ne) {
  __shared__ uint64_t co[3 * kMaxE], so[3 * kMaxE];
  if (threadIdx.x == 0) layer_layout(E, H, F, fmt.v, co, so, nullptr);
  __syncthreads();
  uint32_t* w32 = (uint32_t*)out;
  for (int i = threadIdx.x; i < (int)(kHdrBytes / 4); i += blockDim.x) {
    const uint32_t byte = (uint32_t)i * 4u;
    if (byte < 32u) {
      uint32_t v = 0;
      if (byte == 0) v = kMagic;
      else if (byte == 4) v = 1u;
      else if (byte == 8) v = (uint32_t)E;
      else if (byte == 12) v = (uint32_t)H;
      else if (byte == 16) v = (uint32_t)F;
      w32[i] = v;
    } else if (byte < kOffCode) {
      const int j = (int)(byte - kOffFmt);
      uint32_t v = 0;
      for (int b = 0; b < 4; ++b) {
        const int f = j + b;
        if (f < 3 * E) v |= (uint32_t)fmt.v[f] << (8 * b);
      }
      w32[i] = v;
    } else if (byte < kOffScale) {
      const int j = (int)(byte - kOffCode) / 8, half = ((byte - kOffCode) / 4) & 1;
      const uint64_t v = j < 3 * E ? co[j] : 0u;
      w32[i] = half ? (uint32_t)(v >> 32) : (uint32_t)v;
    } else if (byte < kOffTscale) {
      const int j = (int)(byte - kOffScale) / 8, half = ((byte - kOffScale) / 4) & 1;
      const uint64_t v = j < 3 * E ? so[j] : 0u;
      w32[i] = half ? (uint32_t)(v >> 32) : (uint32_t)v;
    } else if (byte < kOffTscale + 3072u) {
      // tensor scales: integer entries of the packed experts are 0; NVFP4
      // entries are written by the amax kernels; other experts are untouched.
      const int j = (int)(byte - kOffTscale) / 4;
      const int e = j / 3;
      if (j >= 3 * E || (e >= e0 && e < e0 + ne && fmt.v[j] != MOE_FMT_NVFP4)) w32[i] = 0u;
    } else {
      w32[i] = 0u;
    }
  }
}

// ---------------------------------------------------------------- integer
// One thread per (output n, group g).  Threads of a warp take consecutive n
// so the packed words (n fastest) are written coalesced.
template <int BITS>
__global__ void pack_int_kernel(const float* __restrict__ W, int N, int K, uint32_t* __restrict__ codes,
                                uint16_t* __restrict__ scales) {
  constexpr int QMAX = (1 << (BITS - 1)) - 1;
  constexpr int OFF = 1 << (BITS - 1);
  const int G = K / 32;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)N * G) return;
  // tid -> (n-block, g, n%128)
  const int nl = (int)(tid & 127);
  const long long rest = tid >> 7;
  const int g = (int)(rest % G);
  const int nb = (int)(rest / G);
  const int n = nb * 128 + nl;
  const float4* src = reinterpret_cast<const float4*>(W + (size_t)n * K + (size_t)g * 32);
  float w[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = __ldg(src + i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  float amax = 0.0f;
  if (BITS == 1) {  // sign code: the scale is the mean |w| (fp32 sum in input order)
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = __fadd_rn(amax, fabsf(w[i]));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(w[i]));
  }
  __half sh = __float2half_rn(__fdiv_rn(amax, BITS == 1 ? 32.0f : (float)QMAX));
  uint16_t sbits = __half_as_ushort(sh);
  if ((sbits & 0x7FFFu) == 0x7C00u) sbits = 0x7BFFu;  // saturate the scale
  const float s = __half2float(__ushort_as_half(sbits));
  uint32_t u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (BITS == 1) {  // sign bit: u = (q + 1) / 2 with q = +1 for w >= 0
      u[i] = w[i] >= 0.0f ? 1u : 0u;
      continue;
    }
    int q = 0;
    if (s != 0.0f) {
      float r = rintf(__fdiv_rn(w[i], s));
      r = fminf(fmaxf(r, (float)-QMAX), (float)QMAX);
      q = (int)r;
    }
    u[i] = (uint32_t)(q + OFF);
  }
  // Inside a word, the two codes of a pair (2j, 2j+1) sit 16 bits apart, so a
  // mask of the shifted word yields both as the low bits of two half-words.
  const int k0 = g * 32;
  if (BITS == 1) {  // code 2j at bit j, code 2j+1 at bit 16+j
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) v |= (u[2 * j] << j) | (u[2 * j + 1] << (16 + j));
    codes[word_index(n, k0, K, 1, 0)] = v;
  } else if (BITS == 4) {
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t v = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) v |= (u[wd * 8 + 2 * j] << (4 * j)) | (u[wd * 8 + 2 * j + 1] << (16 + 4 * j));
      codes[word_index(n, k0, K, 4, wd)] = v;
    }
  } else {
#pragma unroll
    for (int wd = 0; wd < 2; ++wd) {
      uint32_t v = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v |= ((u[wd * 16 + 2 * j] & 3u) << (2 * j)) | ((u[wd * 16 + 2 * j + 1] & 3u) << (16 + 2 * j));
      codes[word_index(n, k0, K, BITS, wd)] = v;
    }
    if (BITS == 3) {  // bit 2 of pair m = 4c+j at bit 8*(c/2) + c%2 + 2j (low half: even code)
      uint32_t hi = 0;
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int c = m >> 2, pos = 8 * (c >> 1) + (c & 1) + 2 * (m & 3);
        hi |= (((u[2 * m] >> 2) & 1u) << pos) | (((u[2 * m + 1] >> 2) & 1u) << (16 + pos));
      }
      codes[word_index(n, k0, K, 3, 2)] = hi;
    }
  }
  scales[scale_index(n, g, G)] = sbits;
}

// ---------------------------------------------------------------- NVFP4
// amax of the whole matrix (non-negative floats order like their bit patterns).
__global__ void amax_kernel(const float* __restrict__ W, long long count, uint32_t* __restrict__ out) {
  float m = 0.0f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count / 4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// tscale = amax / (448*6), or 1 for an all-zero matrix.
__global__ void tscale_finalize_kernel(float* ts) {
  const float amax = ts[0];
  ts[0] = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// One thread per (output n, group of 32 inputs) = two blocks of 16.
__global__ void pack_nvfp4_kernel(const float* __restrict__ W, int N, int K, const float* __restrict__ ts,
                                  uint32_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int G = K / 32;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)N * G) return;
  const int nl = (int)(tid & 127);
  const long long rest = tid >> 7;
  const int g = (int)(rest % G);
  const int nb = (int)(rest / G);
  const int n = nb * 128 + nl;
  const float sT = *ts;
  const float4* src = reinterpret_cast<const float4*>(W + (size_t)n * K + (size_t)g * 32);
  float w[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = __ldg(src + i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  uint32_t c[32];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(w[16 * b + i]));
    const __nv_fp8_storage_t sb =
        __nv_cvt_float_to_fp8(__fdiv_rn(bmax, __fmul_rn(6.0f, sT)), __NV_SATFINITE, __NV_E4M3);
    const float denom = __fmul_rn(e4m3_value(sb), sT);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      c[16 * b + i] =
          (sb == 0) ? 0u
                    : (uint32_t)__nv_cvt_float_to_fp4(__fdiv_rn(w[16 * b + i], denom), __NV_E2M1,
                                                      cudaRoundNearest) & 15u;
    }
    scales[scale_index(n, 2 * g + b, K / 16)] = sb;
  }
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v |= c[wd * 8 + i] << (4 * i);
    codes[word_index(n, g * 32, K, 4, wd)] = v;
  }
}

cudaError_t launch_pack(const float* W, int e0, int ne, int E, int H, int F, const uint8_t* fmt_host,
                        uint8_t* out, const uint64_t* code_off, const uint64_t* scale_off,
                        cudaStream_t stream) {
  FmtArg fa;
  for (int i = 0; i < 3 * kMaxE; ++i) fa.v[i] = i < 3 * E ? fmt_host[i] : 0;
  pack_header_kernel<<<1, 512, 0, stream>>>(out, E, H, F, fa, e0, ne);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  for (int i = 0; i < ne; ++i) {
    const int e = e0 + i;
    for (int p = 0; p < 3; ++p) {
      int N, K;
      proj_shape(p, H, F, N, K);
      const float* w = W + ((size_t)i * 3 + p) * (size_t)H * F;
      const int f = fmt_host[e * 3 + p];
      uint32_t* codes = (uint32_t*)(out + code_off[e * 3 + p]);
      const long long threads = (long long)N * (K / 32);
      const int blocks = (int)((threads + 255) / 256);
      if (f == MOE_FMT_NVFP4) {
        float* ts = (float*)(out + kOffTscale) + (e * 3 + p);
        err = cudaMemsetAsync(ts, 0, sizeof(float), stream);
        if (err != cudaSuccess) return err;
        amax_kernel<<<148 * 8, 256, 0, stream>>>(w, (long long)N * K, (uint32_t*)ts);
        tscale_finalize_kernel<<<1, 1, 0, stream>>>(ts);
        pack_nvfp4_kernel<<<blocks, 256, 0, stream>>>(w, N, K, ts, codes, out + scale_off[e * 3 + p]);
      } else {
        uint16_t* sc = (uint16_t*)(out + scale_off[e * 3 + p]);
        if (f == MOE_FMT_INT4) pack_int_kernel<4><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc);
        else if (f == MOE_FMT_INT3) pack_int_kernel<3><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc);
        else if (f == MOE_FMT_INT1) pack_int_kernel<1><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc);
        else pack_int_kernel<2><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc);
      }
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
    }
  }
  return cudaSuccess;
}

}  // namespace moe

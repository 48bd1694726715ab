// NVFP4 activations (moe_weights.act = MOE_ACT_NVFP4): per-row quantization of
// the expert inputs x (per token) and of the SwiGLU outputs h (per sorted row)
// with the weights' NVFP4 rule, the row taking the place of the tensor
// ("quantized MoE LLM inference", NVFP4 remarks, for the format; MoE
// mixed-precision page sec. 2.1 for live per-token activation scales):
//   s  = amax(row) / 2688 in fp32 (1 for an all-zero row),
//   sb = e4m3(blockmax / (6*s)) per 16 inputs (round to nearest even, saturating),
//   v  = e2m1(a / (sb*s)) (round to nearest even, saturating; 0 where sb = 0).
// The arithmetic is the packing kernel's, step for step, so the codes are the
// same a CPU restatement of the rule gives.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

// Eight inputs starting at p as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// e2m1 pair (one byte, even code in the low nibble) -> exact f16x2 times the
// block scale (e2m1 x e4m3 has at most 6 significant bits: exact in fp16).
__device__ __forceinline__ uint32_t e2m1x2_scaled(uint32_t byte, __half2 sb2) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(r) : "r"(byte));
  __half2 h = __hmul2(*reinterpret_cast<__half2*>(&r), sb2);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace

// One warp per row of `src` [rows][K] (K a multiple of 128).  Outputs (each nullable):
//   codes [rows][K/2]  packed e2m1, code k in byte k/2 (even k in the low nibble)
//   sf    [rows][ld]   e4m3 block scales (ld >= K/16, a multiple of 16)
//   s     [rows]       row scales
//   bval  [rows][K]    fp16 block values e2m1(v)*sb (exact), for the decode GEMV
//   dbg_codes [rows][K] one code per byte; dbg_sf [rows][K/16]; dbg_s [rows]
template <typename Src>
__global__ void __launch_bounds__(256) act_quant_nvfp4_kernel(const Src* __restrict__ src, int rows, int K,
                                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                              int ld, float* __restrict__ s_out, __half* __restrict__ bval,
                                                              uint8_t* __restrict__ dbg_codes,
                                                              uint8_t* __restrict__ dbg_sf, float* __restrict__ dbg_s) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const Src* row = src + (size_t)r * K;
  float m = 0.0f;
  for (int c = lane; c < K / 8; c += 32) {
    float f[8];
    load8(row + 8 * c, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = (m == 0.0f) ? 1.0f : __fdiv_rn(m, 2688.0f);
  const float six_s = __fmul_rn(6.0f, s);
  for (int b = lane; b < K / 16; b += 32) {
    float f[16];
    load8(row + 16 * b, f);
    load8(row + 16 * b + 8, f + 8);
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(f[i]));
    const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(__fdiv_rn(bmax, six_s), __NV_SATFINITE, __NV_E4M3);
    const float denom = __fmul_rn(e4m3_value(sb), s);
    uint32_t c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      c[i] = (sb == 0) ? 0u
                       : (uint32_t)__nv_cvt_float_to_fp4(__fdiv_rn(f[i], denom), __NV_E2M1, cudaRoundNearest) & 15u;
    uint32_t p[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i >> 3] |= c[i] << (4 * (i & 7));
    if (codes) *reinterpret_cast<uint2*>(codes + (size_t)r * (K / 2) + 8 * b) = make_uint2(p[0], p[1]);
    if (sf) sf[(size_t)r * ld + b] = sb;
    if (dbg_sf) dbg_sf[(size_t)r * (K / 16) + b] = sb;
    if (dbg_codes) {
      uint32_t d[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 16; ++i) d[i >> 2] |= c[i] << (8 * (i & 3));
      *reinterpret_cast<uint4*>(dbg_codes + (size_t)r * K + 16 * b) = make_uint4(d[0], d[1], d[2], d[3]);
    }
    if (bval) {
      const __half_raw sr = __nv_cvt_fp8_to_halfraw(sb, __NV_E4M3);  // exact
      const __half2 sb2 = __halves2half2(__half(sr), __half(sr));
      uint32_t h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) h[j] = e2m1x2_scaled((p[j >> 2] >> (8 * (j & 3))) & 0xFFu, sb2);
      uint4* dst = reinterpret_cast<uint4*>(bval + (size_t)r * K + 16 * b);
      dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
      dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
  }
  if (lane == 0) {
    if (s_out) s_out[r] = s;
    if (dbg_s) dbg_s[r] = s;
  }
}

// Gather the NVFP4 codes and block scales of each sorted row's token (prefill:
// the FP4 GEMM's activation operand).  One thread per 16 bytes.
__global__ void gather_nvfp4_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                    const int32_t* __restrict__ perm, int R, int K, int ld, int k,
                                    uint8_t* __restrict__ codes_out, uint8_t* __restrict__ sf_out) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int per_row = K / 32 + ld / 16;  // 16-byte pieces: codes, then scales
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)R * per_row) return;
  const int r = (int)(i / per_row), c = (int)(i % per_row);
  const int t = perm[r] / k;
  if (c < K / 32) {
    reinterpret_cast<uint4*>(codes_out + (size_t)r * (K / 2))[c] =
        __ldg(reinterpret_cast<const uint4*>(codes + (size_t)t * (K / 2)) + c);
  } else {
    const int cs = c - K / 32;
    reinterpret_cast<uint4*>(sf_out + (size_t)r * ld)[cs] = __ldg(reinterpret_cast<const uint4*>(sf + (size_t)t * ld) + cs);
  }
}

// Gather each sorted row's token as fp16 block values (decode: the GEMV's
// activation operand), and zero the GEMV's work counters.  One thread per 16 inputs.
__global__ void gather_nvfp4_f16_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                        const int32_t* __restrict__ perm, int R, int K, int ld, int k,
                                        __half* __restrict__ xs, int32_t* counters, int n_counters) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)R * (K / 16)) return;
  const int r = (int)(i / (K / 16)), b = (int)(i % (K / 16));
  const int t = perm[r] / k;
  const uint2 p = __ldg(reinterpret_cast<const uint2*>(codes + (size_t)t * (K / 2)) + b);
  const __half_raw sr = __nv_cvt_fp8_to_halfraw(sf[(size_t)t * ld + b], __NV_E4M3);
  const __half2 sb2 = __halves2half2(__half(sr), __half(sr));
  const uint32_t pw[2] = {p.x, p.y};
  uint32_t h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) h[j] = e2m1x2_scaled((pw[j >> 2] >> (8 * (j & 3))) & 0xFFu, sb2);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)r * K + 16 * b);
  dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
  dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
}

cudaError_t launch_gather_nvfp4(const __nv_bfloat16* x, int T, int H, int k, bool tc, const Workspace& ws,
                                uint8_t* dbg_xq, uint8_t* dbg_xsb, float* dbg_sx, cudaStream_t stream) {
  const int R = T * k;
  launch_chained(act_quant_nvfp4_kernel<__nv_bfloat16>, dim3((T + 7) / 8), dim3(256), 0, stream, x, T, H, ws.xq, ws.xsf, ws.ldx, ws.sx,
                                                                         nullptr, dbg_xq, dbg_xsb, dbg_sx);
  if (tc) {
    const long long n = (long long)R * (H / 32 + ws.ldx / 16);
    launch_chained(gather_nvfp4_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream, ws.xq, ws.xsf, ws.perm, R, H, ws.ldx, k,
                                                                       ws.xs4, ws.xsf4);
  } else {
    const long long n = (long long)R * (H / 16);
    launch_chained(gather_nvfp4_f16_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream,
        ws.xq, ws.xsf, ws.perm, R, H, ws.ldx, k, (__half*)ws.xs, ws.counters, ws.counter_len);
  }
  return cudaGetLastError();
}

cudaError_t launch_act_quant_h_nvfp4(int R, int F, bool tc, const Workspace& ws, uint8_t* dbg_hq, uint8_t* dbg_hsb,
                                     float* dbg_sh, cudaStream_t stream) {
  launch_chained(act_quant_nvfp4_kernel<float>, dim3((R + 7) / 8), dim3(256), 0, stream,
      (const float*)ws.h, R, F, tc ? ws.hs4 : nullptr, tc ? ws.hsf4 : nullptr, ws.ldh, ws.sh,
      tc ? nullptr : (__half*)ws.hb, dbg_hq, dbg_hsb, dbg_sh);
  return cudaGetLastError();
}

}  // namespace moe

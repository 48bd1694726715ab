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
// (E, H, F, fmt) with the same rule as the host size query; fmt holds the host
// codes (the header stores their base formats).  With an outlier section it also
// writes the flag word, the section offset and the side-list table.
__global__ void pack_header_kernel(uint8_t* out, int E, int H, int F, FmtArg fmt, int e0, int ne) {
  __shared__ uint64_t co[3 * kMaxE], so[3 * kMaxE], side[3 * kMaxE];
  __shared__ uint8_t base[3 * kMaxE];
  __shared__ uint64_t sec;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3 * kMaxE; ++i) base[i] = (uint8_t)fmt_base(fmt.v[i]);
    uint64_t end = 0, total = 0;
    layer_layout(E, H, F, base, co, so, &end);
    sec = outlier_layout(E, H, F, fmt.v, end, side, &total);
  }
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
      else if (byte == kOffFlags) v = sec ? 1u : 0u;
      else if (byte == kOffOutSec) v = (uint32_t)sec;
      else if (byte == kOffOutSec + 4u) v = (uint32_t)(sec >> 32);
      w32[i] = v;
    } else if (byte < kOffCode) {
      const int j = (int)(byte - kOffFmt);
      uint32_t v = 0;
      for (int b = 0; b < 4; ++b) {
        const int f = j + b;
        if (f < 3 * E) v |= (uint32_t)base[f] << (8 * b);
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
      if (j >= 3 * E || (e >= e0 && e < e0 + ne && base[j] != MOE_FMT_NVFP4)) w32[i] = 0u;
    } else {
      w32[i] = 0u;
    }
  }
  if (sec) {
    uint64_t* table = (uint64_t*)(out + sec);
    for (int i = threadIdx.x; i < 3 * kMaxE; i += blockDim.x) table[i] = i < 3 * E ? side[i] : 0u;
  }
}

// ---------------------------------------------------------------- outliers
// Selection of the n_out largest |w| of one matrix (ties to the lower row-major
// index) as a predicate on (|w| bits, index): |w| > T, or |w| == T and index <= cut.
// T is found by an 8-bit radix select on the bit patterns of |w| (non-negative floats
// order like their bits); the scratch words hold its state:
//   meta[0] prefix, [1] mask, [2] elements still to take, [3] T, [4..5] cut (u64),
//   [8..] counts (256 digit bins, then per-chunk counts of the cut search).
struct OutSel {
  uint32_t T;
  unsigned long long cut;
  bool on;
};
__device__ __forceinline__ OutSel out_sel(const uint32_t* meta) {
  OutSel o;
  o.on = meta != nullptr;
  o.T = o.on ? meta[3] : 0u;
  o.cut = o.on ? ((unsigned long long)meta[5] << 32 | meta[4]) : 0ull;
  return o;
}
__device__ __forceinline__ bool out_is(const OutSel& o, float w, unsigned long long idx) {
  if (!o.on) return false;
  const uint32_t b = __float_as_uint(w) & 0x7FFFFFFFu;
  return b > o.T || (b == o.T && idx <= o.cut);
}

constexpr int kCutChunk = 65536;  // elements per chunk of the tie-cut search

__global__ void out_init_kernel(uint32_t* meta, uint32_t n_out) {
  for (int i = threadIdx.x; i < 8 + 256; i += blockDim.x) meta[i] = 0u;
  if (threadIdx.x == 0) {
    meta[2] = n_out;
    meta[3] = 0xFFFFFFFFu;  // no element is above T until the search ends (n_out == 0)
    meta[4] = 0xFFFFFFFFu;
    meta[5] = 0xFFFFFFFFu;
  }
}

// Histogram of the digit at `shift` among elements matching the prefix found so far.
__global__ void out_hist_kernel(const float* __restrict__ W, long long count, uint32_t* meta, int shift) {
  __shared__ uint32_t h[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  const uint32_t prefix = meta[0], mask = meta[1];
  if (meta[2] != 0u)
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count; i += (long long)gridDim.x * blockDim.x) {
      const uint32_t b = __float_as_uint(__ldg(W + i)) & 0x7FFFFFFFu;
      if ((b & mask) == prefix) atomicAdd(&h[(b >> shift) & 0xFFu], 1u);
    }
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    if (h[i]) atomicAdd(&meta[8 + i], h[i]);
}

// One thread: pick the digit holding the remaining count, from the top.
__global__ void out_pick_kernel(uint32_t* meta, int shift) {
  uint32_t need = meta[2];
  if (need == 0u) return;
  uint32_t acc = 0u;
  int d = 255;
  for (; d > 0; --d) {
    if (acc + meta[8 + d] >= need) break;
    acc += meta[8 + d];
  }
  meta[0] |= (uint32_t)d << shift;
  meta[1] |= 0xFFu << shift;
  meta[2] = need - acc;  // elements equal to the prefix so far still to take
  for (int i = 0; i < 256; ++i) meta[8 + i] = 0u;
  if (shift == 0) meta[3] = meta[0];
}

// Per chunk: count of elements whose |w| equals T.
__global__ void out_cut_count_kernel(const float* __restrict__ W, long long count, uint32_t* meta) {
  __shared__ uint32_t c;
  if (threadIdx.x == 0) c = 0u;
  __syncthreads();
  const uint32_t T = meta[3];
  const long long base = (long long)blockIdx.x * kCutChunk;
  uint32_t mine = 0;
  if (meta[2] != 0u)
    for (long long i = base + threadIdx.x; i < base + kCutChunk && i < count; i += blockDim.x)
      mine += (__float_as_uint(__ldg(W + i)) & 0x7FFFFFFFu) == T;
  if (mine) atomicAdd(&c, mine);
  __syncthreads();
  if (threadIdx.x == 0) meta[8 + blockIdx.x] = c;
}

// One block: the chunk holding the m-th element equal to T, then its index by an
// ordered scan of that chunk.
__global__ void __launch_bounds__(1024) out_cut_find_kernel(const float* __restrict__ W, long long count,
                                                            uint32_t* meta, int nchunks) {
  __shared__ uint32_t warp_c[32];
  __shared__ long long s_base;
  __shared__ uint32_t s_need;
  if (meta[2] == 0u) return;
  if (threadIdx.x == 0) {
    uint32_t need = meta[2];
    int c = 0;
    for (; c < nchunks - 1; ++c) {
      if (meta[8 + c] >= need) break;
      need -= meta[8 + c];
    }
    s_base = (long long)c * kCutChunk;
    s_need = need;
  }
  __syncthreads();
  const uint32_t T = meta[3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t need = s_need;
  for (long long t0 = s_base; t0 < s_base + kCutChunk && t0 < count; t0 += blockDim.x) {
    const long long i = t0 + threadIdx.x;
    const bool eq = i < count && (__float_as_uint(__ldg(W + i)) & 0x7FFFFFFFu) == T;
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_c[warp] = __popc(bal);
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      if (w < warp) before += warp_c[w];
      total += warp_c[w];
    }
    const uint32_t rank = before + __popc(bal & ((1u << lane) - 1u));  // equal elements before i in this tile
    if (eq && rank + 1u == need) {
      meta[4] = (uint32_t)i;
      meta[5] = (uint32_t)((unsigned long long)i >> 32);
    }
    __syncthreads();
    if (total >= need) break;  // found in this tile (block-uniform)
    need -= total;
  }
}

// One warp per row: selected elements of row n -> counts[n + 1] (counts[0] = 0).
__global__ void out_row_count_kernel(const float* __restrict__ W, int N, int K, const uint32_t* meta,
                                     uint32_t* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;
  const OutSel o = out_sel(meta);
  uint32_t c = 0;
  for (int k = lane; k < K; k += 32) c += out_is(o, __ldg(W + (size_t)n * K + k), (unsigned long long)n * K + k);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
  if (lane == 0) row_ptr[n + 1] = c;
  if (n == 0 && lane == 0) row_ptr[0] = 0u;
}

// One block: inclusive scan of counts[1..N] into row offsets.
__global__ void __launch_bounds__(1024) out_row_scan_kernel(uint32_t* __restrict__ row_ptr, int N) {
  __shared__ uint32_t warp_s[32];
  __shared__ uint32_t carry;
  if (threadIdx.x == 0) carry = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t0 = 1; t0 <= N; t0 += blockDim.x) {
    const int i = t0 + threadIdx.x;
    uint32_t v = i <= N ? row_ptr[i] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) warp_s[warp] = v;
    __syncthreads();
    uint32_t add = carry;
    for (int w = 0; w < warp; ++w) add += warp_s[w];
    if (i <= N) row_ptr[i] = v + add;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = v + add;
    __syncthreads();
  }
}

// One warp per row: the row's outliers in column order.  Entry = column | fp16
// residual << 16; the residual is w - dequant at that position rounded once to
// fp16 (the difference taken in double): w itself for every format with a zero
// code, w - s for the 1-bit sign code (a zeroed weight reads +s).
__global__ void out_fill_kernel(const float* __restrict__ W, int N, int K, const uint32_t* meta,
                                const uint32_t* __restrict__ row_ptr, uint32_t* __restrict__ entries,
                                const uint16_t* __restrict__ scales, bool sign_code) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;
  const OutSel o = out_sel(meta);
  uint32_t pos = row_ptr[n];
  for (int k0 = 0; k0 < K; k0 += 32) {
    const int k = k0 + lane;
    const float w = __ldg(W + (size_t)n * K + k);
    const bool sel = out_is(o, w, (unsigned long long)n * K + k);
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      double d = (double)w;
      if (sign_code) d = __dsub_rn(d, (double)__half2float(__ushort_as_half(scales[scale_index(n, k >> 5, K / 32)])));
      const uint16_t r = __half_as_ushort(__double2half(d));
      entries[pos + __popc(bal & ((1u << lane) - 1u))] = (uint32_t)k | ((uint32_t)r << 16);
    }
    pos += __popc(bal);
  }
}


// ---------------------------------------------------------------- integer
// One thread per (output n, group g).  Threads of a warp take consecutive n
// so the packed words (n fastest) are written coalesced.
template <int BITS>
__global__ void pack_int_kernel(const float* __restrict__ W, int N, int K, uint32_t* __restrict__ codes,
                                uint16_t* __restrict__ scales, const uint32_t* out_meta) {
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
  if (out_meta) {  // outliers leave the grid: quantize the matrix with them zeroed
    const OutSel o = out_sel(out_meta);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (out_is(o, w[i], (unsigned long long)n * K + g * 32 + i)) w[i] = 0.0f;
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
__global__ void amax_kernel(const float* __restrict__ W, long long count, uint32_t* __restrict__ out,
                            const uint32_t* out_meta) {
  const OutSel o = out_sel(out_meta);
  float m = 0.0f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count / 4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(W) + i);
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (!out_is(o, f[j], (unsigned long long)(4 * i + j))) m = fmaxf(m, fabsf(f[j]));
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
                                  uint32_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                  const uint32_t* out_meta) {
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
  if (out_meta) {  // outliers leave the grid: quantize the matrix with them zeroed
    const OutSel o = out_sel(out_meta);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (out_is(o, w[i], (unsigned long long)n * K + g * 32 + i)) w[i] = 0.0f;
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

// Outlier selection of one matrix: T and the tie cut into the scratch's meta words.
cudaError_t select_outliers(const float* w, int N, int K, uint32_t* meta, cudaStream_t stream) {
  const long long count = (long long)N * K;
  const uint32_t n_out = (uint32_t)outlier_count(N, K);
  out_init_kernel<<<1, 256, 0, stream>>>(meta, n_out);
  for (int shift = 24; shift >= 0; shift -= 8) {
    out_hist_kernel<<<148 * 4, 256, 0, stream>>>(w, count, meta, shift);
    out_pick_kernel<<<1, 1, 0, stream>>>(meta, shift);
  }
  const int nchunks = (int)((count + kCutChunk - 1) / kCutChunk);
  if (nchunks > 65536) return cudaErrorInvalidValue;
  out_cut_count_kernel<<<nchunks, 256, 0, stream>>>(w, count, meta);
  out_cut_find_kernel<<<1, 1024, 0, stream>>>(w, count, meta, nchunks);
  return cudaGetLastError();
}

cudaError_t launch_pack(const float* W, int e0, int ne, int E, int H, int F, const uint8_t* fmt_host,
                        uint8_t* out, const uint64_t* code_off, const uint64_t* scale_off, uint64_t out_sec,
                        const uint64_t* side_off, cudaStream_t stream) {
  FmtArg fa;
  for (int i = 0; i < 3 * kMaxE; ++i) fa.v[i] = i < 3 * E ? fmt_host[i] : 0;
  pack_header_kernel<<<1, 512, 0, stream>>>(out, E, H, F, fa, e0, ne);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  uint32_t* meta = out_sec ? (uint32_t*)(out + out_sec + kOutTableBytes) : nullptr;  // selection scratch
  for (int i = 0; i < ne; ++i) {
    const int e = e0 + i;
    for (int p = 0; p < 3; ++p) {
      int N, K;
      proj_shape(p, H, F, N, K);
      const float* w = W + ((size_t)i * 3 + p) * (size_t)H * F;
      const int f = fmt_base(fmt_host[e * 3 + p]);
      const bool iso = fmt_outliers(fmt_host[e * 3 + p]);
      const uint32_t* om = iso ? meta : nullptr;
      if (iso && (err = select_outliers(w, N, K, meta, stream)) != cudaSuccess) return err;
      uint32_t* codes = (uint32_t*)(out + code_off[e * 3 + p]);
      const long long threads = (long long)N * (K / 32);
      const int blocks = (int)((threads + 255) / 256);
      if (f == MOE_FMT_NVFP4) {
        float* ts = (float*)(out + kOffTscale) + (e * 3 + p);
        err = cudaMemsetAsync(ts, 0, sizeof(float), stream);
        if (err != cudaSuccess) return err;
        amax_kernel<<<148 * 8, 256, 0, stream>>>(w, (long long)N * K, (uint32_t*)ts, om);
        tscale_finalize_kernel<<<1, 1, 0, stream>>>(ts);
        pack_nvfp4_kernel<<<blocks, 256, 0, stream>>>(w, N, K, ts, codes, out + scale_off[e * 3 + p], om);
      } else {
        uint16_t* sc = (uint16_t*)(out + scale_off[e * 3 + p]);
        if (f == MOE_FMT_INT4) pack_int_kernel<4><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc, om);
        else if (f == MOE_FMT_INT3) pack_int_kernel<3><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc, om);
        else if (f == MOE_FMT_INT1) pack_int_kernel<1><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc, om);
        else pack_int_kernel<2><<<blocks, 256, 0, stream>>>(w, N, K, codes, sc, om);
      }
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
      if (iso) {  // the side list: row offsets, then the entries in (row, column) order
        uint32_t* row_ptr = (uint32_t*)(out + side_off[e * 3 + p]);
        const int rb = (N + 7) / 8;
        out_row_count_kernel<<<rb, 256, 0, stream>>>(w, N, K, meta, row_ptr);
        out_row_scan_kernel<<<1, 1024, 0, stream>>>(row_ptr, N);
        out_fill_kernel<<<rb, 256, 0, stream>>>(w, N, K, meta, row_ptr, row_ptr + N + 1,
                                                (const uint16_t*)(out + scale_off[e * 3 + p]), f == MOE_FMT_INT1);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
      }
    }
  }
  return cudaSuccess;
}

}  // namespace moe

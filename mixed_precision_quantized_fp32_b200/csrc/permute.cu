// Token permutation by expert (histogram -> exclusive scan -> stable scatter),
// the gather of activation rows into expert-sorted order, and the per-row
// dynamic FP8 activation quantization of NVFP4 layers (MoE mixed-precision
// page sec. 2.1: per-token scales from the live min/max; e4m3, amax/448).
#include <cuda_fp8.h>

#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kPermBlock = 1024;

// Pass 1: per block of 1024 entries (t*k+j order), the expert histogram and the
// stable rank of each entry among the block's entries of the same expert.
__global__ void __launch_bounds__(kPermBlock) perm_count_kernel(const int32_t* __restrict__ idx, int R,
                                                                int E, int32_t* __restrict__ blk_hist,
                                                                int32_t* __restrict__ rank) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  __shared__ int32_t wcnt[kPermBlock / 32][kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (kPermBlock / 32) * kMaxE; i += kPermBlock) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int i = blockIdx.x * kPermBlock + tid;
  const bool valid = i < R;
  const int e = valid ? idx[i] : -1;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int rw = __popc(same & ((1u << lane) - 1u));
  if (valid && rw == 0) wcnt[warp][e] = __popc(same);
  __syncthreads();
  if (valid) {
    int r = rw;
    for (int w = 0; w < warp; ++w) r += wcnt[w][e];
    rank[i] = r;
  }
  for (int ee = tid; ee < E; ee += kPermBlock) {
    int s = 0;
    for (int w = 0; w < kPermBlock / 32; ++w) s += wcnt[w][ee];
    blk_hist[(size_t)blockIdx.x * E + ee] = s;
  }
}

// Pass 2 (one block of 256 threads, thread e = expert e): per-expert totals,
// exclusive offsets, per-block bases, and the list of (expert, first row,
// rows) chunks of at most `chunk_rows` rows that the expert GEMMs walk.
__global__ void __launch_bounds__(256) perm_scan_kernel(int32_t* __restrict__ blk_hist, int nblk, int E,
                                                        int R, int chunk_rows, int32_t* __restrict__ counts,
                                                        int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ chunks,
                                                        int32_t* __restrict__ chunk_count,
                                                        int32_t* __restrict__ dbg_counts) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  __shared__ int32_t s_cnt[kMaxE], s_off[kMaxE + 1], s_nc[kMaxE], s_cstart[kMaxE + 1];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int v = blk_hist[(size_t)b * E + e];
      blk_hist[(size_t)b * E + e] = total;
      total += v;
    }
  }
  s_cnt[e] = (e < E) ? total : 0;
  s_nc[e] = (e < E) ? (total + chunk_rows - 1) / chunk_rows : 0;
  __syncthreads();
  if (e == 0) {
    int run = 0, crun = 0;
    for (int j = 0; j < E; ++j) {
      s_off[j] = run;
      run += s_cnt[j];
      s_cstart[j] = crun;
      crun += s_nc[j];
    }
    s_off[E] = run;
    s_cstart[E] = crun;
    *chunk_count = crun;
    offsets[E] = run;
  }
  __syncthreads();
  if (e < E) {
    counts[e] = total;
    offsets[e] = s_off[e];
    if (dbg_counts) dbg_counts[e] = total;
    for (int b = 0; b < nblk; ++b) blk_hist[(size_t)b * E + e] += s_off[e];
    for (int c = 0; c < s_nc[e]; ++c) {
      const int row0 = c * chunk_rows;
      int32_t* ch = chunks + 3 * (size_t)(s_cstart[e] + c);
      ch[0] = e;
      ch[1] = s_off[e] + row0;
      ch[2] = min(chunk_rows, total - row0);
    }
  }
}

// Pass 3: row = block base of the expert + stable rank; perm[row] = entry, inv[entry] = row.
__global__ void __launch_bounds__(kPermBlock) perm_scatter_kernel(const int32_t* __restrict__ idx, int R,
                                                                  int E, const int32_t* __restrict__ blk_hist,
                                                                  const int32_t* __restrict__ rank,
                                                                  int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ inv,
                                                                  int32_t* __restrict__ dbg_perm,
                                                                  int32_t* __restrict__ dbg_inv) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int i = blockIdx.x * kPermBlock + threadIdx.x;
  if (i >= R) return;
  const int e = idx[i];
  const int row = blk_hist[(size_t)blockIdx.x * E + e] + rank[i];
  perm[row] = i;
  inv[i] = row;
  if (dbg_perm) dbg_perm[row] = i;
  if (dbg_inv) dbg_inv[i] = row;
}

// All of the permutation in one block when T*k <= 1024 (decode batches): the
// histogram and stable ranks of pass 1, the scan and chunk list of pass 2 and
// the scatter of pass 3, with the same results.
__global__ void __launch_bounds__(kPermBlock) perm_small_kernel(const int32_t* __restrict__ idx, int R, int E,
                                                                int chunk_rows, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ chunks,
                                                                int32_t* __restrict__ chunk_count,
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                int32_t* __restrict__ dbg_counts,
                                                                int32_t* __restrict__ dbg_perm,
                                                                int32_t* __restrict__ dbg_inv) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  __shared__ int32_t wcnt[kPermBlock / 32][kMaxE];
  __shared__ int32_t s_off[kMaxE + 1], s_cstart[kMaxE + 1], s_cnt[kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (kPermBlock / 32) * kMaxE; i += kPermBlock) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const bool valid = tid < R;
  const int e = valid ? idx[tid] : -1;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int rw = __popc(same & ((1u << lane) - 1u));
  if (valid && rw == 0) wcnt[warp][e] = __popc(same);
  __syncthreads();
  int rank = rw;
  if (valid)
    for (int w = 0; w < warp; ++w) rank += wcnt[w][e];
  for (int ee = tid; ee < E; ee += kPermBlock) {
    int total = 0;
    for (int w = 0; w < kPermBlock / 32; ++w) total += wcnt[w][ee];
    s_cnt[ee] = total;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0, crun = 0;
    for (int j = 0; j < E; ++j) {
      s_off[j] = run;
      run += s_cnt[j];
      s_cstart[j] = crun;
      crun += (s_cnt[j] + chunk_rows - 1) / chunk_rows;
    }
    s_off[E] = run;
    *chunk_count = crun;
    offsets[E] = run;
  }
  __syncthreads();
  for (int ee = tid; ee < E; ee += kPermBlock) {
    const int total = s_cnt[ee];
    counts[ee] = total;
    offsets[ee] = s_off[ee];
    if (dbg_counts) dbg_counts[ee] = total;
    for (int c = 0; c * chunk_rows < total; ++c) {
      int32_t* ch = chunks + 3 * (size_t)(s_cstart[ee] + c);
      ch[0] = ee;
      ch[1] = s_off[ee] + c * chunk_rows;
      ch[2] = min(chunk_rows, total - c * chunk_rows);
    }
  }
  if (valid) {
    const int row = s_off[e] + rank;
    perm[row] = tid;
    inv[tid] = row;
    if (dbg_perm) dbg_perm[row] = tid;
    if (dbg_inv) dbg_inv[tid] = row;
  }
}

// Zero the decode GEMV's work counters (the workspace starts undefined); called
// by one block.
__device__ __forceinline__ void zero_counters(int32_t* counters, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) counters[i] = 0;
}

// Power-of-two prescale that brings a row with max |value| m into fp16 range:
// 1 while m < 2^15, else 2^-e with m * 2^-e in [2^14, 2^15).  Scaling by a power
// of two is exact (values far below m may round into the fp16 subnormals, an
// error far below the row's largest term).
__device__ __forceinline__ int prescale_exp(float m) {
  if (!(m >= 32768.0f)) return 0;
  return (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127 - 14;
}

// Gather x rows into expert-sorted order as fp16 (integer-format layers), with
// the sum of every group of 32 fp16 values (fp32) for the decode GEMV's code
// offset term (xsum may be null).  bf16 covers a far wider range than fp16, so
// a token whose max |x| reaches 2^15 is stored as x * 2^-e and its row's
// xinv = 2^e restores the scale after the gate/up sums (xinv = 1 otherwise, and
// the stored values are exactly fp16(x)).  blockDim.x is 128 and H a multiple
// of 128, so the four threads of a group sit in one warp at every step.
__global__ void __launch_bounds__(128) gather_f16_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const int32_t* __restrict__ perm, int R, int H, int k,
                                                         __half* __restrict__ xs, float* __restrict__ xsum,
                                                         float* __restrict__ xinv, int32_t* counters,
                                                         int n_counters) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  __shared__ float s_max[4];
  if (blockIdx.x == 0 && blockIdx.y == 0) zero_counters(counters, n_counters);
  const int r = blockIdx.x;
  const int t = perm[r] / k;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)r * H);
  // max |x| of the whole token row (every column block reads it; the second
  // block's reads hit the cache)
  float m = 0.0f;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = __ldg(src + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      m = fmaxf(m, fmaxf(__uint_as_float((w[i] << 16) & 0x7FFF0000u), __uint_as_float(w[i] & 0x7FFF0000u)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  m = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
  const int e = prescale_exp(m);
  const float sc = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e (e <= 114)
  if (xinv && blockIdx.y == 0 && threadIdx.x == 0) xinv[r] = __uint_as_float((uint32_t)(127 + e) << 23);
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < H / 8; c += gridDim.y * blockDim.x) {
    const uint4 v = __ldg(src + c);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint4 o;
    __half2* h2 = reinterpret_cast<__half2*>(&o);
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(b2[i]);
      if (e) {
        f.x *= sc;
        f.y *= sc;
      }
      h2[i] = __float22half2_rn(f);
      const float2 g = __half22float2(h2[i]);
      sum += g.x + g.y;
    }
    dst[c] = o;
    const unsigned act = __activemask();  // whole groups of four lanes (H/8 is a multiple of 16)
    sum += __shfl_xor_sync(act, sum, 1);
    sum += __shfl_xor_sync(act, sum, 2);
    if (xsum && (c & 3) == 0) xsum[(size_t)r * (H / 32) + c / 4] = sum;
  }
}

// Per-token e4m3 codes of x: s = amax/448 (1 if amax == 0); q = e4m3(x/s), RNE,
// saturating.  One warp per token; H is a multiple of 128.
__global__ void act_quant_x_kernel(const __nv_bfloat16* __restrict__ x, int T, int H, uint8_t* __restrict__ xq,
                                   float* __restrict__ sx, uint8_t* __restrict__ dbg_xq,
                                   float* __restrict__ dbg_sx) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint2* xr = reinterpret_cast<const uint2*>(x + (size_t)t * H);  // 4 bf16 per load
  float m = 0.0f;
  for (int c = lane; c < H / 4; c += 32) {
    const uint2 v = __ldg(xr + c);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x), b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(__low2float(a)), fabsf(__high2float(a))), fmaxf(fabsf(__low2float(b)), fabsf(__high2float(b)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = (m == 0.0f) ? 1.0f : __fdiv_rn(m, 448.0f);
  for (int c = lane; c < H / 4; c += 32) {
    const uint2 v = __ldg(xr + c);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x), b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    const float f[4] = {__low2float(a), __high2float(a), __low2float(b), __high2float(b)};
    uint32_t q = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(f[i], s), __NV_SATFINITE, __NV_E4M3) << (8 * i);
    reinterpret_cast<uint32_t*>(xq + (size_t)t * H)[c] = q;
    if (dbg_xq) reinterpret_cast<uint32_t*>(dbg_xq + (size_t)t * H)[c] = q;
  }
  if (lane == 0) {
    sx[t] = s;
    if (dbg_sx) dbg_sx[t] = s;
  }
}

// Gather e4m3 activation codes into sorted rows as exact fp16 values: one
// thread per 16 codes (hardware e4m3x2 -> f16x2 conversion).
__global__ void gather_fp8_kernel(const uint8_t* __restrict__ xq, const int32_t* __restrict__ perm, int R,
                                  int H, int k, __half* __restrict__ xs, int32_t* counters, int n_counters) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  if (blockIdx.x == 0) zero_counters(counters, n_counters);
  const int per_row = H / 16;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)R * per_row) return;
  const int r = (int)(i / per_row), c = (int)(i % per_row);
  const int t = perm[r] / k;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(xq + (size_t)t * H) + c);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] >> 16), __NV_E4M3);
    o[2 * j] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
    o[2 * j + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)r * H) + 2 * c;
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// Per-row e4m3 codes of the SwiGLU output (NVFP4 layers) and their exact fp16
// values.  One warp per row; F is a multiple of 128.
__global__ void act_quant_h_kernel(const float* __restrict__ h, int R, int F, uint8_t* __restrict__ hq,
                                   float* __restrict__ sh, __half* __restrict__ hb,
                                   uint8_t* __restrict__ dbg_hq, float* __restrict__ dbg_sh) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= R) return;
  const float4* hr = reinterpret_cast<const float4*>(h + (size_t)r * F);
  float m = 0.0f;
  for (int c = lane; c < F / 4; c += 32) {
    const float4 v = __ldg(hr + c);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = (m == 0.0f) ? 1.0f : __fdiv_rn(m, 448.0f);
  for (int c = lane; c < F / 4; c += 32) {
    const float4 v = __ldg(hr + c);
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint32_t q = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(f[i], s), __NV_SATFINITE, __NV_E4M3) << (8 * i);
    reinterpret_cast<uint32_t*>(hq + (size_t)r * F)[c] = q;
    if (dbg_hq) reinterpret_cast<uint32_t*>(dbg_hq + (size_t)r * F)[c] = q;
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(q & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(q >> 16), __NV_E4M3);
    reinterpret_cast<uint2*>(hb + (size_t)r * F)[c] =
        make_uint2((uint32_t)lo.x | ((uint32_t)lo.y << 16), (uint32_t)hi.x | ((uint32_t)hi.y << 16));
  }
  if (lane == 0) {
    sh[r] = s;
    if (dbg_sh) dbg_sh[r] = s;
  }
}

cudaError_t launch_permute(int T, int k, int E, int chunk_rows, const Workspace& ws, int32_t* dbg_counts,
                           int32_t* dbg_perm, int32_t* dbg_inv, cudaStream_t stream) {
  const int R = T * k;
  const int nblk = (R + kPermBlock - 1) / kPermBlock;
  if (nblk == 1) {
    launch_chained(perm_small_kernel, dim3(1), dim3(kPermBlock), 0, stream, ws.idx, R, E, chunk_rows, ws.counts, ws.offsets, ws.chunks,
                                                    ws.chunk_count, ws.perm, ws.inv, dbg_counts, dbg_perm, dbg_inv);
    return cudaGetLastError();
  }
  launch_chained(perm_count_kernel, dim3(nblk), dim3(kPermBlock), 0, stream, ws.idx, R, E, ws.blk_hist, ws.rank);
  launch_chained(perm_scan_kernel, dim3(1), dim3(256), 0, stream, ws.blk_hist, nblk, E, R, chunk_rows, ws.counts, ws.offsets,
                                          ws.chunks, ws.chunk_count, dbg_counts);
  launch_chained(perm_scatter_kernel, dim3(nblk), dim3(kPermBlock), 0, stream, ws.idx, R, E, ws.blk_hist, ws.rank, ws.perm, ws.inv,
                                                       dbg_perm, dbg_inv);
  return cudaGetLastError();
}

cudaError_t launch_gather(const __nv_bfloat16* x, int T, int H, int k, bool fp4, const Workspace& ws,
                          uint8_t* dbg_xq, float* dbg_sx, cudaStream_t stream) {
  const int R = T * k;
  if (fp4) {
    launch_chained(act_quant_x_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, x, T, H, ws.xq, ws.sx, dbg_xq, dbg_sx);
    const long long n = (long long)R * (H / 16);
    launch_chained(gather_fp8_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream, ws.xq, ws.perm, R, H, k, (__half*)ws.xs,
                                                                     ws.counters, ws.counter_len);
  } else {
    int ny = R < 512 ? (H / 8 + 127) / 128 : 1;  // column blocks: more parallelism for few rows
    if (ny > 8) ny = 8;
    launch_chained(gather_f16_kernel, dim3(R, ny), dim3(128), 0, stream, x, ws.perm, R, H, k, (__half*)ws.xs, ws.xsum, ws.xinv,
                                                       ws.counters, ws.counter_len);
  }
  return cudaGetLastError();
}

cudaError_t launch_act_quant_h(int R, int F, const Workspace& ws, uint8_t* dbg_hq, float* dbg_sh,
                               cudaStream_t stream) {
  launch_chained(act_quant_h_kernel, dim3((R + 7) / 8), dim3(256), 0, stream, (const float*)ws.h, R, F, ws.hq, ws.sh, (__half*)ws.hb,
                                                      dbg_hq, dbg_sh);
  return cudaGetLastError();
}

}  // namespace moe

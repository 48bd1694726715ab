// Router (fp32, never quantized: MoE mixed-precision page sec. 2.1) and top-k
// with a softmax over the chosen k (expert-routing section of the quantized
// MoE inference page).
#include <cfloat>
#include <climits>

#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

// ---------------------------------------------------------------- router, few tokens
// One warp per (token, expert) dot product; lanes stride over H with 8-byte
// bf16 and 16-byte fp32 loads.  Used when T or E is small.
__global__ void router_warp_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ Wr,
                                   const float* __restrict__ b, int T, int H, int E,
                                   float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.y * (blockDim.x >> 5) + warp;
  const int t = blockIdx.x;
  if (e >= E) return;
  const __nv_bfloat16* xr = x + (size_t)t * H;
  const float* wr = Wr + (size_t)e * H;
  float acc = 0.0f;
  for (int h = lane * 4; h < H; h += 128) {
    const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + h));
    const float4 wv = __ldg(reinterpret_cast<const float4*>(wr + h));
    const __nv_bfloat162 x01 = *reinterpret_cast<const __nv_bfloat162*>(&xv.x);
    const __nv_bfloat162 x23 = *reinterpret_cast<const __nv_bfloat162*>(&xv.y);
    acc = fmaf(__low2float(x01), wv.x, acc);
    acc = fmaf(__high2float(x01), wv.y, acc);
    acc = fmaf(__low2float(x23), wv.z, acc);
    acc = fmaf(__high2float(x23), wv.w, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) logits[(size_t)t * E + e] = b ? acc + b[e] : acc;
}

// ---------------------------------------------------------------- router, many tokens
// Tiled fp32 GEMM: block tile 64 tokens x TE experts, k-tile 32; 256 threads,
// each computing 4 tokens x TE/16 experts.  Each k-tile is summed on its own and
// the tile sums are added with Kahan compensation, so the rounding error stays
// near that of a pairwise sum even for H = 12288.
template <int TE>
__global__ void __launch_bounds__(256) router_tile_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ Wr,
                                                          const float* __restrict__ b, int T, int H,
                                                          int E, float* __restrict__ logits) {
  constexpr int TT = 64, BK = 32, PE = TE / 16;
  __shared__ float xs[BK][TT + 4];
  __shared__ float ws[BK][TE + 4];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * TT, e0 = blockIdx.y * TE;
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][PE], comp[4][PE];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < PE; ++j) acc[i][j] = comp[i][j] = 0.0f;

  for (int k0 = 0; k0 < H; k0 += BK) {
    {  // x tile: 64 tokens x 32 h = 256 chunks of 8 bf16
      const int tt = tid >> 2, hh = (tid & 3) * 8;
      const int t = t0 + tt;
      float v[8];
      if (t < T) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + k0 + hh));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = __low2float(p2[i]);
          v[2 * i + 1] = __high2float(p2[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[hh + i][tt] = v[i];
    }
    for (int c = tid; c < TE * (BK / 4); c += 256) {  // Wr tile: TE experts x 32 h
      const int ee = c / (BK / 4), hh = (c % (BK / 4)) * 4;
      const int e = e0 + ee;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) v = __ldg(reinterpret_cast<const float4*>(Wr + (size_t)e * H + k0 + hh));
      ws[hh][ee] = v.x;
      ws[hh + 1][ee] = v.y;
      ws[hh + 2][ee] = v.z;
      ws[hh + 3][ee] = v.w;
    }
    __syncthreads();
    float part[4][PE];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < PE; ++j) part[i][j] = 0.0f;
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], w[PE];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < PE; ++j) w[j] = ws[kk][tx * PE + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < PE; ++j) part[i][j] = fmaf(a[i], w[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < PE; ++j) {  // Kahan: acc += part
        const float y = __fsub_rn(part[i][j], comp[i][j]);
        const float t = __fadd_rn(acc[i][j], y);
        comp[i][j] = __fsub_rn(__fsub_rn(t, acc[i][j]), y);
        acc[i][j] = t;
      }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < PE; ++j) {
      const int e = e0 + tx * PE + j;
      if (e < E) logits[(size_t)t * E + e] = b ? acc[i][j] + b[e] : acc[i][j];
    }
  }
}

// ---------------------------------------------------------------- top-k + softmax
// One warp per token.  Expert e lives in lane e%32, slot e/32.  k passes of a
// warp-wide arg-max over the experts not chosen yet; ties go to the lower
// expert index; NaN ranks below every number.
__global__ void topk_softmax_kernel(const float* __restrict__ logits, int T, int E, int k,
                                    int32_t* __restrict__ idx, float* __restrict__ wts,
                                    int32_t* __restrict__ dbg_idx, float* __restrict__ dbg_w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    float l = (e < E) ? logits[(size_t)t * E + e] : -INFINITY;
    v[i] = (l != l) ? -INFINITY : l;
  }
  uint32_t taken = 0;
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i >= E) taken |= 1u << i;
  float sel[kMaxK];
  int sid[kMaxK];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (taken & (1u << i)) continue;
      const int e = lane + 32 * i;
      if (bi == INT_MAX || v[i] > bv) {  // slots ascend in e: strict '>' keeps the lower index
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel[j] = bv;
    sid[j] = bi;
  }
  if (lane == 0) {
    float den = 0.0f;
    float ex[kMaxK];
    for (int j = 0; j < k; ++j) {
      ex[j] = expf(sel[j] - sel[0]);
      den += ex[j];
    }
    for (int j = 0; j < k; ++j) {
      const float w = ex[j] / den;
      idx[(size_t)t * k + j] = sid[j];
      wts[(size_t)t * k + j] = w;
      if (dbg_idx) dbg_idx[(size_t)t * k + j] = sid[j];
      if (dbg_w) dbg_w[(size_t)t * k + j] = w;
    }
  }
}

cudaError_t launch_router_topk(const __nv_bfloat16* x, const float* Wr, const float* b, int T, int H,
                               int E, int k, const Workspace& ws, int32_t* dbg_idx, float* dbg_w,
                               cudaStream_t stream) {
  if (T <= 64 || E <= 32) {  // one warp per dot product: plenty of parallelism when E is small
    dim3 grid(T, (E + 7) / 8);
    router_warp_kernel<<<grid, 256, 0, stream>>>(x, Wr, b, T, H, E, ws.logits);
  } else {
    dim3 grid((T + 63) / 64, (E + 63) / 64);
    router_tile_kernel<64><<<grid, 256, 0, stream>>>(x, Wr, b, T, H, E, ws.logits);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  topk_softmax_kernel<<<(T + 7) / 8, 256, 0, stream>>>(ws.logits, T, E, k, ws.idx, ws.wts, dbg_idx, dbg_w);
  return cudaGetLastError();
}

}  // namespace moe

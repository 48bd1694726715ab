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
  pdl_enter();  // before any global memory access (see moe_common.cuh)
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

// One block of 128 threads per (token, expert) dot product: each thread sums its
// share of H (8-byte bf16 and 16-byte fp32 loads, several in flight), then the
// block adds the 128 partial sums.  Used for decode-sized batches.
__global__ void __launch_bounds__(128) router_dot_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ Wr, const float* __restrict__ b,
                                                         int T, int H, int E, float* __restrict__ logits) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  __shared__ float red[4];
  const int t = blockIdx.x, e = blockIdx.y;
  const __nv_bfloat16* xr = x + (size_t)t * H;
  const float* wr = Wr + (size_t)e * H;
  float acc = 0.0f;
#pragma unroll 4
  for (int h = threadIdx.x * 4; h < H; h += 512) {
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
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    const float v = (red[0] + red[1]) + (red[2] + red[3]);
    logits[(size_t)t * E + e] = b ? v + b[e] : v;
  }
}

// ---------------------------------------------------------------- router, many tokens
// The fp32 router weights are split exactly into three bf16 terms
// (w = hi + mid + lo up to the last bit of lo), so with bf16 x every product
// x * term is exact and bf16 tensor-core MMAs with fp32 accumulation compute
// the fp32 dot product.  The MMAs accumulate chunks of 64 inputs in
// registers; chunk sums are added with Kahan compensation, so the rounding
// error stays near that of a pairwise sum even for H = 12288.

// Wr fp32 [E][H] -> Wb bf16 [3][E][H] (hi, mid, lo).
__global__ void router_split_kernel(const float* __restrict__ Wr, long long n, __nv_bfloat16* __restrict__ Wb) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float w = Wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = __fsub_rn(w, __bfloat162float(hi));
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = __fsub_rn(r1, __bfloat162float(mid));
    Wb[i] = hi;
    Wb[n + i] = mid;
    Wb[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

constexpr int kRT = 128, kRE = 64, kRK = 32, kRStages = 3, kRChunk = 64;
constexpr int kRRow = kRK + 8;  // bf16 per smem row: 80 bytes, conflict-free ldmatrix
constexpr int kRStageA = kRT * kRRow, kRStageB = 3 * kRE * kRRow;  // bf16 elements
constexpr int kRSmem = kRStages * (kRStageA + kRStageB) * 2;

__device__ __forceinline__ void cp16z(void* dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(ok ? 16u : 0u)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Block tile 128 tokens x 64 experts, 8 warps of 32 x 32; k-stages of 32 inputs
// (cp.async, three in flight).  blockIdx.z selects a part of the inputs
// (split-K for grids smaller than the GPU); each part writes its own logit
// plane, which the top-k kernel adds in double precision.  The bias goes into
// plane 0.
__global__ void __launch_bounds__(256, 2) router_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ Wb,
                                                         const float* __restrict__ b, int T, int H, int E,
                                                         float* __restrict__ logits) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  extern __shared__ __align__(16) __nv_bfloat16 rsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  const int t0 = blockIdx.x * kRT, e0 = blockIdx.y * kRE;
  const int nk = H / kRK;
  const int kb = blockIdx.z * nk / gridDim.z, ke = (blockIdx.z + 1) * nk / gridDim.z;  // k-steps of this part
  logits += (size_t)blockIdx.z * T * E;
  if (blockIdx.z > 0) b = nullptr;
  const size_t plane = (size_t)E * H;

  auto load = [&](int ks, int st) {
    __nv_bfloat16* A = rsm + st * (kRStageA + kRStageB);
    __nv_bfloat16* B = A + kRStageA;
    const int k0 = ks * kRK;
#pragma unroll
    for (int u = 0; u < 2; ++u) {  // A: 128 rows x 4 chunks of 16 bytes
      const int c = tid + 256 * u, r = c >> 2, q = c & 3;
      const bool ok = t0 + r < T;
      cp16z(A + r * kRRow + q * 8, x + (size_t)(ok ? t0 + r : 0) * H + k0 + q * 8, ok);
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {  // B: 3 planes x 64 rows x 4 chunks
      const int c = tid + 256 * u, p = c >> 8, r = (c >> 2) & 63, q = c & 3;
      const bool ok = e0 + r < E;
      cp16z(B + (p * kRE + r) * kRRow + q * 8, Wb + p * plane + (size_t)(ok ? e0 + r : 0) * H + k0 + q * 8, ok);
    }
  };

  float tot[2][4][4], comp[2][4][4], acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int v = 0; v < 4; ++v) tot[i][j][v] = comp[i][j][v] = acc[i][j][v] = 0.0f;

#pragma unroll
  for (int st = 0; st < kRStages - 1; ++st) {
    if (kb + st < ke) load(kb + st, st);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int ks = kb; ks < ke; ++ks) {
    asm volatile("cp.async.wait_group %0;" ::"n"(kRStages - 2) : "memory");
    __syncthreads();
    {  // refill the stage consumed one step ago
      const int kn = ks + kRStages - 1;
      if (kn < ke) load(kn, (kn - kb) % kRStages);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const __nv_bfloat16* A = rsm + ((ks - kb) % kRStages) * (kRStageA + kRStageB);
    const __nv_bfloat16* B = A + kRStageA;
#pragma unroll
    for (int kk = 0; kk < kRK; kk += 16) {
      uint32_t af[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
        ldsm_x4(af[mt], A + (wm * 32 + mt * 16 + (lane & 15)) * kRRow + kk + (lane >> 4) * 8);
#pragma unroll
      for (int p = 0; p < 3; ++p) {
#pragma unroll
        for (int np = 0; np < 2; ++np) {  // n8 tiles 2np, 2np+1
          uint32_t bf[4];
          ldsm_x4(bf, B + (p * kRE + wn * 32 + np * 16 + (lane & 7) + ((lane >> 4) << 3)) * kRRow + kk +
                          ((lane >> 3) & 1) * 8);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_bf16(acc[mt][2 * np], af[mt], bf[0], bf[1]);
            mma_bf16(acc[mt][2 * np + 1], af[mt], bf[2], bf[3]);
          }
        }
      }
    }
    if ((ks - kb + 1) % (kRChunk / kRK) == 0 || ks + 1 == ke) {  // chunk done: Kahan-add into the totals
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float y = __fsub_rn(acc[i][j][v], comp[i][j][v]);
            const float t = __fadd_rn(tot[i][j][v], y);
            comp[i][j][v] = __fsub_rn(__fsub_rn(t, tot[i][j][v]), y);
            tot[i][j][v] = t;
            acc[i][j][v] = 0.0f;
          }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // accumulator element v of tile (mt, nt): token wm*32 + mt*16 + lane/4 + 8*(v >> 1),
  // expert wn*32 + nt*8 + 2*(lane%4) + (v & 1)
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int t = t0 + wm * 32 + mt * 16 + (lane >> 2) + 8 * (v >> 1);
        const int e = e0 + wn * 32 + nt * 8 + 2 * (lane & 3) + (v & 1);
        if (t < T && e < E) logits[(size_t)t * E + e] = b ? tot[mt][nt][v] + b[e] : tot[mt][nt][v];
      }
}

// ---------------------------------------------------------------- top-k + softmax
// One warp per token.  Expert e lives in lane e%32, slot e/32.  k passes of a
// warp-wide arg-max over the experts not chosen yet; ties go to the lower
// expert index; NaN ranks below every number.
__global__ void topk_softmax_kernel(const float* __restrict__ logits, int nparts, int T, int E, int k,
                                    int32_t* __restrict__ idx, float* __restrict__ wts,
                                    int32_t* __restrict__ dbg_idx, float* __restrict__ dbg_w) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    float l = -INFINITY;
    if (e < E) {
      if (nparts == 1) {
        l = logits[(size_t)t * E + e];
      } else {  // split-K planes of the router GEMM
        double sum = 0.0;
        for (int z = 0; z < nparts; ++z) sum += (double)logits[((size_t)z * T + t) * E + e];
        l = (float)sum;
      }
    }
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

// 0: warp-per-dot-product router; otherwise the GEMM with this many K parts
// (enough tiles for two per SM on 148 SMs, parts of at least 512 inputs).
int router_parts(long long T, int H, int E) {
  if (T <= 64 || E <= 32) return 0;
  const long long tiles = ((T + kRT - 1) / kRT) * ((E + kRE - 1) / kRE);
  long long p = (2 * 148 + tiles - 1) / tiles;
  const long long pmax = H / 512 > 1 ? H / 512 : 1;
  if (p > pmax) p = pmax;
  if (p > 8) p = 8;
  return p < 1 ? 1 : (int)p;
}

cudaError_t launch_router_topk(const __nv_bfloat16* x, const float* Wr, const float* b, int T, int H,
                               int E, int k, const Workspace& ws, int32_t* dbg_idx, float* dbg_w,
                               cudaStream_t stream) {
  const int parts = router_parts(T, H, E);
  if (parts == 0 && T <= 64 && E <= 32) {  // decode, few experts: one block per dot product
    launch_chained(router_dot_kernel, dim3(T, E), dim3(128), 0, stream, x, Wr, b, T, H, E, ws.logits);
  } else if (parts == 0) {  // many tokens, few experts: one warp per dot product
    dim3 grid(T, (E + 7) / 8);
    launch_chained(router_warp_kernel, dim3(grid), dim3(256), 0, stream, x, Wr, b, T, H, E, ws.logits);
  } else {
    const long long n = (long long)E * H;
    launch_chained(router_split_kernel, dim3((int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096)), dim3(256), 0, stream, Wr, n, ws.wsplit);
    cudaError_t aerr = cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem);
    if (aerr != cudaSuccess) return aerr;
    dim3 grid((T + kRT - 1) / kRT, (E + kRE - 1) / kRE, parts);
    launch_chained(router_mma_kernel, dim3(grid), dim3(256), kRSmem, stream, x, ws.wsplit, b, T, H, E, ws.logits);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  launch_chained(topk_softmax_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, ws.logits, parts > 1 ? parts : 1, T, E, k, ws.idx, ws.wts,
                                                        dbg_idx, dbg_w);
  return cudaGetLastError();
}

}  // namespace moe

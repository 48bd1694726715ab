// Weighted combine of the k expert outputs of each token (expert-routing
// section of the quantized MoE inference page: output = sum_i w_i * expert_i(x)).
// y[t][n] = bf16( sum_{j ascending} w[t][j] * o[inv[t*k+j]][n] ), summed in fp32.
#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

__global__ void combine_kernel(const float* __restrict__ o, const float* __restrict__ wts,
                               const int32_t* __restrict__ inv, int k, int H,
                               __nv_bfloat16* __restrict__ y) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int t = blockIdx.x;
  int rows[kMaxK];
  float w[kMaxK];
  for (int j = 0; j < k; ++j) {
    rows[j] = inv[t * k + j];
    w[j] = wts[t * k + j];
  }
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < H / 4; c += gridDim.y * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(o + (size_t)rows[j] * H) + c);
      acc.x = fmaf(w[j], v.x, acc.x);
      acc.y = fmaf(w[j], v.y, acc.y);
      acc.z = fmaf(w[j], v.z, acc.z);
      acc.w = fmaf(w[j], v.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&lo);
    out.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y + (size_t)t * H)[c] = out;
  }
}

cudaError_t launch_combine(int T, int k, int H, const Workspace& ws, __nv_bfloat16* y, cudaStream_t stream) {
  int ny = T < 512 ? (H / 4 + 255) / 256 : 1;  // column blocks: more parallelism for few tokens
  if (ny > 8) ny = 8;
  launch_chained(combine_kernel, dim3(T, ny), dim3(256), 0, stream, ws.o, ws.wts, ws.inv, k, H, y);
  return cudaGetLastError();
}

}  // namespace moe

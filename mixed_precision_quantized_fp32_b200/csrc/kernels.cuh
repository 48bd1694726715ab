// Launchers of the CUDA kernels, called by the host ABI (abi.cu).
#pragma once
#include "moe_common.cuh"

namespace moe {

// fmt_host: the caller's codes (MOE_FMT_OUTLIERS kept); out_sec / side_off: the outlier
// section and side-list offsets (0 when absent).
cudaError_t launch_pack(const float* W, int e0, int ne, int E, int H, int F, const uint8_t* fmt_host,
                        uint8_t* out, const uint64_t* code_off, const uint64_t* scale_off, uint64_t out_sec,
                        const uint64_t* side_off, cudaStream_t stream);

// Router K parts (0: warp kernel, no parts); the workspace holds max(1, parts) logit planes.
int router_parts(long long T, int H, int E);

cudaError_t launch_router_topk(const __nv_bfloat16* x, const float* Wr, const float* b, int T, int H,
                               int E, int k, const Workspace& ws, int32_t* dbg_idx, float* dbg_w,
                               cudaStream_t stream);

cudaError_t launch_permute(int T, int k, int E, int chunk_rows, const Workspace& ws, int32_t* dbg_counts,
                           int32_t* dbg_perm, int32_t* dbg_inv, cudaStream_t stream);

cudaError_t launch_gather(const __nv_bfloat16* x, int T, int H, int k, bool fp4, const Workspace& ws,
                          uint8_t* dbg_xq, float* dbg_sx, cudaStream_t stream);

cudaError_t launch_act_quant_h(int R, int F, const Workspace& ws, uint8_t* dbg_hq, float* dbg_sh,
                               cudaStream_t stream);

// Test hooks of the expert GEMMs (moe_debug.test_withhold / wait_cycles).
struct GemmHooks {
  uint32_t withhold;     // nonzero: the copy warps issue no loads
  uint32_t wait_cycles;  // pipeline wait budget, 0: default
};

// Token rows per work chunk of the tcgen05 expert GEMMs (the MMA's largest N):
// fp16-operand GEMM, and the block-scaled FP4 GEMM of NVFP4 activations.
constexpr int kTcChunkRows = 256;
constexpr int kFp4ChunkRows = 128;

cudaError_t launch_expert_gemm_tc(const uint8_t* packed, const uint8_t* fmt_host, int E, int H, int F, int T, int k,
                                  bool fp4, bool gateup, const Workspace& ws, int32_t* status, uint64_t* trace,
                                  GemmHooks hooks, bool outliers, cudaStream_t stream);

// K parts of the decode GEMV for R expert rows on an N x K projection (nmat
// matrices); the workspace holds P*R*N*nmat fp32 partials when P > 1.
int gemv_split(long long R, int E, int N, int K, int nmat);

cudaError_t launch_expert_gemv(const uint8_t* packed, uint64_t packed_bytes, const uint8_t* fmt_host, int E, int H,
                               int F, int R, int k, bool fp4, bool gateup, int max_chunks, int chunk_rows,
                               const Workspace& ws, int32_t* status, uint64_t* trace, GemmHooks hooks,
                               bool outliers, cudaStream_t stream);

// NVFP4 activations: per-token codes of x and their gather into sorted rows
// (prefill: codes + block scales; decode: fp16 block values), and per-row codes of h.
cudaError_t launch_gather_nvfp4(const __nv_bfloat16* x, int T, int H, int k, bool tc, const Workspace& ws,
                                uint8_t* dbg_xq, uint8_t* dbg_xsb, float* dbg_sx, cudaStream_t stream);
cudaError_t launch_act_quant_h_nvfp4(int R, int F, bool tc, const Workspace& ws, uint8_t* dbg_hq, uint8_t* dbg_hsb,
                                     float* dbg_sh, cudaStream_t stream);
// Block-scaled FP4 expert GEMM (prefill of NVFP4 layers with NVFP4 activations).
cudaError_t launch_expert_gemm_fp4(const uint8_t* packed, int E, int H, int F, int T, int k, bool gateup,
                                   const Workspace& ws, int32_t* status, uint64_t* trace, GemmHooks hooks,
                                   cudaStream_t stream);

cudaError_t launch_combine(int T, int k, int H, const Workspace& ws, __nv_bfloat16* y, cudaStream_t stream);

}  // namespace moe

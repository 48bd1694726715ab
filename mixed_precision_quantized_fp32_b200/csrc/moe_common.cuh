// Shared device/host definitions of the packed layer layout and small helpers
// for the CUDA library.  (The CPU oracle has its own, independent copy of the
// layout definition; nothing here is shared with it.)
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/moe.h"

#include <utility>

namespace moe {

// ---------------------------------------------------------------- launch chaining
// The forward's kernels are launched with programmatic dependent launch: a kernel
// may be scheduled while its predecessor on the stream is still draining, so its
// launch and block setup overlap the predecessor's tail.  Every forward kernel
// therefore starts with pdl_enter(): griddepcontrol.wait blocks until the
// predecessor grid has completed and its memory is visible (a no-op for a plain
// launch), and only then may the kernel read or write global memory.  Because each
// kernel waits for its predecessor before it can complete, a kernel also sees the
// results of every earlier kernel of the chain.  The trigger that follows lets the
// next kernel be scheduled as soon as every block of this one has started.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... Exp, typename... Act>
inline cudaError_t launch_chained(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                  Act&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

constexpr uint32_t kMagic = 0x51454F4Du;
constexpr uint32_t kHdrBytes = 16384u;
constexpr uint32_t kOffFmt = 32u;
constexpr uint32_t kOffCode = 800u;
constexpr uint32_t kOffScale = 6944u;
constexpr uint32_t kOffTscale = 13088u;
constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
// Outlier side lists (MoE mixed-precision page sec. 4.2, tip 2: each expert matrix keeps
// its top 0.05% of weights by |w| in fp16 beside the quantized rest).  A matrix opts in
// with MOE_FMT_OUTLIERS on its format code; the header then holds the base format, a flag
// and the offset of the outlier section appended after the expert sections:
//   [u64 side_off[768]] [u32 selection scratch, kOutScratchWords] [one side list per
//   opted-in matrix, 256-byte aligned: u32 row_ptr[N+1], u32 entry[n_out] with the column
//   in bits 0-15 and the fp16 residual in bits 16-31, sorted by (row, column)].
constexpr uint32_t kOffFlags = 20u;    // u32: bit 0 = the layer has an outlier section
constexpr uint32_t kOffOutSec = 24u;   // u64: offset of the outlier section
constexpr int kOutScratchWords = 64 + 65536;
constexpr uint64_t kOutTableBytes = 8u * 3u * kMaxE;

__host__ __device__ inline bool fmt_known(int f) {
  return f == MOE_FMT_INT1 || f == MOE_FMT_INT2 || f == MOE_FMT_INT3 || f == MOE_FMT_INT4 || f == MOE_FMT_NVFP4;
}
// Host format codes may carry MOE_FMT_OUTLIERS; the base format decides codes and scales.
__host__ __device__ inline int fmt_base(int f) { return f & ~MOE_FMT_OUTLIERS; }
__host__ __device__ inline bool fmt_outliers(int f) { return (f & MOE_FMT_OUTLIERS) != 0; }
// Outliers of an N x K matrix: floor(N*K*5/10000), integer arithmetic.
__host__ __device__ inline uint64_t outlier_count(uint64_t N, uint64_t K) { return N * K * 5u / 10000u; }
// u32 words per group of 32 inputs
__host__ __device__ inline int fmt_words(int f) { return f == MOE_FMT_NVFP4 ? 4 : f; }

__host__ __device__ inline uint64_t code_bytes(int f, uint64_t N, uint64_t K) {
  return N * K * (uint64_t)fmt_words(f) / 8u;
}
__host__ __device__ inline uint64_t scale_bytes(int f, uint64_t N, uint64_t K) {
  return f == MOE_FMT_NVFP4 ? N * (K / 16) : N * (K / 32) * 2u;
}
__host__ __device__ inline uint64_t up256(uint64_t x) { return (x + 255u) & ~(uint64_t)255u; }

// N x K of projection p (0 gate, 1 up: F x H; 2 down: H x F)
__host__ __device__ inline void proj_shape(int p, int H, int F, int& N, int& K) {
  if (p < 2) { N = F; K = H; } else { N = H; K = F; }
}

// Section offsets of a whole layer; returns false on an unknown format.
__host__ __device__ inline bool layer_layout(int E, int H, int F, const uint8_t* fmt,
                                             uint64_t* code_off, uint64_t* scale_off,
                                             uint64_t* total) {
  uint64_t pos = kHdrBytes;
  for (int e = 0; e < E; ++e)
    for (int p = 0; p < 3; ++p) {
      const int f = fmt[e * 3 + p];
      if (!fmt_known(f)) return false;
      int N, K;
      proj_shape(p, H, F, N, K);
      pos = up256(pos);
      if (code_off) code_off[e * 3 + p] = pos;
      pos += code_bytes(f, N, K);
      pos = up256(pos);
      if (scale_off) scale_off[e * 3 + p] = pos;
      pos += scale_bytes(f, N, K);
    }
  if (total) *total = up256(pos);
  return true;
}

// The outlier section after the expert sections (which end at `end`): its offset
// (0 when no matrix opts in), each opted-in matrix's side-list offset in side[]
// (0 for the others) and the new total size.  fmt: host codes (flags kept).
__host__ __device__ inline uint64_t outlier_layout(int E, int H, int F, const uint8_t* fmt, uint64_t end,
                                                   uint64_t* side, uint64_t* total) {
  bool any = false;
  for (int i = 0; i < 3 * E; ++i) any |= fmt_outliers(fmt[i]);
  for (int i = 0; i < 3 * E; ++i) side[i] = 0;
  if (!any) {
    *total = end;
    return 0;
  }
  const uint64_t sec = up256(end);
  uint64_t pos = up256(sec + kOutTableBytes + 4u * (uint64_t)kOutScratchWords);
  for (int e = 0; e < E; ++e)
    for (int p = 0; p < 3; ++p) {
      if (!fmt_outliers(fmt[e * 3 + p])) continue;
      int N, K;
      proj_shape(p, H, F, N, K);
      side[e * 3 + p] = pos;
      pos = up256(pos + 4u * ((uint64_t)N + 1u + outlier_count(N, K)));
    }
  *total = pos;
  return sec;
}

// Word index (u32 units) of word w of the group holding input k of output n.
__host__ __device__ inline uint64_t word_index(int n, int k, int K, int wpg, int w) {
  const uint64_t nb = (uint64_t)(n >> 7), kb = (uint64_t)(k >> 7);
  const uint64_t kg = (uint64_t)((k & 127) >> 5);
  return (((nb * (uint64_t)(K >> 7) + kb) * 4u + kg) * (uint64_t)wpg + (uint64_t)w) * 128u +
         (uint64_t)(n & 127);
}
// Scale index of (output n, group g) with `groups` groups per row.
__host__ __device__ inline uint64_t scale_index(int n, int g, int groups) {
  return ((uint64_t)(n >> 7) * (uint64_t)groups + (uint64_t)g) * 128u + (uint64_t)(n & 127);
}

// Device-side view of a packed layer header.
struct LayerHdr {
  int E, H, F;
  const uint8_t* fmt;
  const uint64_t* code_off;
  const uint64_t* scale_off;
  const float* tscale;
  const uint8_t* base;
  const uint64_t* side;  // side-list offsets [768] (null: no outlier section)
};

__host__ __device__ inline LayerHdr hdr_view(const void* packed, int E, int H, int F) {
  LayerHdr h;
  h.base = (const uint8_t*)packed;
  h.E = E;
  h.H = H;
  h.F = F;
  h.fmt = h.base + kOffFmt;
  h.code_off = (const uint64_t*)(h.base + kOffCode);
  h.scale_off = (const uint64_t*)(h.base + kOffScale);
  h.tscale = (const float*)(h.base + kOffTscale);
  h.side = nullptr;
  return h;
}
// The same with the outlier table (reads the header's flag word on the device).
__device__ inline LayerHdr hdr_view_side(const void* packed, int E, int H, int F) {
  LayerHdr h = hdr_view(packed, E, H, F);
  if (*(const uint32_t*)(h.base + kOffFlags) & 1u)
    h.side = (const uint64_t*)(h.base + *(const uint64_t*)(h.base + kOffOutSec));
  return h;
}

// Residual term of weight row n of matrix slot i (e*3+p) against activation row a
// (fp16, length K): sum over the row's outliers of r * a[col].  0 without a side list.
__device__ __forceinline__ float outlier_dot(const LayerHdr& L, int i, int N, int n, const __half* __restrict__ a) {
  if (!L.side) return 0.0f;
  const uint64_t off = L.side[i];
  if (!off) return 0.0f;
  const uint32_t* rp = (const uint32_t*)(L.base + off);
  const uint32_t* ent = rp + N + 1;
  float s = 0.0f;
  for (uint32_t j = __ldg(rp + n), j1 = __ldg(rp + n + 1); j < j1; ++j) {
    const uint32_t v = __ldg(ent + j);
    s = fmaf(__half2float(__ushort_as_half((uint16_t)(v >> 16))), __half2float(a[v & 0xFFFFu]), s);
  }
  return s;
}

// e2m1 code (sign<<3 | exp<<1 | man) -> float
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6
  const float mag = (m < 2u) ? 0.5f * (float)m : (float)((2u | (m & 1u)) << ((m >> 1) - 1u)) * 0.5f;
  return (c & 8u) ? -mag : mag;
}

// e4m3 ("fn") code -> float (NaN codes not produced by this library)
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v = (e == 0u) ? (float)m * 0.001953125f /* 2^-9 */
                      : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80u) ? -v : v;
}

// Workspace layout shared by the host ABI and the kernels.
struct Workspace {
  float* logits;       // [parts][T*E] (parts: router K parts, at least 1)
  __nv_bfloat16* wsplit;  // [3][E*H] bf16 terms of the router weights (router GEMM only)
  int32_t* idx;        // [T*k]
  float* wts;          // [T*k]
  int32_t* counts;     // [E]
  int32_t* offsets;    // [E+1]
  int32_t* blk_hist;   // [nblk*E]
  int32_t* rank;       // [T*k] stable rank of each entry inside its count block
  int32_t* perm;       // [T*k]
  int32_t* inv;        // [T*k]
  int32_t* chunks;     // [max_chunks*3] (expert, row0, rows) + [1] count at chunk_count
  int32_t* chunk_count;// [1]
  uint8_t* xq;         // [T*H] NVFP4 activation codes
  float* sx;           // [T]
  void* xs;            // [T*k*H] fp16 gathered activations (NVFP4: exact e4m3 values)
  void* h;             // [T*k*F] fp16 (int) / fp32 (NVFP4 pre-quant)
  void* hb;            // [T*k*F] fp16 NVFP4 decoded h codes (exact)
  uint8_t* hq;         // [T*k*F] NVFP4 h codes
  float* sh;           // [T*k]
  float* o;            // [T*k*H] fp32 expert outputs, sorted rows
  int32_t* status;     // [1]
  float* part;         // decode GEMV split-K partial sums (null when not split)
  int32_t* counters;   // [counter_len] decode GEMV work counters (gate/up, down)
  int counter_len;
  float* xsum;         // [T*k][H/32] group sums of the gathered fp16 activations (integer layers)
  float* hsum;         // [T*k][F/32] group sums of the fp16 SwiGLU outputs (integer layers)
  float* xinv;         // [T*k] integer layers: 2^e undoing the power-of-two prescale of a row's x
  // NVFP4 activations (moe_weights.act = MOE_ACT_NVFP4); xq then holds packed e2m1 codes [T][H/2]
  int ldx, ldh;        // row pitch of the block-scale arrays of x and h (bytes, a multiple of 16)
  uint8_t* xsf;        // [T][ldx] e4m3 block scales of x per token
  uint8_t* xs4;        // [T*k][H/2] gathered codes of x (prefill)
  uint8_t* xsf4;       // [T*k][ldx] gathered block scales of x (prefill)
  uint8_t* hs4;        // [T*k][F/2] codes of h (prefill)
  uint8_t* hsf4;       // [T*k][ldh] block scales of h (prefill)
};

}  // namespace moe

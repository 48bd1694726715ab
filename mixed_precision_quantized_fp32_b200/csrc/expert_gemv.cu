// Dequant-fused grouped expert GEMV for batches with few token rows per expert
// (decode: chunks of up to 8 rows), bound by streaming the active experts'
// packed weights from HBM.  It follows the pages' observation that a token only
// needs its active experts' weights, and implements the packed-linear operator
// of the MoE mixed-precision page (sec. 2.3 / 3.5).
//
// Work item: (chunk of <= 8*NT8 expert-sorted token rows of one expert, block
// of 128 weight rows, part p of P along K).  Persistent CTAs take items from a
// global counter, so uneven items balance across SMs.  Warp 4 streams each
// 128-input tile of the block through a ring of shared-memory stages:
//   * the packed codes: two 3D TMA loads per matrix, with a 128-byte swizzle so
//     the 16-byte code reads below are bank-conflict free;
//   * the group scales: one bulk copy;
//   * the token rows and their per-group sums: 2D TMA loads.
// None is multicast.  Warps 0-3 own 32 weight rows each.
//
// Per group of 32 inputs, lane (g, c) holds word(s) of rows 4g..4g+3 covering
// inputs 8c..8c+7.  It turns each pair of codes into one fp16x2 A-fragment
// register with one AND (INT3: one more op per pair merges the high-bit plane;
// the 1-bit sign code's fields sit at bit j, the MMA sums (u - 1/2)*x and the
// group scale is doubled):
//   * the masked field is read as an fp16 subnormal: a code u in a field of
//     power-of-two weight f (bit position 2j or 4j of a half-word) is exactly
//     u * f * 2^-24;
//   * the matching activation is prescaled by 1/f (exact), so each product is
//     x * u * 2^-24;
//   * the code offset 2^(b-1) is removed through the MMA's C input:
//     -offset * 2^-24 * (sum of the group's activations), precomputed per token
//     row and group when the activations are written.
// Each group's fp32 MMA result is scaled by its fp16 group scale, and 2^24 is
// restored at the end.  NVFP4 codes become exact fp16 with cvt.e2m1x2 times
// their e4m3 block scale and accumulate directly.
//
// Split-K (P > 1, for batches with too few blocks to fill the GPU) writes
// per-part fp32 partials; a small follow-up kernel sums the parts in a fixed
// order and runs the epilogue.  There are no atomics or fences between CTAs and
// results do not depend on timing.  Every mbarrier wait is bounded; a wait that
// gives up sets MOE_ERR_TIMEOUT in the status word.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "moe_common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kBlockRows = 128;                 // weight rows per work item (one packed tile row)
constexpr int kConsumers = 4;                   // consumer warps, 32 weight rows each
constexpr int kProducer = kConsumers;           // warp index of the TMA warp
constexpr int kGemvThreads = 32 * (kConsumers + 1);
constexpr long long kGemvWait = 2000000000LL;   // clock cycles, ~1 s
constexpr int kMaxSplit = 16;
constexpr int kMaxStages = 32;
constexpr int kCtrlBytes = 3072;                // barriers, item descriptors and flags after the ring

// Shared-memory stage (sizes fixed per launch from the layer's widest formats):
//   [matrix m: code box 0 | code box 1] [scales m] ... [token rows x 128 fp16]
//   [token rows x 4 group sums fp32]
// A code box holds 4 groups x wpg words x 2 row slices x 128 bytes (1024 * wpg).
struct StageLayout {
  int box[2];        // bytes of one code box of matrix 0 / 1
  int code_off[2];   // offset of matrix m's first box
  int scale_off[2];  // offset of matrix m's scales (1024 bytes)
  int x_off;         // offset of the token rows
  int sum_off;       // offset of the group sums (integer layers)
  int bytes;         // stage size (multiple of 1024)
  int stages;        // ring depth
};

struct GemvArgs {
  const uint8_t* packed;
  int E, H, F;
  int N, K;               // weight rows and inputs of this projection
  int proj;               // 0: gate+up with the SwiGLU epilogue; 2: down
  int topk;
  int P;                  // K parts
  int R;                  // expert rows in the batch (T*k)
  const int32_t* chunks;  // (expert, first row, rows)
  const int32_t* chunk_count;
  const float* row_scale; // NVFP4: gate/up -> per-token sx, down -> per-row sh; null for integer layers
  const float* xinv;      // integer gate/up: per-row 2^e undoing the activations' prescale (null otherwise)
  const __half* act16;    // the fp16 activations [R][K] (the residual term of outlier side lists)
  int outliers;           // the layer has outlier side lists
  const int32_t* perm;
  bool sums;              // integer layer: activation group sums are loaded with the tiles
  void* out;              // gate/up: h [R][F] (fp16, or fp32 for NVFP4); down: o fp32 [R][H]
  float* out_sum;         // gate/up, integer layers: group sums of h [R][F/32]
  float* part;            // [P][R][NMAT][N] partial sums (P > 1)
  int32_t* work;          // next work item (zero before the launch)
  int32_t* status;
  unsigned long long* trace;  // diagnostics: clock64 stamps of CTA 0 (or null)
  StageLayout st;
  long long wait;         // budget of the pipeline waits, clock cycles
  int withhold;           // test hook: the TMA warp issues no loads (the waits run out)
};

// Stamp event `ev` of index `i` (CTA 0 only, first MOE_TRACE_STAGES indices).
__device__ __forceinline__ void gtrace(unsigned long long* tr, int ev, int i) {
  if (tr && blockIdx.x == 0 && i < MOE_TRACE_STAGES) tr[ev * MOE_TRACE_STAGES + i] = (unsigned long long)clock64();
}

__device__ __forceinline__ const CUtensorMap* map_of(int wpg, const CUtensorMap* m1, const CUtensorMap* m2,
                                                     const CUtensorMap* m3, const CUtensorMap* m4) {
  return wpg == 1 ? m1 : wpg == 2 ? m2 : wpg == 3 ? m3 : m4;
}

// ------------------------------------------------------------------ small PTX helpers
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          ptx::smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(ptx::smem_u32(bar))
      : "memory");
}
// shared-space loads through 32-bit shared addresses
__device__ __forceinline__ uint4 lds128(uint32_t a) { return ptx::lds_v4(a); }
__device__ __forceinline__ uint2 lds64(uint32_t a) { return ptx::lds_v2(a); }
__device__ __forceinline__ uint32_t lds32(uint32_t a) { return ptx::lds_u32(a); }
__device__ __forceinline__ float ldsf(uint32_t a) { return ptx::lds_f32(a); }
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory"); }

// Bounded wait that ignores the abort flag (used to drain copies before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity) && clock64() - t0 < kGemvWait / 4) {
  }
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t* o) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1, const float* c) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}
__device__ __forceinline__ float half_lo(uint32_t v) { return __half2float(__ushort_as_half((uint16_t)(v & 0xFFFFu))); }
__device__ __forceinline__ float half_hi(uint32_t v) { return __half2float(__ushort_as_half((uint16_t)(v >> 16))); }

constexpr uint32_t h2c(uint32_t h) { return h | (h << 16); }

// Activation multiplier 1/f_j (fp16x2) for pair j (j = 0..3) of a lane's eight
// inputs, whose codes sit in a field of weight f_j: INT4 1, 16, 1, 16 (fields at
// bits 0 and 4; pairs 2, 3 after >> 8); INT2 and INT3 4^j (fields at bits 2j);
// INT1 2^j (fields at bit j).  Every multiplier is at most 1, so the products
// stay in range for any fp16 activation.
__host__ __device__ constexpr uint32_t act_mul(int fmt, int j) {
  return fmt == MOE_FMT_NVFP4 ? h2c(0x3C00u)
         : fmt == MOE_FMT_INT1 ? (j == 0 ? h2c(0x3C00u) : j == 1 ? h2c(0x3800u) : j == 2 ? h2c(0x3400u) : h2c(0x3000u))
         : fmt == MOE_FMT_INT4 ? ((j & 1) ? h2c(0x2C00u) : h2c(0x3C00u))   // 1, 1/16
         : (j == 0 ? h2c(0x3C00u) : j == 1 ? h2c(0x3400u) : j == 2 ? h2c(0x2C00u) : h2c(0x2400u));  // 4^-j
}
// -offset * 2^-24: times the group sum of the activations, the MMA's C input.
// INT1: the sign code q = 2u - 1 = 2(u - 1/2), so the MMA sums (u - 1/2) x and
// the group scale is doubled (group_scale_mul).
__host__ __device__ constexpr float offset_term(int fmt) {
  return fmt == MOE_FMT_INT4 ? -8.0f / 16777216.0f
         : fmt == MOE_FMT_INT3 ? -4.0f / 16777216.0f
         : fmt == MOE_FMT_INT1 ? -0.5f / 16777216.0f
                               : -2.0f / 16777216.0f;
}
__host__ __device__ constexpr float group_scale_mul(int fmt) { return fmt == MOE_FMT_INT1 ? 2.0f : 1.0f; }

// Address of the 16-byte chunk of rows 4g..4g+3 in word-row z of a code box
// (lines of 128 bytes: line = 2z + slice; 128-byte swizzle: chunk ^= line % 8).
__device__ __forceinline__ uint32_t code_chunk(uint32_t box, int z, int y, int g) {
  const int line = 2 * z + y;
  return box + (uint32_t)(line * 128 + ((g ^ (line & 7)) << 4));
}

// One group (kg) of one matrix: unpack the lane's rows, run the MMAs for every
// token tile and accumulate.  All addresses are shared-window addresses.  box:
// this warp's code box; sc: the matrix's scale tile; xs: the lane's 16
// activation bytes of the group in token tile 0 (token tiles follow at 8 rows x
// 256 bytes); gs: the group sum of token 2c in token tile 0 (token 2c+1 follows
// at +16 bytes, tile nt at nt * 128 bytes).
template <int FMT, int NT8>
__device__ __forceinline__ void group_mma(uint32_t box, uint32_t sc, int kg, int y, int s, int g, int c,
                                          uint32_t xs, uint32_t gs, float (&acc)[2][NT8][4]) {
  uint32_t p[4][4];   // [row i][pair j]
  if (FMT == MOE_FMT_NVFP4) {
    const uint4 w = lds128(code_chunk(box, 4 * kg + c, y, g));
    const uint32_t bs = lds32(sc + (2 * kg + (c >> 1)) * 128 + 32 * s + 4 * g);  // e4m3 block scales of rows 4g..
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    // e4m3 pairs -> f16 pairs (hardware conversion, exact), then each row's scale in both halves
    const __half2_raw s01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(bs & 0xFFFFu), __NV_E4M3);
    const __half2_raw s23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(bs >> 16), __NV_E4M3);
    const uint32_t w01 = (uint32_t)s01.x | ((uint32_t)s01.y << 16), w23 = (uint32_t)s23.x | ((uint32_t)s23.y << 16);
    const uint32_t sp[4] = {__byte_perm(w01, 0u, 0x1010u), __byte_perm(w01, 0u, 0x3232u), __byte_perm(w23, 0u, 0x1010u),
                            __byte_perm(w23, 0u, 0x3232u)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      e2m1x8_to_f16(wv[i], p[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) p[i][j] = hmul2(p[i][j], sp[i]);  // exact: <= 6 significant bits
    }
#pragma unroll
    for (int nt = 0; nt < NT8; ++nt) {
      const uint4 xr = lds128(xs + nt * 2048);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t A1[4] = {p[2 * t][0], p[2 * t + 1][0], p[2 * t][1], p[2 * t + 1][1]};
        const uint32_t A2[4] = {p[2 * t][2], p[2 * t + 1][2], p[2 * t][3], p[2 * t + 1][3]};
        mma16816(acc[t][nt], A1, xr.x, xr.y, acc[t][nt]);
        mma16816(acc[t][nt], A2, xr.z, xr.w, acc[t][nt]);
      }
    }
    return;
  }
  if (FMT == MOE_FMT_INT1) {
    // one word per row and group: the lane's pairs j at bits 4c + j (and 16 above)
    const uint4 w = lds128(code_chunk(box, kg, y, g));
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t ws = wv[i] >> (4 * c);
#pragma unroll
      for (int j = 0; j < 4; ++j) p[i][j] = ws & (0x00010001u << j);
    }
  } else if (FMT == MOE_FMT_INT4) {
    const uint4 w = lds128(code_chunk(box, 4 * kg + c, y, g));
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w8 = wv[i] >> 8;
      p[i][0] = wv[i] & 0x000F000Fu;
      p[i][1] = wv[i] & 0x00F000F0u;
      p[i][2] = w8 & 0x000F000Fu;
      p[i][3] = w8 & 0x00F000F0u;
    }
  } else {
    const int wpg = FMT == MOE_FMT_INT3 ? 3 : 2;
    const uint4 w = lds128(code_chunk(box, wpg * kg + (c >> 1), y, g));
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    const int sh = 8 * (c & 1);
    if (FMT == MOE_FMT_INT2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t ws = wv[i] >> sh;
#pragma unroll
        for (int j = 0; j < 4; ++j) p[i][j] = ws & (0x00030003u << (2 * j));
      }
    } else {
      // INT3: bit 2 of pair m = 4c+j sits at bit 8*(c/2) + c%2 + 2j of word 2 (and
      // 16 above for the odd code), so one rotation per row puts all four of the
      // lane's high bits on bit 2j+2, right above each pair's two low bits.
      const uint4 hw = lds128(code_chunk(box, 3 * kg + 2, y, g));
      const uint32_t hv[4] = {hw.x, hw.y, hw.z, hw.w};
      const uint32_t rot = (uint32_t)(8 * (c >> 1) + (c & 1) + 30) & 31u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t ws = wv[i] >> sh;
        const uint32_t hh = __funnelshift_r(hv[i], hv[i], rot);
#pragma unroll
        for (int j = 0; j < 4; ++j) p[i][j] = (ws & (0x00030003u << (2 * j))) | (hh & (0x00040004u << (2 * j)));
      }
    }
  }
  const uint2 s4 = lds64(sc + kg * 256 + (32 * s + 4 * g) * 2);  // fp16 scales of rows 4g..4g+3
  constexpr float kSm = group_scale_mul(FMT);
  const float sr[4] = {kSm * half_lo(s4.x), kSm * half_hi(s4.x), kSm * half_lo(s4.y), kSm * half_hi(s4.y)};
#pragma unroll
  for (int nt = 0; nt < NT8; ++nt) {
    const uint4 xr = lds128(xs + nt * 2048);
    const uint32_t b0 = xr.x, b1 = hmul2(xr.y, act_mul(FMT, 1));  // act_mul(FMT, 0) == 1
    const uint32_t b2 = FMT == MOE_FMT_INT4 ? xr.z : hmul2(xr.z, act_mul(FMT, 2));
    const uint32_t b3 = hmul2(xr.w, act_mul(FMT, 3));
    const float d0 = offset_term(FMT) * ldsf(gs + nt * 128), d1 = offset_term(FMT) * ldsf(gs + nt * 128 + 16);
    const float D[4] = {d0, d1, d0, d1};  // -offset * sum(x) * 2^-24 for tokens 2c, 2c+1
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t A1[4] = {p[2 * t][0], p[2 * t + 1][0], p[2 * t][1], p[2 * t + 1][1]};
      const uint32_t A2[4] = {p[2 * t][2], p[2 * t + 1][2], p[2 * t][3], p[2 * t + 1][3]};
      float d[4];
      mma16816(d, A1, b0, b1, D);
      mma16816(d, A2, b2, b3, d);
      acc[t][nt][0] = fmaf(sr[2 * t], d[0], acc[t][nt][0]);
      acc[t][nt][1] = fmaf(sr[2 * t], d[1], acc[t][nt][1]);
      acc[t][nt][2] = fmaf(sr[2 * t + 1], d[2], acc[t][nt][2]);
      acc[t][nt][3] = fmaf(sr[2 * t + 1], d[3], acc[t][nt][3]);
    }
  }
}

// Consume the k-tiles of one work item (formats F0, F1 of the first and second
// matrix) from the ring; the first tile's stage has already been waited for.
// Waits that give up clear `ok`; the loop still runs to the end (without waiting
// or computing) so all consumer warps stay in step.
template <int NMAT, int NT8, int F0, int F1>
__device__ __forceinline__ void consume_tiles(const StageLayout& L, uint8_t* smem, uint64_t* full, uint64_t* empty,
                                              volatile int* abort_flag, int ntiles, int& stage, uint32_t& phase,
                                              bool& ok, float (&acc)[NMAT][2][NT8][4], unsigned long long* tr,
                                              int& gtile, long long wait) {
  const int s = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  for (int kt = 0; kt < ntiles; ++kt) {
    if (kt > 0 && ok && !__all_sync(0xffffffffu, ptx::mbar_wait(&full[stage], phase, abort_flag, wait)))
      ok = false;
    if (threadIdx.x == 0) gtrace(tr, 2, gtile);
    if (ok) {
      const uint32_t sb = ptx::smem_u32(smem) + (uint32_t)(stage * L.bytes);
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) {
        const uint32_t xs = sb + (uint32_t)(L.x_off + g * 256 + (32 * kg + 8 * c) * 2);
        const uint32_t gs = sb + (uint32_t)(L.sum_off + (2 * c) * 16 + kg * 4);
        group_mma<F0, NT8>(sb + L.code_off[0] + (s >> 1) * L.box[0], sb + L.scale_off[0], kg, s & 1, s, g, c, xs,
                           gs, acc[0]);
        if (NMAT == 2)
          group_mma<F1, NT8>(sb + L.code_off[1] + (s >> 1) * L.box[1], sb + L.scale_off[1], kg, s & 1, s, g, c, xs,
                             gs, acc[NMAT - 1]);
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[stage]);
    if (threadIdx.x == 0) gtrace(tr, 3, gtile);
    ++gtile;
    if (++stage == L.stages) {
      stage = 0;
      phase ^= 1u;
    }
  }
}

// I1: the launch meets 1-bit matrices.  Their cases are compiled only into the
// I1 instantiations, so kernels for layers without them keep their size and
// register allocation.
template <int NMAT, int NT8, int F0, bool I1>
__device__ __forceinline__ void consume_f1(int f1, const StageLayout& L, uint8_t* smem, uint64_t* full,
                                           uint64_t* empty, volatile int* abort_flag, int ntiles, int& stage,
                                           uint32_t& phase, bool& ok, float (&acc)[NMAT][2][NT8][4],
                                           unsigned long long* tr, int& gtile, long long wait) {
  if (NMAT == 1 || F0 == MOE_FMT_NVFP4)
    return consume_tiles<NMAT, NT8, F0, F0>(L, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, tr, gtile, wait);
  if constexpr (I1) {
    if (f1 == MOE_FMT_INT1)
      return consume_tiles<NMAT, NT8, F0, MOE_FMT_INT1>(L, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, tr, gtile, wait);
  }
  switch (f1) {
    case MOE_FMT_INT2: return consume_tiles<NMAT, NT8, F0, MOE_FMT_INT2>(L, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, tr, gtile, wait);
    case MOE_FMT_INT3: return consume_tiles<NMAT, NT8, F0, MOE_FMT_INT3>(L, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, tr, gtile, wait);
    default: return consume_tiles<NMAT, NT8, F0, MOE_FMT_INT4>(L, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, tr, gtile, wait);
  }
}

// Work item `it` -> (chunk, weight block, K part): block-major, so the chunks of
// one expert (adjacent in the chunk list) read the same weight tiles close in
// time and the second read hits L2.
struct Item {
  int chunk, nb, p;
};
__device__ __forceinline__ Item item_of(int it, int P, int nchunks) {
  Item r;
  r.p = it % P;
  const int rest = it / P;
  r.chunk = rest % nchunks;
  r.nb = rest / nchunks;
  return r;
}

// What the consumers need about an item, written by the producer into the
// shared-memory slot of the item's first stage (it < 0 ends the stream).
struct ItemDesc {
  int it, chunk, nb, p, row0, rows, ntiles, f0, f1;
  float ts0, ts1;
  int e;  // expert
};
static_assert(sizeof(ItemDesc) == 48, "descriptor size");

// Producer-side view of an item: descriptor plus the copy sources.
template <int NMAT>
struct ItemSrc {
  ItemDesc d;
  int kt0;
  int z0[NMAT], wpg[NMAT];
  const uint8_t* sptr[NMAT];
  uint32_t bytes;
};

template <int NMAT, int NT8>
__device__ __forceinline__ void load_item(ItemSrc<NMAT>& s, int it, int total, int nchunks, const GemvArgs& a,
                                          const LayerHdr& L, int KT) {
  s.d.it = it < total ? it : -1;
  s.bytes = (uint32_t)(8 * NT8 * 256) + (a.sums ? (uint32_t)(8 * NT8 * 16) : 0u);
  if (it >= total) return;
  const Item w = item_of(it, a.P, nchunks);
  const int e = a.chunks[3 * w.chunk];
  s.d.chunk = w.chunk;
  s.d.e = e;
  s.d.nb = w.nb;
  s.d.p = w.p;
  s.d.row0 = a.chunks[3 * w.chunk + 1];
  s.d.rows = a.chunks[3 * w.chunk + 2];
  s.kt0 = w.p * KT / a.P;
  s.d.ntiles = (w.p + 1) * KT / a.P - s.kt0;
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    const int i = e * 3 + a.proj + m;
    const int f = L.fmt[i];
    if (m == 0) {
      s.d.f0 = f;
      s.d.ts0 = f == MOE_FMT_NVFP4 ? L.tscale[i] : 1.0f;
    }
    if (m == NMAT - 1) {
      s.d.f1 = f;
      s.d.ts1 = f == MOE_FMT_NVFP4 ? L.tscale[i] : 1.0f;
    }
    s.wpg[m] = fmt_words(f);
    s.z0[m] = (int)(L.code_off[i] >> 9) + (w.nb * KT) * 4 * s.wpg[m];
    s.sptr[m] = L.base + L.scale_off[i] + (size_t)w.nb * KT * 1024u;
    s.bytes += 2u * 1024u * (uint32_t)s.wpg[m] + 1024u;
  }
}

// Epilogue of one output (row r, weight row n) from the matrices' sums v[m]
// (integer formats: already multiplied by 2^24).  Gate/up returns h as stored
// (fp16-rounded for integer layers), for the group sums of the down GEMV, and
// sets `range` when that fp16 h overflowed.
// Outlier side lists add sum r * a over the row's outliers to the raw sums (in the
// units of the fp16 activations, before the row and tensor scales).
template <int NMAT>
__device__ __forceinline__ float store_output(const GemvArgs& a, int r, int n, const float* v, const float* ts,
                                              bool& range, int e) {
  float dot[NMAT];
#pragma unroll
  for (int m = 0; m < NMAT; ++m) dot[m] = 0.0f;
  if (a.outliers) {
    const LayerHdr L = hdr_view_side(a.packed, a.E, a.H, a.F);
#pragma unroll
    for (int m = 0; m < NMAT; ++m) dot[m] = outlier_dot(L, e * 3 + a.proj + m, a.N, n, a.act16 + (size_t)r * a.K);
  }
  if (NMAT == 2) {
    float gv = v[0], uv = v[1];
    if (a.row_scale) {
      const float sx = a.row_scale[a.perm[r] / a.topk];
      if (a.outliers) {
        gv = (gv * ts[0] + dot[0]) * sx;
        uv = (uv * ts[1] + dot[NMAT - 1]) * sx;
      } else {
        gv *= sx * ts[0];
        uv *= sx * ts[1];
      }
      const float h = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
      reinterpret_cast<float*>(a.out)[(size_t)r * a.N + n] = h;
      return h;
    }
    gv += dot[0];
    uv += dot[NMAT - 1];
    if (a.xinv) {
      const float xi = a.xinv[r];
      gv *= xi;
      uv *= xi;
    }
    const __half h = __float2half_rn(__fdividef(gv, 1.0f + __expf(-gv)) * uv);
    range |= __hisinf(h) != 0;
    reinterpret_cast<__half*>(a.out)[(size_t)r * a.N + n] = h;
    return __half2float(h);
  }
  float o = v[0];
  if (a.row_scale) o = a.outliers ? (o * ts[0] + dot[0]) * a.row_scale[r] : o * (a.row_scale[r] * ts[0]);
  else o += dot[0];
  reinterpret_cast<float*>(a.out)[(size_t)r * a.N + n] = o;
  return o;
}

// Record an SwiGLU output beyond fp16 range (the first error is kept).
__device__ __forceinline__ void report_range(int32_t* status) {
  if (status) atomicCAS(status, 0, (int32_t)MOE_ERR_RANGE);
}

template <int NMAT, int NT8, bool I1>
__global__ void __launch_bounds__(kGemvThreads, NT8 == 1 ? (NMAT == 1 ? 4 : 3) : 2) expert_gemv_kernel(const __grid_constant__ CUtensorMap tm_w1,
                                                                   const __grid_constant__ CUtensorMap tm_w2,
                                                                   const __grid_constant__ CUtensorMap tm_w3,
                                                                   const __grid_constant__ CUtensorMap tm_w4,
                                                                   const __grid_constant__ CUtensorMap tm_x,
                                                                   const __grid_constant__ CUtensorMap tm_s,
                                                                   const GemvArgs a) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer arithmetic
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  const StageLayout& SL = a.st;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SL.stages * SL.bytes);
  uint64_t* empty = full + kMaxStages;
  ItemDesc* slot = reinterpret_cast<ItemDesc*>(empty + kMaxStages);  // item starting at a stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + kMaxStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < SL.stages; ++st) {
      ptx::mbar_init(&full[st], 1);
      ptx::mbar_init(&empty[st], kConsumers);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducer && lane == 0) {
    ptx::prefetch_tmap(&tm_w1);
    ptx::prefetch_tmap(&tm_w2);
    ptx::prefetch_tmap(&tm_w3);
    ptx::prefetch_tmap(&tm_w4);
    ptx::prefetch_tmap(&tm_x);
    if (a.sums) ptx::prefetch_tmap(&tm_s);
  }
  __syncthreads();

  const int NB = a.N / kBlockRows, KT = a.K / 128;
  const int nchunks = *a.chunk_count;
  const int total = nchunks * NB * a.P;
  const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
  bool ok = true;

  if (warp == kProducer) {
    // Items are taken from a global counter (dynamic balance), one item ahead:
    // the next item's index and sources load while this item's tiles are issued.
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_par = 0;
    int nxt = 0, gtile = 0, gitem = 0;
    if (lane == 0) nxt = atomicAdd(a.work, 1);
    nxt = __shfl_sync(0xffffffffu, nxt, 0);
    ItemSrc<NMAT> cur, ahead;
    load_item<NMAT, NT8>(ahead, nxt, total, nchunks, a, L, KT);
    while (ok) {
      cur = ahead;
      const bool done = cur.d.it < 0;
      if (!done) {
        if (lane == 0) nxt = atomicAdd(a.work, 1);
        nxt = __shfl_sync(0xffffffffu, nxt, 0);
      }
      const int ntiles = done ? 1 : cur.d.ntiles;
      for (int kt = 0; kt < ntiles; ++kt) {
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.wait))) {
          ok = false;
          break;
        }
        if (lane == 0) gtrace(a.trace, 0, gtile);
        if (lane == 0) {
          uint8_t* sb = smem + stage * SL.bytes;
          if (kt == 0) slot[stage] = cur.d;
          if (done) {
            ptx::mbar_arrive(&full[stage]);
          } else if (!a.withhold) {
            ptx::mbar_arrive_expect_tx(&full[stage], cur.bytes);
            const int k = cur.kt0 + kt;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              const int z = cur.z0[m] + k * 4 * cur.wpg[m];
              const CUtensorMap* map = map_of(cur.wpg[m], &tm_w1, &tm_w2, &tm_w3, &tm_w4);
              tma_load_3d(sb + SL.code_off[m], map, 0, 0, z, &full[stage]);
              tma_load_3d(sb + SL.code_off[m] + SL.box[m], map, 0, 2, z, &full[stage]);
              ptx::bulk_load(sb + SL.scale_off[m], cur.sptr[m] + (size_t)k * 1024u, 1024u, &full[stage]);
            }
            ptx::tma_load_2d(sb + SL.x_off, &tm_x, k * 128, cur.d.row0, &full[stage]);
            if (a.sums) ptx::tma_load_2d(sb + SL.sum_off, &tm_s, k * 4, cur.d.row0, &full[stage]);
          }
          gtrace(a.trace, 1, gtile);
        }
        ++gtile;
        __syncwarp();
        if (!done && !a.withhold) {
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        } else if (done) {
          armed &= ~(1u << stage);  // released by the consumers: its last copy has landed
        }
        if (++stage == SL.stages) {
          stage = 0;
          phase ^= 1u;
        }
        if (kt == 0 && !done) {
          load_item<NMAT, NT8>(ahead, nxt, total, nchunks, a, L, KT);
          if (lane == 0) gtrace(a.trace, 4, gitem);
        }
      }
      ++gitem;
      if (done) break;
    }
    // No copy may still be landing when the CTA exits.  Without an abort every
    // armed stage was consumed; after one, consumers skip their waits, so wait here.
    if (lane == 0 && (!ok || *abort_flag))
      for (int st = 0; st < SL.stages; ++st)
        if (armed & (1u << st)) mbar_drain(&full[st], (armed_par >> st) & 1u);
    __syncwarp();
  } else {
    const int s = warp, g = lane >> 2, c = lane & 3;
    int stage = 0, gtile = 0, gitem = 0;
    uint32_t phase = 0;
    while (true) {
      // first stage of the next item (or the end marker); all consumer warps agree
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&full[stage], phase, abort_flag, a.wait))) *abort_flag = 1;
      consumer_sync();
      if (*abort_flag) {
        ok = false;
        break;
      }
      const ItemDesc w = slot[stage];
      if (w.it < 0) break;
      if (threadIdx.x == 0) gtrace(a.trace, 6, gitem);
      const int row0 = w.row0, rows = w.rows, ntiles = w.ntiles;
      const int fm[2] = {w.f0, w.f1};
      const float ts[2] = {w.ts0, w.ts1};
      float fscale[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) fscale[m] = fm[m] == MOE_FMT_NVFP4 ? 1.0f : 16777216.0f;  // integer sums carry 2^-24
      float acc[NMAT][2][NT8][4];
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[m][t][nt][j] = 0.0f;
      bool first_1bit = false;
      if constexpr (I1) {
        if (fm[0] == MOE_FMT_INT1) {
          consume_f1<NMAT, NT8, MOE_FMT_INT1, I1>(fm[1], SL, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, a.trace, gtile, a.wait);
          first_1bit = true;
        }
      }
      if (!first_1bit) switch (fm[0]) {
        case MOE_FMT_INT2: consume_f1<NMAT, NT8, MOE_FMT_INT2, I1>(fm[1], SL, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, a.trace, gtile, a.wait); break;
        case MOE_FMT_INT3: consume_f1<NMAT, NT8, MOE_FMT_INT3, I1>(fm[1], SL, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, a.trace, gtile, a.wait); break;
        case MOE_FMT_INT4: consume_f1<NMAT, NT8, MOE_FMT_INT4, I1>(fm[1], SL, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, a.trace, gtile, a.wait); break;
        default: consume_f1<NMAT, NT8, MOE_FMT_NVFP4, I1>(fm[1], SL, smem, full, empty, abort_flag, ntiles, stage, phase, ok, acc, a.trace, gtile, a.wait); break;
      }
      // lane outputs: weight row nl = 32s + 4g + 2t + (j >> 1), token row nt*8 + 2c + (j & 1)
      if (ok && a.P == 1) {
        bool range = false;
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt) {
          float hs[2] = {0.0f, 0.0f};  // this lane's part of the group sums of h for tokens 2c, 2c+1
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int tk = nt * 8 + 2 * c + (j & 1);
              if (tk < rows) {
                float v[NMAT];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) v[m] = acc[m][t][nt][j] * fscale[m];
                hs[j & 1] += store_output<NMAT>(a, row0 + tk, w.nb * kBlockRows + 32 * s + 4 * g + 2 * t + (j >> 1),
                                                v, ts, range, w.e);
              }
            }
          if (a.out_sum) {  // warp s owns the 32 weight rows of one down-projection input group
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
              hs[0] += __shfl_xor_sync(0xffffffffu, hs[0], o);
              hs[1] += __shfl_xor_sync(0xffffffffu, hs[1], o);
            }
            const int grp = (w.nb * kBlockRows + 32 * s) / 32, G = a.N / 32;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int tk = nt * 8 + 2 * c + u;
              if (g == 0 && tk < rows) a.out_sum[(size_t)(row0 + tk) * G + grp] = hs[u];
            }
          }
        }
        if (range) report_range(a.status);
      } else if (ok) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int tk = nt * 8 + 2 * c + (j & 1);
              if (tk < rows) {
                const int n = w.nb * kBlockRows + 32 * s + 4 * g + 2 * t + (j >> 1);
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
                  a.part[(((size_t)w.p * a.R + row0 + tk) * NMAT + m) * a.N + n] = acc[m][t][nt][j] * fscale[m];
              }
            }
      }
      if (threadIdx.x == 0) gtrace(a.trace, 7, gitem);
      ++gitem;
    }
  }

  if (!ok) {
    *abort_flag = 1;
    if (a.status) atomicExch(a.status, (int32_t)MOE_ERR_TIMEOUT);
  }
  __syncthreads();
}

// Split-K epilogue: block (r, b) sums the P parts of outputs 256b..256b+255 of
// expert row r in order, then applies SwiGLU (gate/up) or writes o (down).
// Gate/up of integer layers also writes the group sums of h for the down GEMV.
template <int NMAT>
__global__ void __launch_bounds__(256) gemv_fixup_kernel(GemvArgs a, const int32_t* idx) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  const int r = blockIdx.x;
  const int e = idx[a.perm[r]];
  const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
  float ts[2];
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int i = e * 3 + a.proj + (m < NMAT ? m : 0);
    ts[m] = L.fmt[i] == MOE_FMT_NVFP4 ? L.tscale[i] : 1.0f;
  }
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.y * 256 + threadIdx.x - lane;  // warp-uniform: 32 outputs = one group
  if (n0 < a.N) {
    const int n = n0 + lane;
    float v[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      float sum = 0.0f;
      for (int q = 0; q < a.P; ++q) sum += a.part[(((size_t)q * a.R + r) * NMAT + m) * a.N + n];
      v[m] = sum;
    }
    bool range = false;
    float h = store_output<NMAT>(a, r, n, v, ts, range, e);
    if (range) report_range(a.status);
    if (a.out_sum) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) h += __shfl_xor_sync(0xffffffffu, h, o);
      if (lane == 0) a.out_sum[(size_t)r * (a.N / 32) + n0 / 32] = h;
    }
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 gemv_tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int gemv_sm_count() {
  static int n[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

// The packed buffer as 3D tensor of u32: x = 32 words (128 bytes), y = 4 such
// lines per 512-byte word row, z = word rows.  Box: 32 x 2 x (4 groups * wpg).
bool encode_code_map(CUtensorMap* map, const uint8_t* packed, uint64_t packed_bytes, int wpg) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gemv_tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {32u, 4u, (cuuint64_t)(packed_bytes / 512u)};
  const cuuint64_t strides[2] = {128u, 512u};
  const cuuint32_t box[3] = {32u, 2u, (cuuint32_t)(4 * wpg)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(packed), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major [rows][cols] matrix of 2- or 4-byte elements; box of box_cols x box_rows.
bool encode_rows_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, int rows, int cols,
                     int box_cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gemv_tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * (cuuint64_t)esize};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stage layout for the widest formats of the layer at each matrix position.
// Shared memory is budgeted for the CTAs per SM that the registers allow: four
// (one matrix, one token tile), three (two matrices, one token tile) or two
// (two token tiles).
StageLayout stage_layout(int nmat, int nt8, const int* wmax) {
  StageLayout L{};
  int off = 0;
  for (int m = 0; m < nmat; ++m) {
    L.box[m] = 1024 * wmax[m];
    L.code_off[m] = off;
    off += 2 * L.box[m];
  }
  for (int m = 0; m < nmat; ++m) {
    L.scale_off[m] = off;
    off += 1024;
  }
  L.x_off = off;
  off += nt8 * 8 * 256;
  L.sum_off = off;
  off += nt8 * 8 * 16;
  L.bytes = (off + 1023) / 1024 * 1024;
  const int cta_per_sm = nt8 == 1 ? (nmat == 1 ? 4 : 3) : 2;
  const int budget = 227 * 1024 / cta_per_sm - 1024 - kCtrlBytes - 1024;  // minus alignment, control, per-CTA reserve
  L.stages = budget / L.bytes;
  if (L.stages > kMaxStages) L.stages = kMaxStages;
  if (L.stages < 2) L.stages = 2;
  return L;
}

template <int NMAT, int NT8, bool I1>
cudaError_t launch_n(GemvArgs g, const uint8_t* packed, uint64_t packed_bytes, const void* act, const float* sums,
                     const int* wmax, int max_chunks, cudaStream_t stream) {
  CUtensorMap m1, m2, m3, m4, mx, ms;
  if (!encode_code_map(&m1, packed, packed_bytes, 1) || !encode_code_map(&m2, packed, packed_bytes, 2) ||
      !encode_code_map(&m3, packed, packed_bytes, 3) ||
      !encode_code_map(&m4, packed, packed_bytes, 4) ||
      !encode_rows_map(&mx, act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, g.R, g.K, 128, 8 * NT8))
    return cudaErrorInvalidValue;
  g.sums = sums != nullptr;
  if (g.sums) {
    if (!encode_rows_map(&ms, sums, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, g.R, g.K / 32, 4, 8 * NT8))
      return cudaErrorInvalidValue;
  } else {
    ms = mx;  // unused
  }
  g.st = stage_layout(NMAT, NT8, wmax);
  const int smem = g.st.stages * g.st.bytes + 1024 + kCtrlBytes;
  auto kern = expert_gemv_kernel<NMAT, NT8, I1>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (err != cudaSuccess) return err;
  const long long items = (long long)max_chunks * (g.N / kBlockRows) * g.P;
  long long grid = (long long)gemv_sm_count() * (per_sm > 0 ? per_sm : 1);
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  launch_chained(kern, dim3((unsigned)grid), dim3(kGemvThreads), smem, stream, m1, m2, m3, m4, mx, ms, g);
  return cudaGetLastError();
}

}  // namespace

int gemv_split(long long R, int E, int N, int K, int nmat) {
  const long long chunks = R < E ? R : E;  // active experts at most
  long long base = chunks * (N / kBlockRows);
  if (base < 1) base = 1;
  const long long target = 4LL * 3 * 148;  // about four items per CTA at three CTAs per SM
  long long P = (target + base - 1) / base;
  const long long per_part = R * (long long)N * nmat * 4;
  const long long mem_cap = (8LL << 20) / (per_part > 0 ? per_part : 1);
  const int kt = K / 128;
  long long cap = kt / 4 > 1 ? kt / 4 : 1;  // parts of at least four tiles
  if (cap > kMaxSplit) cap = kMaxSplit;
  if (P > cap) P = cap;
  if (P > mem_cap) P = mem_cap;
  return P < 1 ? 1 : (int)P;
}

cudaError_t launch_expert_gemv(const uint8_t* packed, uint64_t packed_bytes, const uint8_t* fmt_host, int E, int H,
                               int F, int R, int k, bool fp4, bool gateup, int max_chunks, int chunk_rows,
                               const Workspace& ws, int32_t* status, uint64_t* trace, GemmHooks hooks,
                               bool outliers, cudaStream_t stream) {
  GemvArgs g{};
  g.outliers = outliers ? 1 : 0;
  g.trace = reinterpret_cast<unsigned long long*>(trace);
  g.wait = hooks.wait_cycles ? (long long)hooks.wait_cycles : kGemvWait;
  g.withhold = hooks.withhold ? 1 : 0;
  g.packed = packed;
  g.E = E;
  g.H = H;
  g.F = F;
  g.topk = k;
  g.R = R;
  g.chunks = ws.chunks;
  g.chunk_count = ws.chunk_count;
  g.perm = ws.perm;
  g.part = ws.part;
  g.work = ws.counters + (gateup ? 0 : 1);
  g.status = status;
  const void* act;
  const float* sums;
  int wmax[2] = {2, 2};
  for (int e = 0; e < E; ++e)
    for (int m = 0; m < (gateup ? 2 : 1); ++m) {
      const int w = fmt_words(fmt_host[e * 3 + (gateup ? m : 2)]);
      if (w > wmax[m]) wmax[m] = w;
    }
  if (gateup) {
    g.N = F;
    g.K = H;
    g.proj = 0;
    act = ws.xs;
    sums = fp4 ? nullptr : ws.xsum;
    g.row_scale = fp4 ? ws.sx : nullptr;
    g.xinv = fp4 ? nullptr : ws.xinv;
    g.out = ws.h;
    g.out_sum = fp4 ? nullptr : ws.hsum;
  } else {
    g.N = H;
    g.K = F;
    g.proj = 2;
    act = fp4 ? ws.hb : ws.h;
    sums = fp4 ? nullptr : ws.hsum;
    g.row_scale = fp4 ? ws.sh : nullptr;
    g.out = ws.o;
    g.out_sum = nullptr;
  }
  const int nmat = gateup ? 2 : 1;
  g.P = gemv_split(R, E, g.N, g.K, nmat);
  g.act16 = (const __half*)act;
  if (chunk_rows != 8) return cudaErrorInvalidValue;  // the host plans 8-row chunks (one token tile)
  bool any1 = false;  // a 1-bit matrix among this projection's
  for (int e = 0; e < E; ++e)
    for (int m = 0; m < (gateup ? 2 : 1); ++m) any1 |= fmt_host[e * 3 + (gateup ? m : 2)] == MOE_FMT_INT1;
  cudaError_t err;
  if (gateup)
    err = any1 ? launch_n<2, 1, true>(g, packed, packed_bytes, act, sums, wmax, max_chunks, stream)
               : launch_n<2, 1, false>(g, packed, packed_bytes, act, sums, wmax, max_chunks, stream);
  else
    err = any1 ? launch_n<1, 1, true>(g, packed, packed_bytes, act, sums, wmax, max_chunks, stream)
               : launch_n<1, 1, false>(g, packed, packed_bytes, act, sums, wmax, max_chunks, stream);
  if (err != cudaSuccess || g.P == 1) return err;
  if (gateup)
    launch_chained(gemv_fixup_kernel<2>, dim3(R, (g.N + 255) / 256), dim3(256), 0, stream, g, ws.idx);
  else
    launch_chained(gemv_fixup_kernel<1>, dim3(R, (g.N + 255) / 256), dim3(256), 0, stream, g, ws.idx);
  return cudaGetLastError();
}

}  // namespace moe

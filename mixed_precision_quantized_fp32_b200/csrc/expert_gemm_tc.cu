// Dequant-fused grouped expert GEMM on the 5th-generation tensor cores
// (tcgen05.mma kind::f16, fp32 accumulators in TMEM) for batches with many
// token rows per expert (prefill).
//
// This is the pages' "packed linear" operator (MoE mixed-precision page,
// sec. 2.3 / 3.5: experts stored as independently quantized 128-column blocks
// that a custom kernel unpacks) with the activation fused into the epilogue
// (its sec. 3.6, "fused linear + activation"), built for sm_100a:
//   * persistent clusters of two CTAs (one CTA per SM) walk (token chunk, weight
//     tiles) work items; chunk = up to 256 consecutive expert-sorted rows of one
//     expert; each CTA owns 128-row weight tiles (gate + up, or two down tiles);
//   * three rings of shared-memory slots per CTA: raw slots hold a stage's packed
//     codes + scales (64 inputs = two quantization groups) and are freed as soon
//     as they are dequantized, so their copies run many stages ahead; A slots
//     hold the dequantized weight tiles and B slots this CTA's half of the
//     activation tile, both freed by the MMA commit;
//   * warp 16 (one lane) streams the codes and scales of this CTA's weight tiles
//     into the raw ring with 1D bulk copies; warp 18 (one lane) loads the
//     activation half-tile into the B ring with a 2D TMA load (128-byte swizzle;
//     a half-height box for chunks of at most 128 rows); no copy is multicast;
//   * warps 0-15 turn codes into fp16 operands (exponent-bias unpack: a code u
//     OR'ed into the mantissa of 1024.0 gives 1024+u exactly; one FMA removes
//     the bias and the code offset, one multiply applies the group scale),
//     release the raw slot, and write the operands straight into the swizzled
//     K-major layout the tensor core reads, then arrive on the even CTA's barrier;
//   * warp 17 of the even CTA issues tcgen05.mma.cta_group::2 M=256 (128 weight
//     rows from each CTA) x N<=256 (token rows, half from each CTA) x K=16,
//     warp-wide with one elected lane, and commits to both CTAs' mbarriers;
//     warp 17 of the odd CTA reports its activation tiles to the even CTA;
//   * warps 0-15 then drain their own TMEM (tcgen05.ld) into the SwiGLU / scale
//     epilogue (plus the outlier side lists' residual dot in OUT instantiations).
// Shapes whose weight tiles do not pair run the same kernel on single CTAs
// (cta_group::1, M=128, the whole token chunk per CTA).
// Every mbarrier wait is bounded; a wait that gives up raises the abort flags
// of both CTAs so every role leaves its loop and MOE_ERR_TIMEOUT goes to the
// status word.  Copies and MMAs still in flight are waited for, and the pair
// meets at a cluster barrier, before TMEM is freed and the CTAs return.
#include <algorithm>
#include <type_traits>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "moe_common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kTcBM = 128;   // weight rows per work item (MMA M)
constexpr int kTcBN = kTcChunkRows;  // token rows per work item (max MMA N)
#ifndef MOE_TC_BK
#define MOE_TC_BK 64
#endif
constexpr int kTcBK = MOE_TC_BK;        // inputs per pipeline stage (32 or 64)
constexpr int kGroups = kTcBK / 32;     // quantization groups per stage
constexpr int kRowBytes = kTcBK * 2;    // bytes of one fp16 tile row = swizzle span (64 or 128)
static_assert(kTcBK == 32 || kTcBK == 64, "stage depth");
#ifndef MOE_TC_DEQ_WARPS
#define MOE_TC_DEQ_WARPS 16
#endif
constexpr int kDeqWarps = MOE_TC_DEQ_WARPS;  // dequantize + epilogue warps (8 or 16)
static_assert(kDeqWarps == 8 || kDeqWarps == 16, "dequant warps");
constexpr int kThreadsPerRow = kDeqWarps * 32 / 128;
constexpr int kRawWarp = kDeqWarps, kMmaWarp = kDeqWarps + 1, kBWarp = kDeqWarps + 2;
constexpr int kTcThreads = 32 * (kDeqWarps + 3);
constexpr long long kWaitLimit = 4000000000LL;  // clock cycles, ~2 s

// CG2: the work item runs on a pair of CTAs (one cluster) with cta_group::2
// MMAs, each CTA holding half of the activation tile's token rows.
// Three rings of shared-memory slots per CTA:
//  * raw slots: the packed codes and scales of NMAT weight tiles for one stage,
//    freed as soon as the dequant warps have read them, so their copies run many
//    stages ahead;
//  * A slots: the NMAT dequantized weight tiles the tensor core reads;
//  * B slots: the activation tile; its own ring, so activation loads are issued
//    several stages ahead instead of waiting for a weight-tile slot to free.
// A and B slots are freed by the MMA commit.  The code slot is sized for the
// widest format the launch meets (Ring).
template <int NMAT, bool CG2 = false>
struct TcCfg {
  static constexpr int kBRows = CG2 ? kTcBN / 2 : kTcBN;
  static constexpr int kBBytes = kBRows * kRowBytes;  // activation tile (this CTA's rows), one B slot
  static constexpr int kABytes = kTcBM * kRowBytes;   // dequantized weight tile
  static constexpr int kASlotBytes = NMAT * kABytes;  // one A slot
  static constexpr int kScaleBytes = kGroups * 256;   // one fp16 group or two e4m3 blocks x 128 rows
};
constexpr int kMaxRaw = 16, kMaxA = 4, kMaxB = 8;
constexpr int kBarBytes = 640;                       // barriers, TMEM slot and abort flag
constexpr int kSmemMax = 232448;                     // opt-in shared memory per CTA
static_assert(8 * (2 * kMaxRaw + 2 * kMaxA + 3 * kMaxB + 2) + 16 <= kBarBytes, "barrier area");

struct Ring {
  int a_slots;      // weight-tile slots (<= kMaxA)
  int b_slots;      // activation-tile slots (<= kMaxB)
  int raw_slots;    // raw slots (<= kMaxRaw)
  int code_bytes;   // one matrix's code slot: kGroups x 512 bytes per code word of the widest format
  int raw_bytes;    // one raw slot: NMAT code slots, then NMAT scale slots
  int off_b;        // offset of the B ring (after the A slots)
  int off_raw;      // offset of the raw ring (after the B slots)
};

template <int NMAT, bool CG2>
Ring make_ring(int max_words) {
  using C = TcCfg<NMAT, CG2>;
  Ring r;
  r.a_slots = CG2 ? 4 : 2;
  r.b_slots = CG2 ? 4 : 3;
  r.code_bytes = kGroups * 512 * max_words;
  r.raw_bytes = (NMAT * (r.code_bytes + C::kScaleBytes) + 127) / 128 * 128;
  for (;;) {
    r.off_b = r.a_slots * C::kASlotBytes;
    r.off_raw = r.off_b + r.b_slots * C::kBBytes;
    r.raw_slots = min(kMaxRaw, (kSmemMax - kBarBytes - 1024 - r.off_raw) / r.raw_bytes);
    if (r.raw_slots >= 4 || r.b_slots <= 2) break;
    --r.b_slots;  // keep the raw ring at least 4 deep
  }
  return r;
}
inline int ring_smem(const Ring& r) { return r.off_raw + r.raw_slots * r.raw_bytes + kBarBytes + 1024; }

struct TcArgs {
  const uint8_t* packed;
  int E, H, F;
  int N, K;                // output rows (weight rows) and inputs of this GEMM
  int proj;                // 0: gate+up with SwiGLU epilogue; 2: down
  int pair;                // down with NMAT == 2: the two "matrices" are weight tiles 2p, 2p+1 of one
                           // matrix, sharing each activation tile (half the activation reads per FLOP)
  const int32_t* chunks;   // (expert, first row, rows) triples
  const int32_t* chunk_count;
  const float* row_scale;  // NVFP4: gate/up -> per-token sx, down -> per-row sh; null for integer layers
  const float* xinv;       // integer gate/up: per-row 2^e undoing the activations' prescale (null otherwise)
  const __half* act16;     // the fp16 activations [rows][K] (the residual term of outlier side lists)
  const int32_t* perm;
  int topk;
  void* out;               // gate/up: h [rows][F] (fp16, or fp32 for NVFP4); down: o fp32 [rows][H]
  int32_t* status;
  unsigned long long* trace;  // diagnostics: per-stage clock64 stamps of CTA 0 (or null)
  Ring ring;
  long long wait;             // budget of the pipeline waits, clock cycles
  int withhold;               // test hook: the TMA warp issues no loads (the waits run out)
};

// Stamp event `ev` of global stage counter `i` (CTA 0 only, first MOE_TRACE_STAGES stages).
__device__ __forceinline__ void trace_stamp(unsigned long long* tr, int ev, int i) {
  if (tr && blockIdx.x == 0 && i < MOE_TRACE_STAGES) tr[ev * MOE_TRACE_STAGES + i] = (unsigned long long)clock64();
}

__device__ __forceinline__ uint32_t h2fma(uint32_t a, uint32_t b, uint32_t c) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b), *reinterpret_cast<__half2*>(&c));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2mul(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Four e2m1 pairs (one 32-bit word, byte b = codes 2b, 2b+1) -> four fp16 pairs.
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t* o) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// Eight inputs (chunk c = inputs 8c..8c+7 of the staged group) of weight row n
// as four fp16 pairs in natural order.  codes: shared address of the group's
// words [word][128 rows]; scales: shared address of [128] fp16 (integer) or
// [2 blocks][128] e4m3 (NVFP4).  The format is a template parameter so a
// stage's chunks are straight-line code.
template <int FMT>
__device__ __forceinline__ uint4 dequant_chunk(uint32_t codes, uint32_t scales, int n, int c) {
  uint32_t v[4];
  if (FMT == MOE_FMT_NVFP4) {
    const __half_raw sr =
        __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)ptx::lds_u8(scales + (c >> 1) * 128 + n), __NV_E4M3);  // exact
    const uint32_t p = (uint32_t)sr.x | ((uint32_t)sr.x << 16);
    e2m1x8_to_f16(ptx::lds_u32(codes + 4 * (c * 128 + n)), v);
#pragma unroll
    for (int b = 0; b < 4; ++b) v[b] = h2mul(v[b], p);  // exact: <= 6 significant bits
  } else {
    // A field u of weight f (bit position log2 f of both half-words) OR'ed into
    // the mantissa of 1024.0 reads as 1024 + f*u; one FMA with 1/f and
    // -(1024/f + offset) gives q = u - offset exactly, then one multiply by the
    // group scale rounds s*q once.
    const uint32_t s = ptx::lds_u16(scales + 2 * n);
    const uint32_t s2 = s | (s << 16);
    constexpr uint32_t kMagic = 0x64006400u;
    if (FMT == MOE_FMT_INT1) {
      // sign code, pair j of chunk c at bit 4c + j (and 16 above): 1024 + 2^j u after
      // the OR; one FMA with 2^-j and -1024*2^-j gives u, a second with 2s and -s
      // gives s*(2u - 1) = +-s in one rounding
      constexpr uint32_t kMul1[4] = {0x3C003C00u, 0x38003800u, 0x34003400u, 0x30003000u};  // 2^-j
      constexpr uint32_t kSub1[4] = {0xE400E400u, 0xE000E000u, 0xDC00DC00u, 0xD800D800u};  // -1024*2^-j
      const uint32_t w = ptx::lds_u32(codes + 4 * n) >> (4 * c);
      const uint32_t s2x2 = h2mul(s2, 0x40004000u), neg_s2 = s2 ^ 0x80008000u;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[j] = h2fma(h2fma((w & (0x00010001u << j)) | kMagic, kMul1[j], kSub1[j]), s2x2, neg_s2);
    } else if (FMT == MOE_FMT_INT4) {
      const uint32_t w = ptx::lds_u32(codes + 4 * (c * 128 + n)), w8 = w >> 8;
      v[0] = h2mul(h2fma((w & 0x000F000Fu) | kMagic, 0x3C003C00u, 0xE408E408u), s2);   // u - 8
      v[1] = h2mul(h2fma((w & 0x00F000F0u) | kMagic, 0x2C002C00u, 0xD480D480u), s2);   // 16u / 16 + 64 - 72
      v[2] = h2mul(h2fma((w8 & 0x000F000Fu) | kMagic, 0x3C003C00u, 0xE408E408u), s2);
      v[3] = h2mul(h2fma((w8 & 0x00F000F0u) | kMagic, 0x2C002C00u, 0xD480D480u), s2);
    } else {
      // fields of pair j at bits 2j (weight 4^j); INT3 adds bit 2 of the pair's
      // codes from word 2 (pair m = 4c+j at bits 8*(c/2) + c%2 + 2j and 16 above),
      // which one rotation moves to bit 2j+2
      constexpr uint32_t kMul[4] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u};        // 4^-j
      constexpr uint32_t kSub2[4] = {0xE402E402u, 0xDC08DC08u, 0xD420D420u, 0xCC80CC80u};       // -(1024/4^j + 2)
      constexpr uint32_t kSub3[4] = {0xE404E404u, 0xDC10DC10u, 0xD440D440u, 0xCD00CD00u};       // -(1024/4^j + 4)
      const uint32_t lo = ptx::lds_u32(codes + 4 * ((c >> 1) * 128 + n)) >> (8 * (c & 1));
      uint32_t hh = 0u;
      if (FMT == MOE_FMT_INT3) {
        const uint32_t hw = ptx::lds_u32(codes + 4 * (2 * 128 + n));
        hh = __funnelshift_r(hw, hw, (uint32_t)(8 * (c >> 1) + (c & 1) + 30) & 31u);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t raw = (lo & (0x00030003u << (2 * j))) | kMagic;
        if (FMT == MOE_FMT_INT3) raw |= hh & (0x00040004u << (2 * j));
        v[j] = h2mul(h2fma(raw, kMul[j], FMT == MOE_FMT_INT3 ? kSub3[j] : kSub2[j]), s2);
      }
    }
  }
  return make_uint4(v[0], v[1], v[2], v[3]);
}

// Byte offset of 16-byte chunk c of row n in a K-major tile of kRowBytes rows
// with the matching swizzle (8-row atoms; chunk index XOR'ed with the row bits
// the swizzle mode uses: row%8 for 128-byte rows, (row/2)%4 for 64-byte rows).
__device__ __forceinline__ int tile_offset(int n, int c) {
  if (kRowBytes == 128) return (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4);
  return (n >> 3) * 512 + (n & 7) * 64 + ((c ^ ((n >> 1) & 3)) << 4);
}
__device__ __forceinline__ uint64_t tile_desc(uint32_t start) {
  return kRowBytes == 128 ? ptx::sw128_desc(start) : ptx::sw64_desc(start);
}

// Byte offset of the words of groups g..g+kGroups-1 (inputs 32g..) of weight tile
// mt: [group][word][128 rows], contiguous kGroups*wpg*512 bytes (g % kGroups == 0).
__device__ __forceinline__ uint64_t code_stage_offset(int mt, int g, int K, int wpg) {
  return ((((uint64_t)mt * (uint64_t)(K >> 7) + (uint64_t)(g >> 2)) * 4u + (uint64_t)(g & 3)) * (uint64_t)wpg *
          128u) * 4u;
}
// Byte offset of the scales of groups g..g+kGroups-1 of weight tile mt (kGroups*256 bytes).
__device__ __forceinline__ uint64_t scale_stage_offset(int mt, int g, int K, int fmt) {
  if (fmt == MOE_FMT_NVFP4) return ((uint64_t)mt * (uint64_t)(K >> 4) + (uint64_t)g * 2u) * 128u;
  return ((uint64_t)mt * (uint64_t)(K >> 5) + (uint64_t)g) * 256u;
}

// The mbarriers after the rings.
struct Bars {
  uint64_t* raw_full;   // [kMaxRaw] codes + scales landed (tx count)
  uint64_t* raw_empty;  // [kMaxRaw] this CTA's dequant warps have read them
  uint64_t* a_full;     // [kMaxA] the dequant warps of the pair wrote the weight tiles (the even CTA's counts)
  uint64_t* a_empty;    // [kMaxA] the MMAs reading the weight tiles are done
  uint64_t* b_full;     // [kMaxB] this CTA's activation tile landed (tx count)
  uint64_t* b_empty;    // [kMaxB] the MMAs reading the activation tile are done
  uint64_t* b_peer;     // [kMaxB] (even CTA) the odd CTA's activation tile landed
  uint64_t* acc_full;
  uint64_t* acc_empty;
};
__device__ __forceinline__ Bars bars_at(uint64_t* b) {
  Bars r;
  r.raw_full = b;
  r.raw_empty = b + kMaxRaw;
  r.a_full = b + 2 * kMaxRaw;
  r.a_empty = r.a_full + kMaxA;
  r.b_full = r.a_empty + kMaxA;
  r.b_empty = r.b_full + kMaxB;
  r.b_peer = r.b_empty + kMaxB;
  r.acc_full = r.b_peer + kMaxB;
  r.acc_empty = r.acc_full + 1;
  return r;
}

// Position of the dequant warps in the raw and A rings, and the global stage
// counter (trace index).
struct Cursor {
  int rs;
  uint32_t rph;
  int as;
  uint32_t aph;
  int g;
};

// Dequantize every stage of one work item (formats F0 = first matrix, F1 =
// second): wait for the stage's codes in a raw slot, convert this thread's units
// to registers and release the raw slot, wait for the A slot to be free (its
// previous MMAs done), write the units in the tensor core's layout and arrive on
// the A slot's barrier (the even CTA's, for a pair).  Returns false if a bounded
// wait gave up.
template <int NMAT, bool CG2, int F0, int F1>
__device__ __noinline__ bool dequant_item(const Ring R, long long wait, uint32_t smem, uint64_t* bars,
                                          volatile int* abort_flag, int ksteps, int n, int u0, Cursor& cursor,
                                          unsigned long long* trace) {
  using C = TcCfg<NMAT, CG2>;
  constexpr int kUnits = NMAT * kGroups * 4 / kThreadsPerRow;
  static_assert(NMAT == 1 || kUnits % 2 == 0, "units must alternate matrices evenly");
  const Bars B = bars_at(bars);
  const int lane = threadIdx.x & 31;
  const int cg0 = u0 / NMAT;
  // the cursor lives in registers for the loop (a reference would be re-read after every
  // shared-memory store)
  int rs = cursor.rs, as = cursor.as, g = cursor.g;
  uint32_t rph = cursor.rph, aph = cursor.aph;
  bool ok = true;
  for (int ks = 0; ks < ksteps; ++ks) {
    if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.raw_full[rs], rph, abort_flag, wait))) {
      ok = false;
      break;
    }
    if (threadIdx.x == 0) trace_stamp(trace, 2, g);
    const uint32_t rb = smem + (uint32_t)(R.off_raw + rs * R.raw_bytes);  // shared address of the raw slot
    uint4 v[kUnits];
#pragma unroll
    for (int i = 0; i < kUnits; ++i) {
      const int m = i % NMAT, cg = cg0 + i / NMAT, gr = cg >> 2;
      const uint32_t scales = rb + (uint32_t)(NMAT * R.code_bytes + m * C::kScaleBytes + gr * 256);
      if (m == 0) {
        v[i] = dequant_chunk<F0>(rb + (uint32_t)(gr * fmt_words(F0) * 512), scales, n, cg & 3);
      } else {
        v[i] = dequant_chunk<F1>(rb + (uint32_t)(R.code_bytes + gr * fmt_words(F1) * 512), scales, n, cg & 3);
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&B.raw_empty[rs]);  // release orders this warp's reads before it
    if (++rs == R.raw_slots) {
      rs = 0;
      rph ^= 1u;
    }
    // the A slot's previous MMAs are done
    if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.a_empty[as], aph ^ 1u, abort_flag, wait))) {
      ok = false;
      break;
    }
    const uint32_t ab = smem + (uint32_t)(as * C::kASlotBytes);
#pragma unroll
    for (int i = 0; i < kUnits; ++i) {
      const int m = i % NMAT, cg = cg0 + i / NMAT;
      ptx::sts_v4(ab + (uint32_t)(m * C::kABytes + tile_offset(n, cg)), v[i]);
    }
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (CG2)
        ptx::mbar_arrive_cluster(&B.a_full[as], 0);  // the even CTA issues the pair's MMAs
      else
        ptx::mbar_arrive(&B.a_full[as]);
    }
    if (threadIdx.x == 0) trace_stamp(trace, 3, g);
    ++g;
    if (++as == R.a_slots) {
      as = 0;
      aph ^= 1u;
    }
  }
  cursor = Cursor{rs, rph, as, aph, g};
  return ok;
}

// Runtime format pair -> the matching dequant_item instantiation.  I1: the launch
// meets 1-bit matrices; their cases are compiled only into the I1 kernels, so the
// kernels for layers without them keep their size and register allocation.
template <int NMAT, bool CG2, bool I1, int F0>
__device__ __forceinline__ bool dequant_item_f1(int f1, const Ring R, long long wait, uint32_t smem, uint64_t* bars,
                                                volatile int* abort_flag, int ksteps, int n, int u0, Cursor& cur,
                                                unsigned long long* trace) {
  if (NMAT == 1) return dequant_item<NMAT, CG2, F0, F0>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
  if constexpr (I1) {
    if (f1 == MOE_FMT_INT1)
      return dequant_item<NMAT, CG2, F0, MOE_FMT_INT1>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
  }
  switch (f1) {
    case MOE_FMT_INT2: return dequant_item<NMAT, CG2, F0, MOE_FMT_INT2>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    case MOE_FMT_INT3: return dequant_item<NMAT, CG2, F0, MOE_FMT_INT3>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    case MOE_FMT_INT4: return dequant_item<NMAT, CG2, F0, MOE_FMT_INT4>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    default: return dequant_item<NMAT, CG2, F0, MOE_FMT_NVFP4>(R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
  }
}
template <int NMAT, bool CG2, bool I1>
__device__ __forceinline__ bool dequant_item_any(int f0, int f1, const Ring R, long long wait, uint32_t smem,
                                                 uint64_t* bars, volatile int* abort_flag, int ksteps, int n, int u0,
                                                 Cursor& cur, unsigned long long* trace) {
  if constexpr (I1) {
    if (f0 == MOE_FMT_INT1)
      return dequant_item_f1<NMAT, CG2, I1, MOE_FMT_INT1>(f1, R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
  }
  switch (f0) {
    case MOE_FMT_INT2: return dequant_item_f1<NMAT, CG2, I1, MOE_FMT_INT2>(f1, R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    case MOE_FMT_INT3: return dequant_item_f1<NMAT, CG2, I1, MOE_FMT_INT3>(f1, R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    case MOE_FMT_INT4: return dequant_item_f1<NMAT, CG2, I1, MOE_FMT_INT4>(f1, R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
    default: return dequant_item_f1<NMAT, CG2, I1, MOE_FMT_NVFP4>(f1, R, wait, smem, bars, abort_flag, ksteps, n, u0, cur, trace);
  }
}

// OUT: the layer has outlier side lists (their residuals are added in the epilogue)
template <int NMAT, bool CG2, bool I1, bool OUT>
__global__ void __launch_bounds__(kTcThreads, 1)
    expert_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_bh,
                          const TcArgs a) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  using C = TcCfg<NMAT, CG2>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer arithmetic (an
  // integer round trip would turn every access through it into a generic one)
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  const Ring R = a.ring;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + R.off_raw + R.raw_slots * R.raw_bytes);
  const Bars B = bars_at(bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(B.acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs: the even CTA (rank 0) issues the MMAs of both, so the dequant and
  // epilogue warps of both CTAs arrive on its barriers (a plain remote arrive:
  // release at CTA scope, as a cluster-scope release costs ~1600 cycles here);
  // its commits reach both CTAs.
  const uint32_t rank = CG2 ? ptx::cluster_ctarank() : 0u;
  constexpr int kPairCtas = CG2 ? 2 : 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < R.raw_slots; ++s) {
      ptx::mbar_init(&B.raw_full[s], 1);
      ptx::mbar_init(&B.raw_empty[s], kDeqWarps);  // this CTA's dequant warps
    }
    for (int s = 0; s < R.a_slots; ++s) {
      ptx::mbar_init(&B.a_full[s], kDeqWarps * kPairCtas);  // one arrival per dequant warp of the pair
      ptx::mbar_init(&B.a_empty[s], 1);
    }
    for (int s = 0; s < R.b_slots; ++s) {
      ptx::mbar_init(&B.b_full[s], 1);
      ptx::mbar_init(&B.b_empty[s], 1);
      ptx::mbar_init(&B.b_peer[s], 1);
    }
    ptx::mbar_init(B.acc_full, 1);
    ptx::mbar_init(B.acc_empty, kDeqWarps * kPairCtas);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    if (CG2) {
      ptx::tmem_alloc2(tmem_slot, 512);
      ptx::tmem_relinquish2();
    } else {
      ptx::tmem_alloc(tmem_slot, 512);
      ptx::tmem_relinquish();
    }
  }
  if (warp == kBWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_b);
    ptx::prefetch_tmap(&tmap_bh);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (CG2) ptx::cluster_sync();  // the peer's barriers are initialised before any remote arrival
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // work items per chunk: 128-row weight tiles (pairs of them in pair mode), two
  // per item on a CTA pair, the even CTA taking the first
  const int m_tiles = a.N / kTcBM / (a.pair ? 2 : 1) / kPairCtas;
  const int total = *a.chunk_count * m_tiles;
  const int first = CG2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int stride = CG2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int ksteps = a.K / kTcBK;
  const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
  const LayerHdr LS = OUT ? hdr_view_side(a.packed, a.E, a.H, a.F) : L;  // with the side-list table
  bool ok = true;

  // Every role runs its loop with whole warps: waits are taken by all lanes and
  // made warp-uniform, and only lane 0 issues TMA / MMA / commit, so no warp
  // reaches the final block barrier diverged.
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort_flag, a.wait)) != 0;
  };

  if (warp == kRawWarp) {
    // ---------------------------------------------------------- packed codes + scales
    int rs = 0, g = 0;
    uint32_t rph = 0;
    uint32_t issued = 0, issued_phase = 0;  // per raw slot: a load was armed, and its parity
    for (int t = first; t < total && ok; t += stride) {
      const int c = t / m_tiles, mt = (t % m_tiles) * kPairCtas + (int)rank;
      const int e = a.chunks[3 * c];
      // A weight tile's codes (and scales) are contiguous along K, so each stage's
      // slice is the tile base plus ks times a fixed stride.
      const uint8_t* cptr[NMAT];
      const uint8_t* sptr[NMAT];
      uint32_t cbytes[NMAT];
      uint32_t bytes = 0;
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const int i = e * 3 + a.proj + (a.pair ? 0 : m);
        const int mtm = a.pair ? 2 * mt + m : mt;
        const int f = L.fmt[i];
        cbytes[m] = (uint32_t)(fmt_words(f) * 512 * kGroups);
        cptr[m] = L.base + L.code_off[i] + code_stage_offset(mtm, 0, a.K, fmt_words(f));
        sptr[m] = L.base + L.scale_off[i] + scale_stage_offset(mtm, 0, a.K, f);
        bytes += cbytes[m] + (uint32_t)C::kScaleBytes;
      }
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&B.raw_empty[rs], rph ^ 1u)) {
          ok = false;
          break;
        }
        if (lane == 0 && !a.withhold) {
          trace_stamp(a.trace, 0, g);
          uint8_t* rb = smem + R.off_raw + rs * R.raw_bytes;
          ptx::mbar_arrive_expect_tx(&B.raw_full[rs], bytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            ptx::bulk_load(rb + m * R.code_bytes, cptr[m] + (size_t)ks * cbytes[m], cbytes[m], &B.raw_full[rs]);
            ptx::bulk_load(rb + NMAT * R.code_bytes + m * C::kScaleBytes, sptr[m] + (size_t)ks * C::kScaleBytes,
                           (uint32_t)C::kScaleBytes, &B.raw_full[rs]);
          }
          trace_stamp(a.trace, 1, g);
        }
        ++g;
        __syncwarp();
        if (!a.withhold) {
          issued |= 1u << rs;
          issued_phase = (issued_phase & ~(1u << rs)) | (rph << rs);
        }
        if (++rs == R.raw_slots) {
          rs = 0;
          rph ^= 1u;
        }
      }
    }
    // never leave while a copy may still be landing in shared memory
    for (int s2 = 0; s2 < R.raw_slots; ++s2)
      if (issued & (1u << s2)) ptx::mbar_drain(&B.raw_full[s2], (issued_phase >> s2) & 1u, kWaitLimit / 4);
    __syncwarp();
  } else if (warp == kBWarp) {
    // ---------------------------------------------------------- activation tiles
    int bs = 0;
    uint32_t bph = 0;
    uint32_t issued = 0, issued_phase = 0;  // per B slot: a load was armed, and its parity
    for (int t = first; t < total && ok; t += stride) {
      const int c = t / m_tiles;
      // this CTA's token rows of the MMA's N = nmma columns: the first or second half
      const int nmma = min(kTcBN, (a.chunks[3 * c + 2] + 15) & ~15);
      const int row0 = a.chunks[3 * c + 1] + (int)rank * (nmma / 2);
      // a chunk whose rows fit half the tile loads a half-height box: the MMA reads
      // only the first rows of the slot, and the rest would be another chunk's rows
      const bool half = (CG2 ? nmma / 2 : nmma) <= C::kBRows / 2;
      const CUtensorMap* bmap = half ? &tmap_bh : &tmap_b;
      const uint32_t bbytes = half ? (uint32_t)C::kBBytes / 2u : (uint32_t)C::kBBytes;
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&B.b_empty[bs], bph ^ 1u)) {
          ok = false;
          break;
        }
        if (lane == 0 && !a.withhold) {
          ptx::mbar_arrive_expect_tx(&B.b_full[bs], bbytes);
          ptx::tma_load_2d(smem + R.off_b + bs * C::kBBytes, bmap, ks * kTcBK, row0, &B.b_full[bs]);
        }
        __syncwarp();
        if (!a.withhold) {
          issued |= 1u << bs;
          issued_phase = (issued_phase & ~(1u << bs)) | (bph << bs);
        }
        if (++bs == R.b_slots) {
          bs = 0;
          bph ^= 1u;
        }
      }
    }
    for (int s2 = 0; s2 < R.b_slots; ++s2)
      if (issued & (1u << s2)) ptx::mbar_drain(&B.b_full[s2], (issued_phase >> s2) & 1u, kWaitLimit / 4);
    __syncwarp();
  } else if (warp == kMmaWarp && rank != 0) {
    // ---------------------------------------------------------- odd CTA: report its activation tiles
    // The even CTA's MMAs read this CTA's half of every activation tile; once it has
    // landed, say so on the even CTA's barrier.
    int bs = 0;
    uint32_t bph = 0;
    for (int t = first; t < total && ok; t += stride)
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&B.b_full[bs], bph)) {
          ok = false;
          break;
        }
        if (lane == 0) ptx::mbar_arrive_cluster(&B.b_peer[bs], 0);
        __syncwarp();
        if (++bs == R.b_slots) {
          bs = 0;
          bph ^= 1u;
        }
      }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issue (even CTA)
    int as = 0, bs = 0, g = 0;
    uint32_t aph = 0, bph = 0, acc_phase = 0;
    // Shared-memory descriptors of slot 0, built once: a slot, a weight tile and a
    // K=16 step only add to the 14-bit start-address field (16-byte units; every
    // shared address here is below 256 KB, so the field never carries).
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint64_t dA0 = tile_desc(sbase), dB0 = tile_desc(sbase + (uint32_t)R.off_b);
    constexpr uint64_t kASlotStep = C::kASlotBytes >> 4, kBSlotStep = C::kBBytes >> 4;
    constexpr uint64_t kTileStep = C::kABytes >> 4, kKStep = 32 >> 4;
    bool committed = false;
    for (int t = first; t < total && ok; t += stride) {
      const int c = t / m_tiles;
      const int rows = a.chunks[3 * c + 2];
      const int nmma = min(kTcBN, (rows + 15) & ~15);
      const uint32_t idesc = ptx::idesc_f16_f32(kTcBM * kPairCtas, nmma);
      if (!wait_all(B.acc_empty, acc_phase ^ 1u)) {
        ok = false;
        break;
      }
      acc_phase ^= 1u;
      ptx::tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&B.a_full[as], aph) || !wait_all(&B.b_full[bs], bph) ||
            (CG2 && !wait_all(&B.b_peer[bs], bph))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (lane == 0) trace_stamp(a.trace, 4, g);
        {
          // the whole warp runs this with uniform operands; one elected lane issues
          const uint64_t da = dA0 + (uint64_t)as * kASlotStep, db = dB0 + (uint64_t)bs * kBSlotStep;
          const uint32_t acc0 = ks != 0;
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int k16 = 0; k16 < kTcBK / 16; ++k16) {
              const uint64_t ad = da + (uint64_t)m * kTileStep + (uint64_t)k16 * kKStep;
              const uint64_t bd = db + (uint64_t)k16 * kKStep;
              if (CG2)
                ptx::mma2_f16_ss_warp(tmem + (uint32_t)(m * 256), ad, bd, idesc, k16 ? 1u : acc0);
              else
                ptx::mma_f16_ss_warp(tmem + (uint32_t)(m * 256), ad, bd, idesc, k16 ? 1u : acc0);
            }
          if (CG2) {
            ptx::mma2_commit_mc_warp(&B.a_empty[as], 0x3);
            ptx::mma2_commit_mc_warp(&B.b_empty[bs], 0x3);
          } else {
            ptx::mma_commit_warp(&B.a_empty[as]);
            ptx::mma_commit_warp(&B.b_empty[bs]);
          }
          if (lane == 0) trace_stamp(a.trace, 5, g);
        }
        ++g;
        __syncwarp();
        committed = true;
        if (++as == R.a_slots) {
          as = 0;
          aph ^= 1u;
        }
        if (++bs == R.b_slots) {
          bs = 0;
          bph ^= 1u;
        }
      }
      if (!ok) break;
      if (CG2)
        ptx::mma2_commit_mc_warp(B.acc_full, 0x3);
      else
        ptx::mma_commit_warp(B.acc_full);
      __syncwarp();
    }
    if (committed) {  // the last commit lands once every MMA issued by this CTA has completed
      const int last = (bs + R.b_slots - 1) % R.b_slots;
      const uint32_t par = (bs == 0) ? (bph ^ 1u) : bph;
      ptx::mbar_drain(&B.b_empty[last], par, kWaitLimit / 4);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- dequant + epilogue
    // kThreadsPerRow threads per weight row n.  The row's units of a stage (chunk
    // of 8 inputs x matrix, matrices alternating) are split evenly: thread
    // sel = tid/128 takes kUnits consecutive units, as many of each matrix.
    const int n = threadIdx.x & 127, sel = threadIdx.x >> 7;
    constexpr int kColGroups = kDeqWarps / 4;            // epilogue column groups
    constexpr int kColsPerWarp = kTcBN / kColGroups;
    const int q = warp & 3, cq = warp >> 2;               // epilogue: TMEM lane quarter, column group
    constexpr int kUnits = NMAT * kGroups * 4 / kThreadsPerRow;
    const int u0 = sel * kUnits;
    Cursor cur{0, 0u, 0, 0u, 0};
    int item = 0;
    uint32_t acc_phase = 0;
    for (int t = first; t < total && ok; t += stride, ++item) {
      const int c = t / m_tiles, mt = (t % m_tiles) * kPairCtas + (int)rank;
      const int e = a.chunks[3 * c], row0 = a.chunks[3 * c + 1], rows = a.chunks[3 * c + 2];
      int fmt[NMAT];
      float tsc[NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const int i = e * 3 + a.proj + (a.pair ? 0 : m);
        fmt[m] = L.fmt[i];
        tsc[m] = fmt[m] == MOE_FMT_NVFP4 ? L.tscale[i] : 1.0f;
      }
      if (!dequant_item_any<NMAT, CG2, I1>(fmt[0], fmt[NMAT - 1], a.ring, a.wait, ptx::smem_u32(smem), bars,
                                           abort_flag, ksteps, n, u0, cur, a.trace)) {
        ok = false;
        break;
      }
      if (!ok) break;
      if (!wait_all(B.acc_full, acc_phase)) {
        ok = false;
        break;
      }
      acc_phase ^= 1u;
      if (threadIdx.x == 0) trace_stamp(a.trace, 6, item);
      ptx::tc_fence_after();
      const int nrow = (a.pair ? 2 * mt : mt) * kTcBM + q * 32 + lane;
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
      // the chunk's columns (tokens) split evenly over the kColGroups column groups, in
      // steps of 16, so that every epilogue warp has work when a chunk holds few rows
      const int cpw = ((rows + 16 * kColGroups - 1) / (16 * kColGroups)) * 16, c0 = cq * cpw;
      bool range = false;  // an fp16 SwiGLU output overflowed
      if (a.row_scale) {
        // NVFP4 layers: the row scales of the warp's (at most 64) tokens (gate/up: the
        // token's sx through perm; down: the row's sh), two per lane, loaded before any
        // store and broadcast with shuffles -- loaded inside the store loop, each would
        // wait for the stores before it.
        static_assert(kColsPerWarp == 64, "two token scales per lane");
        float fac[2] = {0.0f, 0.0f};
#pragma unroll
        for (int u2 = 0; u2 < 2; ++u2) {
          const int tok = c0 + 32 * u2 + lane;
          if (32 * u2 + lane < cpw && tok < rows) {
            const int r = row0 + tok;
            fac[u2] = (NMAT == 2 && !a.pair) ? a.row_scale[a.perm[r] / a.topk] : a.row_scale[r];
          }
        }
        float* __restrict__ out = reinterpret_cast<float*>(a.out);
        for (int cb = c0; cb < c0 + cpw && cb < rows; cb += 16) {
          uint32_t r0[16], r1[16];
          ptx::tmem_ld16(lane_base + (uint32_t)cb, r0);
          if (NMAT == 2) ptx::tmem_ld16(lane_base + 256u + (uint32_t)cb, r1);
          ptx::tmem_ld_wait();
          const float fu = ((cb - c0) >> 5) ? fac[1] : fac[0];  // warp-uniform choice
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = cb + j;
            const float f = __shfl_sync(0xffffffffu, fu, (tok - c0) & 31);
            if (tok >= rows) continue;
            const size_t o = (size_t)(row0 + tok) * a.N + nrow;
            if (OUT) {  // residuals of the side lists, in the units of the fp16 activations
              const __half* av = a.act16 + (size_t)(row0 + tok) * a.K;
              const int i0 = e * 3 + a.proj;
              float d0, d1 = 0.0f;
              if (NMAT == 2 && a.pair) {
                d0 = outlier_dot(LS, i0, a.N, nrow, av);
                d1 = outlier_dot(LS, i0, a.N, nrow + kTcBM, av);
                out[o] = (__uint_as_float(r0[j]) * tsc[0] + d0) * f;
                out[o + kTcBM] = (__uint_as_float(r1[j]) * tsc[0] + d1) * f;
              } else if (NMAT == 2) {
                d0 = outlier_dot(LS, i0, a.N, nrow, av);
                d1 = outlier_dot(LS, i0 + 1, a.N, nrow, av);
                const float g = (__uint_as_float(r0[j]) * tsc[0] + d0) * f, u = (__uint_as_float(r1[j]) * tsc[1] + d1) * f;
                out[o] = __fdividef(g, 1.0f + __expf(-g)) * u;
              } else {
                out[o] = (__uint_as_float(r0[j]) * tsc[0] + outlier_dot(LS, i0, a.N, nrow, av)) * f;
              }
            } else if (NMAT == 2 && a.pair) {  // two weight tiles of the down matrix: rows nrow and nrow + 128
              const float sc = f * tsc[0];
              out[o] = __uint_as_float(r0[j]) * sc;
              out[o + kTcBM] = __uint_as_float(r1[j]) * sc;
            } else if (NMAT == 2) {
              const float g = __uint_as_float(r0[j]) * (f * tsc[0]), u = __uint_as_float(r1[j]) * (f * tsc[1]);
              out[o] = __fdividef(g, 1.0f + __expf(-g)) * u;
            } else {
              out[o] = __uint_as_float(r0[j]) * (f * tsc[0]);
            }
          }
        }
      } else {
        // integer layers: SwiGLU into fp16 h (gate/up) or fp32 o (down)
        for (int cb = c0; cb < c0 + cpw && cb < rows; cb += 16) {
          uint32_t r0[16], r1[16];
          ptx::tmem_ld16(lane_base + (uint32_t)cb, r0);
          if (NMAT == 2) ptx::tmem_ld16(lane_base + 256u + (uint32_t)cb, r1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = cb + j;
            if (tok >= rows) break;
            const int r = row0 + tok;
            float d0 = 0.0f, d1 = 0.0f;  // residuals of the side lists, in the units of the fp16 activations
            if (OUT) {
              const __half* av = a.act16 + (size_t)r * a.K;
              const int i0 = e * 3 + a.proj;
              d0 = outlier_dot(LS, i0, a.N, nrow, av);
              if (NMAT == 2) d1 = a.pair ? outlier_dot(LS, i0, a.N, nrow + kTcBM, av) : outlier_dot(LS, i0 + 1, a.N, nrow, av);
            }
            if (NMAT == 2 && a.pair) {  // two weight tiles of the down matrix: rows nrow and nrow + 128
              reinterpret_cast<float*>(a.out)[(size_t)r * a.N + nrow] = __uint_as_float(r0[j]) + d0;
              reinterpret_cast<float*>(a.out)[(size_t)r * a.N + nrow + kTcBM] = __uint_as_float(r1[j]) + d1;
            } else if (NMAT == 2) {
              const float xi = a.xinv[r];  // 2^e: exact, 1 unless the token was prescaled
              const float g = (__uint_as_float(r0[j]) + d0) * xi, u = (__uint_as_float(r1[j]) + d1) * xi;
              const __half h = __float2half_rn(__fdividef(g, 1.0f + __expf(-g)) * u);
              range |= __hisinf(h) != 0;
              reinterpret_cast<__half*>(a.out)[(size_t)r * a.N + nrow] = h;
            } else {
              reinterpret_cast<float*>(a.out)[(size_t)r * a.N + nrow] = __uint_as_float(r0[j]) + d0;
            }
          }
        }
      }
      if (range && a.status) atomicCAS(a.status, 0, (int32_t)MOE_ERR_RANGE);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG2)
          ptx::mbar_arrive_cluster(B.acc_empty, 0);
        else
          ptx::mbar_arrive(B.acc_empty);
      }
      if (threadIdx.x == 0) trace_stamp(a.trace, 7, item);
    }
  }

  if (!ok) {
    *abort_flag = 1;
    if (CG2) ptx::st_cluster_u32(abort_flag, rank ^ 1u, 1);  // the peer's waits give up too
    if (a.status) atomicExch(a.status, (int32_t)MOE_ERR_TIMEOUT);
  }
  ptx::tc_fence_before();
  __syncthreads();
  // a pair leaves together: the even CTA's MMAs read the odd CTA's shared memory
  // and write its tensor memory, and the odd CTA arrives on the even one's barriers
  if (CG2) ptx::cluster_sync();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    if (CG2)
      ptx::tmem_dealloc2(tmem, 512);
    else
      ptx::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

int sm_count() {
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

template <int NMAT, bool CG2, bool I1, bool OUT>
cudaError_t launch_tc(TcArgs a, int max_words, const void* act, int rows_total, cudaStream_t stream) {
  using C = TcCfg<NMAT, CG2>;
  a.act16 = static_cast<const __half*>(act);
  a.ring = make_ring<NMAT, CG2>(max_words);
  if (a.ring.raw_slots < 2) return cudaErrorInvalidConfiguration;
  const int smem = ring_smem(a.ring);
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map, map_half;  // activation tiles of kBRows rows, and of kBRows / 2
  const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)rows_total};
  const cuuint64_t strides[1] = {(cuuint64_t)a.K * 2u};
  const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)C::kBRows};
  const cuuint32_t box_half[2] = {(cuuint32_t)kTcBK, (cuuint32_t)(C::kBRows / 2)};
  const CUtensorMapSwizzle swz = kRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const cuuint32_t estr[2] = {1u, 1u};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(act), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&map_half, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(act), dims, strides, box_half, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = expert_gemm_tc_kernel<NMAT, CG2, I1, OUT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  if (!CG2) {
    launch_chained(kern, dim3(sm_count()), dim3(kTcThreads), smem, stream, map, map_half, a);
    return cudaGetLastError();
  }
  // one persistent pair of CTAs per pair of SMs: as many clusters as can be
  // resident at once (a GPC with an odd number of free SMs leaves one idle)
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // chained like the other kernels
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
  int clusters = 0;
  err = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
  if (err != cudaSuccess) return err;
  if (clusters < 1) return cudaErrorInvalidConfiguration;
  cfg.gridDim = dim3((unsigned)(2 * min(clusters, sm_count() / 2)));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, map, map_half, a);
}

}  // namespace

cudaError_t launch_expert_gemm_tc(const uint8_t* packed, const uint8_t* fmt_host, int E, int H, int F, int T, int k,
                                  bool fp4, bool gateup, const Workspace& ws, int32_t* status, uint64_t* trace,
                                  GemmHooks hooks, bool outliers, cudaStream_t stream) {
  // widest code format of the projections this launch reads (sizes the code slots),
  // and whether any of them is the 1-bit code (selects the kernels that decode it)
  int max_words = 1;
  bool any1 = false;
  for (int e = 0; e < E; ++e)
    for (int p = gateup ? 0 : 2; p <= (gateup ? 1 : 2); ++p) {
      max_words = std::max(max_words, fmt_words(fmt_host[e * 3 + p]));
      any1 |= fmt_host[e * 3 + p] == MOE_FMT_INT1;
    }
  TcArgs a{};
  a.trace = gateup ? reinterpret_cast<unsigned long long*>(trace) : nullptr;
  a.wait = hooks.wait_cycles ? (long long)hooks.wait_cycles : kWaitLimit;
  a.withhold = hooks.withhold ? 1 : 0;
  a.packed = packed;
  a.E = E;
  a.H = H;
  a.F = F;
  a.chunks = ws.chunks;
  a.chunk_count = ws.chunk_count;
  a.perm = ws.perm;
  a.topk = k;
  a.status = status;
  const int R = T * k;
  // kernel variant: tile shape, 1-bit decoding, side lists
  auto go = [&](auto nmat, auto cg2, const void* act) -> cudaError_t {
    constexpr int NM = decltype(nmat)::value;
    constexpr bool P = decltype(cg2)::value;
    if (outliers)
      return any1 ? launch_tc<NM, P, true, true>(a, max_words, act, R, stream)
                  : launch_tc<NM, P, false, true>(a, max_words, act, R, stream);
    return any1 ? launch_tc<NM, P, true, false>(a, max_words, act, R, stream)
                : launch_tc<NM, P, false, false>(a, max_words, act, R, stream);
  };
  using Two = std::integral_constant<int, 2>;
  using One = std::integral_constant<int, 1>;
  using Pair = std::true_type;
  using Single = std::false_type;
  if (gateup) {
    a.N = F;
    a.K = H;
    a.proj = 0;
    a.row_scale = fp4 ? ws.sx : nullptr;
    a.xinv = fp4 ? nullptr : ws.xinv;
    a.out = ws.h;
    if ((F / kTcBM) % 2 == 0) return go(Two{}, Pair{}, ws.xs);  // weight tiles in pairs of CTAs
    return go(Two{}, Single{}, ws.xs);
  }
  a.N = H;
  a.K = F;
  a.proj = 2;
  a.row_scale = fp4 ? ws.sh : nullptr;
  a.out = ws.o;
  const void* act = fp4 ? ws.hb : ws.h;
  if ((H / kTcBM) % 2 == 0) {  // pairs of weight tiles share each activation tile
    a.pair = 1;
    if ((H / kTcBM) % 4 == 0) return go(Two{}, Pair{}, act);
    return go(Two{}, Single{}, act);
  }
  return go(One{}, Single{}, act);
}

}  // namespace moe

// Dequant-fused grouped expert GEMV for batches with few token rows per expert
// (decode: 1-16 rows), bound by streaming the active experts' packed weights
// from HBM (the pages' observation that only the active experts' weights are
// read, and the packed-linear operator of the MoE mixed-precision page, sec.
// 2.3 / 3.5).
//
// Work item: (chunk of <= 16 expert-sorted rows of one expert, 32 weight rows).
// A persistent CTA of kWarps warps walks its work items; every warp owns a
// fixed 1/kWarps of the inputs of each item (split-K inside the CTA, summed
// through shared memory when the item ends).  Per group of 32 inputs a thread
// (g = lane/4, c = lane%4) needs word c of four consecutive weight rows of each
// matrix, their scales and eight activations per token tile; it copies them
// with cp.async straight into its own slots of a shared-memory ring that runs
// kStages groups ahead, across item boundaries, so each SM keeps well over
// 100 KB of weight loads in flight without spending registers on them.
//
// Compute per group: the codes 8c..8c+7 of a row become four fp16 pairs
// (exponent-bias unpack: code u OR'ed into the mantissa of 1024.0 gives 1024+u
// exactly, minus 1024+offset exactly) that are the A fragments of two
// mma.sync m16n8k16 per 16-row tile.  The input order inside an MMA is permuted
// consistently for both operands: thread c supplies inputs 8c..8c+7 of the
// group for A and the same eight activations for B.  Integer groups are scaled
// after their MMAs (one fp32 FMA per output); NVFP4 codes are multiplied by
// their e4m3 block scale before (exact in fp16).
#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kRowsPerCta = 32;
constexpr int kWarps = 4;          // K-split warps per CTA
constexpr int kTokMax = 16;        // token rows per chunk
constexpr int kStages = 4;         // ring stages per warp (kStages-1 groups in flight)
constexpr int kPartStride = kTokMax + 1;

__device__ __forceinline__ uint32_t h2sub_u(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2mul_u(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ void e2m1x8_to_f16_v(uint32_t w, uint32_t* o) {
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

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
// 16-byte copy that reads src_bytes (0 or 16) and zero-fills the rest.
__device__ __forceinline__ void cp16z(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct GemvArgs {
  const uint8_t* packed;
  int E, H, F;
  int N, K;
  int proj;                 // 0: gate+up (SwiGLU), 2: down
  const __half* act;        // [rows][K] fp16 activations, sorted rows
  const int32_t* chunks;
  const int32_t* chunk_count;
  const float* row_scale;   // NVFP4 only (sx per token for gate/up, sh per row for down)
  const int32_t* perm;
  int topk;
  void* out;
};

// Where one work item's data lives; shared by the copy and compute sides.
struct ItemView {
  int e, row0, rows, slice;
  int f0, f1;
  const uint32_t* codes0;
  const uint8_t* scales0;
  const uint32_t* codes1;
  const uint8_t* scales1;
};

template <int NMAT>
__device__ __forceinline__ ItemView item_view(const GemvArgs& a, int item, int slices) {
  ItemView v;
  const int chunk = item / slices;
  v.slice = item % slices;
  v.e = a.chunks[3 * chunk];
  v.row0 = a.chunks[3 * chunk + 1];
  v.rows = a.chunks[3 * chunk + 2];
  const uint8_t* fmt = a.packed + kOffFmt;
  const uint64_t* co = reinterpret_cast<const uint64_t*>(a.packed + kOffCode);
  const uint64_t* so = reinterpret_cast<const uint64_t*>(a.packed + kOffScale);
  const int i0 = v.e * 3 + a.proj, i1 = i0 + NMAT - 1;
  v.f0 = fmt[i0];
  v.f1 = fmt[i1];
  v.codes0 = reinterpret_cast<const uint32_t*>(a.packed + co[i0]);
  v.scales0 = a.packed + so[i0];
  v.codes1 = reinterpret_cast<const uint32_t*>(a.packed + co[i1]);
  v.scales1 = a.packed + so[i1];
  return v;
}

// Slot layout of one group (16-byte slots, [slot][lane] so 128-bit shared
// accesses are conflict-free): 2m, 2m+1 words of matrix m (the second: 3-bit
// high bits), 2*NMAT scales (matrix 0 in .xy, matrix 1 in .zw), 2*NMAT+1+nt
// activations of token tile nt.
template <int NMAT, int NT8>
struct Slots {
  static constexpr int kItems = 2 * NMAT + 1 + NT8;
  static constexpr int kScale = 2 * NMAT;
  static constexpr int kAct = 2 * NMAT + 1;
};
template <int NMAT, int NT8>
__device__ __forceinline__ uint4* slot_ptr(uint4* ring, int stage, int slot, int lane) {
  return ring + (stage * Slots<NMAT, NT8>::kItems + slot) * 32 + lane;
}

// Copy side.  A cursor walks this warp's stream of (item, group) elements; its
// per-thread source pointers advance by a fixed stride per group and are
// recomputed only when the stream moves to the next work item.
template <int NMAT, int NT8>
struct Cursor {
  int j, g, n_items, g0, g1, slices;
  int fm[NMAT];
  const uint32_t* cw[NMAT];   // word (4-bit / NVFP4: word c; 2-, 3-bit: low word c/2) of the thread's 4 rows
  const uint32_t* ch[NMAT];   // 3-bit: high-bit word
  const uint8_t* cs[NMAT];    // scales of the thread's 4 rows
  int wstride[NMAT];          // words per group
  const __half* cx[NT8];      // 8 activations of token gl (+8)
  uint32_t xbytes[NT8];       // 16, or 0 beyond the chunk (zero fill)
};

template <int NMAT, int NT8>
__device__ __forceinline__ void cursor_item(Cursor<NMAT, NT8>& cu, const GemvArgs& a, int lane) {
  const ItemView v = item_view<NMAT>(a, blockIdx.x + cu.j * gridDim.x, cu.slices);
  const int gl = lane >> 2, c = lane & 3;
  const int nb4 = v.slice * kRowsPerCta + 4 * gl;
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    const int f = m == 0 ? v.f0 : v.f1;
    const uint32_t* codes = m == 0 ? v.codes0 : v.codes1;
    const uint8_t* scales = m == 0 ? v.scales0 : v.scales1;
    const int wpg = fmt_words(f);
    const int wsel = (f == MOE_FMT_INT4 || f == MOE_FMT_NVFP4) ? c : (c >> 1);
    cu.fm[m] = f;
    cu.wstride[m] = wpg * 128;
    cu.cw[m] = codes + word_index(nb4, cu.g0 * 32, a.K, wpg, wsel);
    cu.ch[m] = codes + word_index(nb4, cu.g0 * 32, a.K, wpg, 2);
    cu.cs[m] = f == MOE_FMT_NVFP4 ? scales + scale_index(nb4, 2 * cu.g0 + (c >> 1), a.K / 16)
                                  : scales + 2 * scale_index(nb4, cu.g0, a.K / 32);
  }
#pragma unroll
  for (int nt = 0; nt < NT8; ++nt) {
    const int tok = nt * 8 + gl;
    const bool ok = tok < v.rows;
    cu.cx[nt] = a.act + (size_t)(v.row0 + (ok ? tok : 0)) * a.K + cu.g0 * 32 + 8 * c;
    cu.xbytes[nt] = ok ? 16u : 0u;
  }
}

// Issue the cursor's element into ring stage `stage` and advance the cursor.
template <int NMAT, int NT8>
__device__ __forceinline__ void cursor_issue(Cursor<NMAT, NT8>& cu, const GemvArgs& a, uint4* ring, int stage,
                                             int lane) {
  if (cu.j >= cu.n_items) return;
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    cp16(slot_ptr<NMAT, NT8>(ring, stage, 2 * m, lane), cu.cw[m]);
    if (cu.fm[m] == MOE_FMT_INT3) cp16(slot_ptr<NMAT, NT8>(ring, stage, 2 * m + 1, lane), cu.ch[m]);
    uint8_t* sdst = reinterpret_cast<uint8_t*>(slot_ptr<NMAT, NT8>(ring, stage, Slots<NMAT, NT8>::kScale, lane)) + 8 * m;
    if (cu.fm[m] == MOE_FMT_NVFP4) cp4(sdst, cu.cs[m]);
    else cp8(sdst, cu.cs[m]);
    cu.cw[m] += cu.wstride[m];
    cu.ch[m] += cu.wstride[m];
    cu.cs[m] += 256;  // 128 fp16 scales, or 2 x 128 e4m3 block scales, per group
  }
#pragma unroll
  for (int nt = 0; nt < NT8; ++nt) {
    cp16z(slot_ptr<NMAT, NT8>(ring, stage, Slots<NMAT, NT8>::kAct + nt, lane), cu.cx[nt], cu.xbytes[nt]);
    cu.cx[nt] += 32;
  }
  if (++cu.g == cu.g1) {
    cu.g = cu.g0;
    if (++cu.j < cu.n_items) cursor_item(cu, a, lane);
  }
}

__device__ __forceinline__ uint32_t h2fma_u(uint32_t a, uint32_t b, uint32_t c) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b), *reinterpret_cast<__half2*>(&c));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t c) { return (a & mask) | c; }

// fp16 pair constants (both halves equal)
constexpr uint32_t kMagic = 0x64006400u;  // 1024.0
__host__ __device__ constexpr uint32_t h2c(uint32_t h) { return h | (h << 16); }

// The four fp16 pairs (inputs 8c..8c+7 of the group) of row i (0..3) of the
// thread, as the signed code q = u - offset (NVFP4: e2m1 value times block scale).
// Unpack: masking bits [b, b+w) of both half-words and OR'ing 1024.0 gives
// 1024 + 2^b * u exactly (b + w <= 10); one FMA with 2^-b and -(1024/2^b + offset)
// then gives u - offset exactly (the exact result is representable).
template <int FMT>
__device__ __forceinline__ void unpack_row(uint4 w0, uint4 w1, uint32_t sc, int i, int c, uint32_t* p) {
  const uint32_t w = i == 0 ? w0.x : i == 1 ? w0.y : i == 2 ? w0.z : w0.w;
  if (FMT == MOE_FMT_NVFP4) {
    e2m1x8_to_f16_v(w, p);
    const __half2 s2 = __float2half2_rn(e4m3_value((sc >> (8 * i)) & 255u));
    const uint32_t sp = *reinterpret_cast<const uint32_t*>(&s2);
#pragma unroll
    for (int j = 0; j < 4; ++j) p[j] = h2mul_u(p[j], sp);  // exact: <= 6 significant bits
  } else if (FMT == MOE_FMT_INT4) {
    // pairs 0,1 at bits 0-3 / 4-7; pairs 2,3 at bits 8-11 / 12-15 (after >> 8)
    const uint32_t w8 = w >> 8;
    p[0] = h2fma_u(lop_or(w, 0x000F000Fu, kMagic), h2c(0x3C00u), h2c(0xE408u));    // x*1 - 1032
    p[1] = h2fma_u(lop_or(w, 0x00F000F0u, kMagic), h2c(0x2C00u), h2c(0xD480u));    // x/16 - 72
    p[2] = h2fma_u(lop_or(w8, 0x000F000Fu, kMagic), h2c(0x3C00u), h2c(0xE408u));
    p[3] = h2fma_u(lop_or(w8, 0x00F000F0u, kMagic), h2c(0x2C00u), h2c(0xD480u));
  } else if (FMT == MOE_FMT_INT2) {
    const uint32_t ws = w >> (8 * (c & 1));  // the 4 pairs of inputs 8c..8c+7 at bits 0-7 / 16-23
    p[0] = h2fma_u(lop_or(ws, 0x00030003u, kMagic), h2c(0x3C00u), h2c(0xE402u));   // x - 1026
    p[1] = h2fma_u(lop_or(ws, 0x000C000Cu, kMagic), h2c(0x3400u), h2c(0xDC08u));   // x/4 - 258
    p[2] = h2fma_u(lop_or(ws, 0x00300030u, kMagic), h2c(0x2C00u), h2c(0xD420u));   // x/16 - 66
    p[3] = h2fma_u(lop_or(ws, 0x00C000C0u, kMagic), h2c(0x2400u), h2c(0xCC80u));   // x/64 - 18
  } else {  // INT3: low bits as INT2; bit 2 of pair J at bits J and 16+J of the high word
    const uint32_t lo = w >> (8 * (c & 1));
    const uint32_t hw = i == 0 ? w1.x : i == 1 ? w1.y : i == 2 ? w1.z : w1.w;
    const uint32_t hi = hw >> (4 * c);  // pair j's high bits at bits j, 16+j
    // pair j's 3-bit code at bits [2j, 2j+3): low bits from lo, high bit = (hi << (j+2)) at 2j+2
    p[0] = h2fma_u((lop_or(lo, 0x00030003u, kMagic) | ((hi << 2) & 0x00040004u)), h2c(0x3C00u), h2c(0xE404u));  // - 1028
    p[1] = h2fma_u((lop_or(lo, 0x000C000Cu, kMagic) | ((hi << 3) & 0x00100010u)), h2c(0x3400u), h2c(0xDC10u));  // /4 - 260
    p[2] = h2fma_u((lop_or(lo, 0x00300030u, kMagic) | ((hi << 4) & 0x00400040u)), h2c(0x2C00u), h2c(0xD440u));  // /16 - 68
    p[3] = h2fma_u((lop_or(lo, 0x00C000C0u, kMagic) | ((hi << 5) & 0x01000100u)), h2c(0x2400u), h2c(0xCD00u));  // /64 - 20
  }
}

__device__ __forceinline__ float half_at(uint32_t lohi, int hi) {
  return __half2float(__ushort_as_half((uint16_t)(hi ? (lohi >> 16) : (lohi & 0xFFFFu))));
}

// Compute side for one group held in ring stage `stage`; formats F0/F1 known at
// compile time.  acc[m][t][nt][4]: matrix m, 16-row tile t (rows 2t, 2t+1 of the
// thread's four), token tile nt, mma accumulator element.
template <int NMAT, int F0, int F1, int NT8>
__device__ __forceinline__ void compute_group(uint4* ring, int stage, int lane, float (&acc)[NMAT][2][NT8][4]) {
  const int c = lane & 3;
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
  const uint4 sc = *slot_ptr<NMAT, NT8>(ring, stage, Slots<NMAT, NT8>::kScale, lane);
  uint4 x[NT8];
#pragma unroll
  for (int nt = 0; nt < NT8; ++nt) x[nt] = *slot_ptr<NMAT, NT8>(ring, stage, Slots<NMAT, NT8>::kAct + nt, lane);
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    constexpr int kF[2] = {F0, F1};
    const int FMT = kF[m];
    const uint4 w0 = *slot_ptr<NMAT, NT8>(ring, stage, 2 * m, lane);
    const uint4 w1 = FMT == MOE_FMT_INT3 ? *slot_ptr<NMAT, NT8>(ring, stage, 2 * m + 1, lane) : make_uint4(0, 0, 0, 0);
    const uint32_t s_lo = m == 0 ? sc.x : sc.z, s_hi = m == 0 ? sc.y : sc.w;  // 4 fp16 scales or 4 e4m3 bytes in s_lo
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      uint32_t pa[4], pb[4];  // rows 2t (MMA row g) and 2t+1 (MMA row g+8)
      if (m == 0) {
        unpack_row<F0>(w0, w1, s_lo, 2 * t, c, pa);
        unpack_row<F0>(w0, w1, s_lo, 2 * t + 1, c, pb);
      } else {
        unpack_row<F1>(w0, w1, s_lo, 2 * t, c, pa);
        unpack_row<F1>(w0, w1, s_lo, 2 * t + 1, c, pb);
      }
      const uint32_t A1[4] = {pa[0], pb[0], pa[1], pb[1]};
      const uint32_t A2[4] = {pa[2], pb[2], pa[3], pb[3]};
#pragma unroll
      for (int nt = 0; nt < NT8; ++nt) {
        if (FMT == MOE_FMT_NVFP4) {  // codes already carry their block scale: accumulate directly
          mma16816(acc[m][t][nt], A1, x[nt].x, x[nt].y, acc[m][t][nt]);
          mma16816(acc[m][t][nt], A2, x[nt].z, x[nt].w, acc[m][t][nt]);
        } else {  // the group's raw sum, then one fp32 FMA per output with the row's scale
          float d[4];
          mma16816(d, A1, x[nt].x, x[nt].y, zero4);
          mma16816(d, A2, x[nt].z, x[nt].w, d);
          const uint32_t sw = t == 0 ? s_lo : s_hi;  // rows 2t, 2t+1 -> halves of one scale word
          const float sa = half_at(sw, 0), sb = half_at(sw, 1);
          acc[m][t][nt][0] = fmaf(sa, d[0], acc[m][t][nt][0]);
          acc[m][t][nt][1] = fmaf(sa, d[1], acc[m][t][nt][1]);
          acc[m][t][nt][2] = fmaf(sb, d[2], acc[m][t][nt][2]);
          acc[m][t][nt][3] = fmaf(sb, d[3], acc[m][t][nt][3]);
        }
      }
    }
  }
}

// Consume the ng groups of one item from the ring (formats F0/F1), keeping the
// ring kStages-1 groups ahead: each consumed group frees its stage, which is
// refilled with stream element s+kStages-1 (possibly of a later item).  The
// warp's partial sums go to shared memory at the end.
template <int NMAT, int F0, int F1, int NT8>
__device__ __forceinline__ void consume_item(const GemvArgs& a, uint4* ring, float* part, int ng, int& s,
                                          Cursor<NMAT, NT8>& cu, int warp, int lane) {
  float acc[NMAT][2][NT8][4];
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[m][t][nt][j] = 0.0f;
  for (int i = 0; i < ng; ++i) {
    cp_wait<kStages - 2>();  // this element has landed (the thread's own copies)
    compute_group<NMAT, F0, F1, NT8>(ring, s, lane, acc);
    // refill the stage consumed one element ago with the element kStages-1 ahead
    cursor_issue(cu, a, ring, s == 0 ? kStages - 1 : s - 1, lane);
    cp_commit();  // one (possibly empty) group per element keeps the wait count fixed
    if (++s == kStages) s = 0;
  }
  const int gl = lane >> 2, c = lane & 3;
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          part[((warp * NMAT + m) * kRowsPerCta + 4 * gl + 2 * t + (j >> 1)) * kPartStride + nt * 8 + 2 * c + (j & 1)] =
              acc[m][t][nt][j];
}

template <int NMAT, int F0, int NT8>
__device__ __forceinline__ void consume_f1(int f1, const GemvArgs& a, uint4* ring, float* part, int ng, int& s,
                                           Cursor<NMAT, NT8>& cu, int warp, int lane) {
  if (NMAT == 1) return consume_item<NMAT, F0, F0, NT8>(a, ring, part, ng, s, cu, warp, lane);
  switch (f1) {
    case MOE_FMT_INT2: return consume_item<NMAT, F0, MOE_FMT_INT2, NT8>(a, ring, part, ng, s, cu, warp, lane);
    case MOE_FMT_INT3: return consume_item<NMAT, F0, MOE_FMT_INT3, NT8>(a, ring, part, ng, s, cu, warp, lane);
    case MOE_FMT_INT4: return consume_item<NMAT, F0, MOE_FMT_INT4, NT8>(a, ring, part, ng, s, cu, warp, lane);
    default: return consume_item<NMAT, F0, MOE_FMT_NVFP4, NT8>(a, ring, part, ng, s, cu, warp, lane);
  }
}

template <int NMAT, int NT8>
__global__ void __launch_bounds__(32 * kWarps) expert_gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int kItems = Slots<NMAT, NT8>::kItems;
  uint4* ring_all = reinterpret_cast<uint4*>(smem_raw);                                // [kWarps][kStages][kItems][32]
  float* part = reinterpret_cast<float*>(ring_all + kWarps * kStages * kItems * 32);  // [kWarps][NMAT][32][17]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* ring = ring_all + warp * kStages * kItems * 32;

  const int slices = a.N / kRowsPerCta;
  const int total = *a.chunk_count * slices;
  const int n_items = total > (int)blockIdx.x ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const int G = a.K / 32;
  const int g0 = (G * warp) / kWarps, g1 = (G * (warp + 1)) / kWarps, ng = g1 - g0;
  // this warp's stream: (item, group) elements in item order, issued kStages-1 ahead
  Cursor<NMAT, NT8> cu;
  cu.j = 0;
  cu.g = g0;
  cu.n_items = n_items;
  cu.g0 = g0;
  cu.g1 = g1;
  cu.slices = slices;
  if (n_items > 0) cursor_item(cu, a, lane);
  for (int st = 0; st < kStages - 1; ++st) {
    cursor_issue(cu, a, ring, st, lane);
    cp_commit();
  }

  int s = 0;  // ring stage of the next element to consume
  for (int j = 0; j < n_items; ++j) {
    const ItemView v = item_view<NMAT>(a, blockIdx.x + j * gridDim.x, slices);
    switch (v.f0) {
      case MOE_FMT_INT2: consume_f1<NMAT, MOE_FMT_INT2, NT8>(v.f1, a, ring, part, ng, s, cu, warp, lane); break;
      case MOE_FMT_INT3: consume_f1<NMAT, MOE_FMT_INT3, NT8>(v.f1, a, ring, part, ng, s, cu, warp, lane); break;
      case MOE_FMT_INT4: consume_f1<NMAT, MOE_FMT_INT4, NT8>(v.f1, a, ring, part, ng, s, cu, warp, lane); break;
      default: consume_f1<NMAT, MOE_FMT_NVFP4, NT8>(v.f1, a, ring, part, ng, s, cu, warp, lane); break;
    }
    __syncthreads();
    // reduce the K-split partials and run the epilogue of this item
    const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
    const float ts0 = v.f0 == MOE_FMT_NVFP4 ? L.tscale[v.e * 3 + a.proj] : 1.0f;
    const float ts1 = v.f1 == MOE_FMT_NVFP4 ? L.tscale[v.e * 3 + a.proj + NMAT - 1] : 1.0f;
    for (int idx = threadIdx.x; idx < kRowsPerCta * NT8 * 8; idx += blockDim.x) {
      const int rl = idx % kRowsPerCta, tok = idx / kRowsPerCta;
      if (tok >= v.rows) continue;
      const int n = v.slice * kRowsPerCta + rl, r = v.row0 + tok;
      float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        s0 += part[((w * NMAT + 0) * kRowsPerCta + rl) * kPartStride + tok];
        if (NMAT == 2) s1 += part[((w * NMAT + NMAT - 1) * kRowsPerCta + rl) * kPartStride + tok];
      }
      if (NMAT == 2) {
        if (a.row_scale) {
          const float sx = a.row_scale[a.perm[r] / a.topk];
          s0 *= sx * ts0;
          s1 *= sx * ts1;
          reinterpret_cast<float*>(a.out)[(size_t)r * a.N + n] = s0 / (1.0f + __expf(-s0)) * s1;
        } else {
          reinterpret_cast<__half*>(a.out)[(size_t)r * a.N + n] = __float2half_rn(s0 / (1.0f + __expf(-s0)) * s1);
        }
      } else {
        if (a.row_scale) s0 *= a.row_scale[r] * ts0;
        reinterpret_cast<float*>(a.out)[(size_t)r * a.N + n] = s0;
      }
    }
    __syncthreads();
  }
  cp_wait<0>();  // no copy may still be landing when the CTA exits
}

template <int NMAT, int NT8>
constexpr size_t smem_bytes() {
  return (size_t)kWarps * kStages * Slots<NMAT, NT8>::kItems * 32 * 16 +
         (size_t)kWarps * NMAT * kRowsPerCta * kPartStride * 4;
}

int sm_count_gemv() {
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

template <int NMAT, int NT8>
cudaError_t launch_n(const GemvArgs& g, int max_chunks, cudaStream_t stream) {
  auto kern = expert_gemv_kernel<NMAT, NT8>;
  constexpr size_t kSmemBytes = smem_bytes<NMAT, NT8>();
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kWarps, kSmemBytes);
  if (err != cudaSuccess) return err;
  const long long items = (long long)max_chunks * (g.N / kRowsPerCta);
  long long grid = (long long)sm_count_gemv() * (per_sm > 0 ? per_sm : 1);
  if (grid > items) grid = items;
  kern<<<(unsigned)grid, 32 * kWarps, kSmemBytes, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expert_gemv(const uint8_t* packed, int E, int H, int F, int k, bool fp4, bool gateup,
                               int max_chunks, int chunk_rows, const Workspace& ws, cudaStream_t stream) {
  GemvArgs g{};
  g.packed = packed;
  g.E = E;
  g.H = H;
  g.F = F;
  g.chunks = ws.chunks;
  g.chunk_count = ws.chunk_count;
  g.perm = ws.perm;
  g.topk = k;
  const bool two = chunk_rows > 8;
  if (gateup) {
    g.N = F;
    g.K = H;
    g.proj = 0;
    g.act = reinterpret_cast<const __half*>(ws.xs);
    g.row_scale = fp4 ? ws.sx : nullptr;
    g.out = ws.h;
    return two ? launch_n<2, 2>(g, max_chunks, stream) : launch_n<2, 1>(g, max_chunks, stream);
  }
  g.N = H;
  g.K = F;
  g.proj = 2;
  g.act = reinterpret_cast<const __half*>(fp4 ? ws.hb : ws.h);
  g.row_scale = fp4 ? ws.sh : nullptr;
  g.out = ws.o;
  return two ? launch_n<1, 2>(g, max_chunks, stream) : launch_n<1, 1>(g, max_chunks, stream);
}

}  // namespace moe

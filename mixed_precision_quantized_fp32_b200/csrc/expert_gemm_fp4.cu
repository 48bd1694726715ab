// Native block-scaled FP4 grouped expert GEMM for NVFP4 layers with NVFP4
// activations (moe_weights.act = MOE_ACT_NVFP4), prefill batches: both operands
// stay as e2m1 codes with e4m3 scales per 16 inputs, and the 5th-generation
// tensor cores form the block-scaled products directly
// (tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X, fp32 accumulators in
// TMEM).  The per-row activation scale and the weights' per-matrix tensor scale
// multiply the sums in the epilogue ("quantized MoE LLM inference", NVFP4
// remarks; the packed-linear operator of the MoE mixed-precision page).
//
// One CTA per SM walks (chunk of <= 128 expert-sorted token rows, weight tiles)
// work items: gate/up items hold the gate and up tiles of the same 128 rows
// (SwiGLU epilogue), down items two adjacent 128-row tiles of the down matrix
// sharing each activation tile.  A stage covers 256 inputs:
//   * warp 8 (one lane) loads, into one ring slot, the two matrices' packed codes
//     (two 128-input tiles each) and e4m3 block scales with 1D bulk copies, the
//     chunk's activation codes with a 2D TMA load (128-byte swizzle) and their
//     block scales with a 2D TMA load; nothing is multicast;
//   * warps 0-7 rearrange the packed weight codes in place into K-major rows
//     of 128 bytes (the swizzled layout the MMA reads; the packed layout stores a
//     group's four words 512 bytes apart) and both operands' block scales into
//     the 512-byte atoms tcgen05.cp moves to TMEM (row r of 128 at byte
//     16*(r%32) + 4*(r/32), four scales per row per MMA);
//   * warp 9 (one elected lane) copies the scale atoms to TMEM and issues per
//     matrix four MMAs of M=128 x N<=128 x K=64, then commits the slot;
//   * warps 0-7 drain the accumulators into the epilogue.
// Every wait is bounded; a wait that gives up raises the abort flag and writes
// MOE_ERR_TIMEOUT to the status word; copies and MMAs still in flight are waited
// for before TMEM is freed.
#include <algorithm>
#include <cudaTypedefs.h>

#include "moe_common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kF4Threads = 320;                // warps 0-7 transform + epilogue, 8 loads, 9 MMAs
constexpr int kF4LoadWarp = 8, kF4MmaWarp = 9;
constexpr int kF4BM = 128;                     // weight rows per tile (MMA M)
constexpr int kF4BN = kFp4ChunkRows;           // token rows per item (max MMA N)
constexpr int kF4BK = 256;                     // inputs per stage (128 bytes of codes per row)
constexpr long long kF4WaitLimit = 4000000000LL;
// one ring slot
constexpr int kF4OffA = 0;                     // 2 matrices x 16 KB: packed codes, rearranged in place
constexpr int kF4OffSfaRaw = 32768;            // 2 x 2 KB: packed e4m3 scales [16 blocks][128 rows]
constexpr int kF4OffB = 36864;                 // 128 rows x 128 bytes, 128-byte swizzle (TMA)
constexpr int kF4OffSfbRaw = 53248;            // 128 rows x 16 bytes (TMA)
constexpr int kF4OffSfa = 55296;               // 2 matrices x 4 MMAs x 512-byte scale atoms
constexpr int kF4OffSfb = 59392;               // 4 MMAs x 512-byte scale atoms
constexpr int kF4SlotBytes = 61440;
constexpr int kF4Slots = 3;
constexpr int kF4Smem = kF4Slots * kF4SlotBytes + 256 + 1024;
// tensor memory: accumulator of matrix m at columns m*128; scale factors of a stage
// after them (matrix m's A scales at 256 + 16m + 4j for MMA j, B scales at 288 + 4j)
constexpr uint32_t kF4TmemSfa = 256, kF4TmemSfb = 288;

struct F4Args {
  const uint8_t* packed;
  int E, H, F;
  int N, K;                 // weight rows and inputs of this GEMM
  int proj;                 // 0: gate+up with the SwiGLU epilogue; 2: down (two tiles per item)
  const int32_t* chunks;
  const int32_t* chunk_count;
  const float* row_scale;   // gate/up: per-token sx (via perm); down: per-row sh
  const int32_t* perm;
  int topk;
  float* out;               // gate/up: h [rows][F]; down: o [rows][H]
  int32_t* status;
  unsigned long long* trace;  // diagnostics: clock64 stamps of CTA 0 (or null)
  long long wait;
  int withhold;
};

// Stamp event `ev` of index `i` (CTA 0 only, first MOE_TRACE_STAGES indices).
__device__ __forceinline__ void f4_trace(unsigned long long* tr, int ev, int i) {
  if (tr && blockIdx.x == 0 && i < MOE_TRACE_STAGES) tr[ev * MOE_TRACE_STAGES + i] = (unsigned long long)clock64();
}

__device__ __forceinline__ int swz128(int row, int chunk) {
  return (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
}

// Warp-wide forms (one elected lane issues; operands are warp-uniform).
__device__ __forceinline__ void sf_copy_warp(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}
__device__ __forceinline__ void mma_fp4_warp(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                             uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}
// Shared-memory descriptor of a 512-byte scale atom (K-major, no swizzle: core
// matrices of 8 rows x 16 bytes, 128 bytes apart).
__device__ __forceinline__ uint64_t atom_desc(uint32_t start) {
  return (uint64_t)((start >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 32) | (1ull << 46);
}
// Instruction descriptor, kind::mxf4nvf4: e2m1 A and B (format 1), K-major,
// e4m3 scales (scale type 0), scale-factor ids 0, M = 128.
__host__ __device__ constexpr uint32_t idesc_fp4(int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kF4BM >> 4) << 24);
}

__global__ void __launch_bounds__(kF4Threads, 1)
    expert_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_sfb,
                           const F4Args a) {
  pdl_enter();  // before any global memory access (see moe_common.cuh)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kF4Slots * kF4SlotBytes);
  uint64_t* ready = full + kF4Slots;
  uint64_t* empty = ready + kF4Slots;
  uint64_t* rd = empty + kF4Slots;  // the rearranging warps have read the slot's packed words
  uint64_t* acc_full = rd + kF4Slots;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kF4Slots; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&ready[s], 8);
      ptx::mbar_init(&empty[s], 1);
      ptx::mbar_init(&rd[s], 8);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 8);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kF4MmaWarp) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  if (warp == kF4LoadWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_b);
    ptx::prefetch_tmap(&tmap_sfb);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // items per chunk: gate+up tiles of the same rows, or pairs of down tiles (the
  // last one alone when the tile count is odd)
  const int gate_up = a.proj == 0;
  const int n_tiles = a.N / kF4BM;
  const int m_items = gate_up ? n_tiles : (n_tiles + 1) / 2;
  const int total = *a.chunk_count * m_items;
  const int ksteps = (a.K + kF4BK - 1) / kF4BK;  // the last stage may hold one 128-input tile
  const int ktiles = a.K / 128;
  const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
  bool ok = true;
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort_flag, a.wait)) != 0;
  };

  if (warp == kF4LoadWarp) {
    int s = 0, g = 0;
    uint32_t ph = 0, issued = 0, issued_phase = 0;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int c = t / m_items, mi = t % m_items;
      const int e = a.chunks[3 * c], row0 = a.chunks[3 * c + 1];
      const int nmat = (gate_up || 2 * mi + 1 < n_tiles) ? 2 : 1;  // weight tiles in this item
      const uint8_t* cbase[2];
      const uint8_t* sbase[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int i = e * 3 + (gate_up ? m : 2);
        const int mt = gate_up ? mi : min(2 * mi + m, n_tiles - 1);
        cbase[m] = L.base + L.code_off[i] + (size_t)mt * ktiles * 8192u;      // 128x128 tiles of 8 KB, K minor
        sbase[m] = L.base + L.scale_off[i] + (size_t)mt * (a.K / 16) * 128u;  // [N/128][K/16][128]
      }
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&empty[s], ph ^ 1u)) {
          ok = false;
          break;
        }
        const int nt = min(2, ktiles - 2 * ks);  // 128-input tiles in this stage
        if (lane == 0 && !a.withhold) {
          f4_trace(a.trace, 0, g);
          uint8_t* sb = smem + s * kF4SlotBytes;
          const uint32_t bytes = (uint32_t)nmat * (uint32_t)nt * 9216u + 16384u + 2048u;  // codes + scales, B, B scales
          ptx::mbar_arrive_expect_tx(&full[s], bytes);
          for (int m = 0; m < nmat; ++m) {
            ptx::bulk_load(sb + kF4OffA + m * 16384, cbase[m] + (size_t)(2 * ks) * 8192u, (uint32_t)nt * 8192u,
                           &full[s]);
            ptx::bulk_load(sb + kF4OffSfaRaw + m * 2048, sbase[m] + (size_t)(16 * ks) * 128u, (uint32_t)nt * 1024u,
                           &full[s]);
          }
          ptx::tma_load_2d(sb + kF4OffB, &tmap_b, ks * 128, row0, &full[s]);
          ptx::tma_load_2d(sb + kF4OffSfbRaw, &tmap_sfb, ks * 16, row0, &full[s]);
          f4_trace(a.trace, 1, g);
        }
        ++g;
        __syncwarp();
        if (!a.withhold) {
          issued |= 1u << s;
          issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
        }
        if (++s == kF4Slots) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    for (int s2 = 0; s2 < kF4Slots; ++s2)
      if (issued & (1u << s2)) ptx::mbar_drain(&full[s2], (issued_phase >> s2) & 1u, kF4WaitLimit / 4);
    __syncwarp();
  } else if (warp == kF4MmaWarp) {
    int s = 0, g = 0;
    uint32_t ph = 0, acc_phase = 0;
    const uint32_t sb0 = ptx::smem_u32(smem);
    bool committed = false;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int c = t / m_items;
      const int nmma = min(kF4BN, (a.chunks[3 * c + 2] + 15) & ~15);
      const uint32_t idesc = idesc_fp4(nmma);
      if (!wait_all(acc_empty, acc_phase ^ 1u)) {
        ok = false;
        break;
      }
      acc_phase ^= 1u;
      ptx::tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&ready[s], ph)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (lane == 0) f4_trace(a.trace, 4, g);
        const uint32_t sb = sb0 + (uint32_t)(s * kF4SlotBytes);
        // this stage's scale atoms to TMEM (after the previous stage's MMAs, in issue order)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sf_copy_warp(tmem + kF4TmemSfa + 4u * j, atom_desc(sb + kF4OffSfa + j * 512));
          sf_copy_warp(tmem + kF4TmemSfa + 16u + 4u * j, atom_desc(sb + kF4OffSfa + 2048 + j * 512));
          sf_copy_warp(tmem + kF4TmemSfb + 4u * j, atom_desc(sb + kF4OffSfb + j * 512));
        }
        const uint64_t da = ptx::sw128_desc(sb + kF4OffA), db = ptx::sw128_desc(sb + kF4OffB);
        const uint32_t acc0 = ks != 0;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_fp4_warp(tmem + (uint32_t)(m * kF4BN), da + (uint64_t)(m * (16384 >> 4) + 2 * j), db + (uint64_t)(2 * j),
                         idesc, tmem + kF4TmemSfa + 16u * m + 4u * j, tmem + kF4TmemSfb + 4u * j, j ? 1u : acc0);
        ptx::mma_commit_warp(&empty[s]);
        if (lane == 0) f4_trace(a.trace, 5, g);
        ++g;
        __syncwarp();
        committed = true;
        if (++s == kF4Slots) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      ptx::mma_commit_warp(acc_full);
      __syncwarp();
    }
    if (committed) {
      const int last = (s + kF4Slots - 1) % kF4Slots;
      ptx::mbar_drain(&empty[last], (s == 0) ? (ph ^ 1u) : ph, kF4WaitLimit / 4);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- rearrange + epilogue (warps 0-7)
    const int n = threadIdx.x & 127, half = threadIdx.x >> 7;  // weight row (or token row), which 128-input tile
    int s = 0, g = 0, item = 0;
    uint32_t ph = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int c = t / m_items, mi = t % m_items;
      const int e = a.chunks[3 * c], row0 = a.chunks[3 * c + 1], rows = a.chunks[3 * c + 2];
      const int nmat = (gate_up || 2 * mi + 1 < n_tiles) ? 2 : 1;
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!wait_all(&full[s], ph)) {
          ok = false;
          break;
        }
        if (threadIdx.x == 0) f4_trace(a.trace, 2, g);
        const int nt = min(2, ktiles - 2 * ks);
        const bool have = half < nt;  // this thread's 128-input tile exists
        const uint32_t sb = ptx::smem_u32(smem) + (uint32_t)(s * kF4SlotBytes);
        // weight codes: the group's four words (512 bytes apart) -> one 16-byte K-major chunk
        uint32_t w[2][4][4];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int kg = 0; kg < 4; ++kg)
#pragma unroll
            for (int wd = 0; wd < 4; ++wd)
              w[m][kg][wd] = (have && m < nmat)
                                 ? ptx::lds_u32(sb + kF4OffA + m * 16384 + half * 8192 + ((kg * 4 + wd) * 128 + n) * 4)
                                 : 0u;
        // scales of this thread's two MMAs (k-blocks j = 2*half, 2*half+1): A rows n, B row n
        uint32_t sa[2][2], sbw[2];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * half + jj;
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            uint32_t v = 0;
            if (have && m < nmat)
#pragma unroll
              for (int k1 = 0; k1 < 4; ++k1)
                v |= ptx::lds_u8(sb + kF4OffSfaRaw + m * 2048 + (4 * j + k1) * 128 + n) << (8 * k1);
            sa[m][jj] = v;
          }
          sbw[jj] = have ? ptx::lds_u32(sb + kF4OffSfbRaw + 16 * n + 4 * j) : 0u;
        }
        // every packed word is read before any is overwritten (a bounded wait, unlike a
        // named barrier, so a warp that gave up earlier cannot leave the others stuck)
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&rd[s]);
        if (!wait_all(&rd[s], ph)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int kg = 0; kg < 4; ++kg)
            ptx::sts_v4(sb + kF4OffA + m * 16384 + swz128(n, 4 * half + kg),
                        make_uint4(w[m][kg][0], w[m][kg][1], w[m][kg][2], w[m][kg][3]));
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * half + jj;
          const int at = 16 * (n & 31) + 4 * (n >> 5);
#pragma unroll
          for (int m = 0; m < 2; ++m)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sb + kF4OffSfa + m * 2048 + j * 512 + at), "r"(sa[m][jj])
                         : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sb + kF4OffSfb + j * 512 + at), "r"(sbw[jj]) : "memory");
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ready[s]);
        if (threadIdx.x == 0) f4_trace(a.trace, 3, g);
        ++g;
        if (++s == kF4Slots) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      if (!wait_all(acc_full, acc_phase)) {
        ok = false;
        break;
      }
      acc_phase ^= 1u;
      ptx::tc_fence_after();
      if (threadIdx.x == 0) f4_trace(a.trace, 6, item);
      // epilogue: warp w reads TMEM lane quarter w%4 and half w/4 of the chunk's columns
      // (tokens), split in steps of 16 so both halves have work on short chunks
      const int q = warp & 3, ch = warp >> 2;
      const int cpw = ((rows + 31) / 32) * 16, c0 = ch * cpw;
      const int nrow0 = (gate_up ? mi : 2 * mi) * kF4BM + q * 32 + lane;
      float ts[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) ts[m] = L.tscale[e * 3 + (gate_up ? m : 2)];
      // the warp's 64 token scales, two per lane, loaded before any store (they are
      // broadcast with shuffles below)
      float scl[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int tok = c0 + 32 * u + lane;
        scl[u] = 0.0f;
        if (32 * u + lane < cpw && tok < rows) {
          const int r = row0 + tok;
          scl[u] = gate_up ? a.row_scale[a.perm[r] / a.topk] : a.row_scale[r];
        }
      }
      float* __restrict__ out = a.out;
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
      for (int cb = c0; cb < c0 + cpw && cb < rows; cb += 16) {
        uint32_t r0[16], r1[16];
        ptx::tmem_ld16(lane_base + (uint32_t)cb, r0);
        ptx::tmem_ld16(lane_base + (uint32_t)(kF4BN + cb), r1);
        ptx::tmem_ld_wait();
        const int u = (cb - c0) >> 5;  // which of the lane's two scales (warp-uniform)
        const float su = u ? scl[1] : scl[0];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int tok = cb + j;
          const float sc = __shfl_sync(0xffffffffu, su, (tok - c0) & 31);
          if (tok >= rows) continue;
          const size_t o = (size_t)(row0 + tok) * a.N + nrow0;
          if (gate_up) {
            const float g = __uint_as_float(r0[j]) * (sc * ts[0]), uu = __uint_as_float(r1[j]) * (sc * ts[1]);
            out[o] = __fdividef(g, 1.0f + __expf(-g)) * uu;
          } else {
            const float f = sc * ts[0];
            out[o] = __uint_as_float(r0[j]) * f;
            if (nmat == 2) out[o + kF4BM] = __uint_as_float(r1[j]) * f;
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty);
      if (threadIdx.x == 0) f4_trace(a.trace, 7, item);
      ++item;
    }
  }

  if (!ok) {
    *abort_flag = 1;
    if (a.status) atomicExch(a.status, (int32_t)MOE_ERR_TIMEOUT);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kF4MmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 fp4_tmap_encoder() {
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

int fp4_sm_count() {
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

// A row-major byte matrix [rows][cols] with a box of box_cols x 128 rows.
bool encode_bytes_map(CUtensorMap* map, const void* base, int rows, int cols, int box_cols, bool swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = fp4_tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)kF4BN};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_expert_gemm_fp4(const uint8_t* packed, int E, int H, int F, int T, int k, bool gateup,
                                   const Workspace& ws, int32_t* status, uint64_t* trace, GemmHooks hooks,
                                   cudaStream_t stream) {
  F4Args a{};
  a.trace = gateup ? reinterpret_cast<unsigned long long*>(trace) : nullptr;
  a.packed = packed;
  a.E = E;
  a.H = H;
  a.F = F;
  a.chunks = ws.chunks;
  a.chunk_count = ws.chunk_count;
  a.perm = ws.perm;
  a.topk = k;
  a.status = status;
  a.wait = hooks.wait_cycles ? (long long)hooks.wait_cycles : kF4WaitLimit;
  a.withhold = hooks.withhold ? 1 : 0;
  const int R = T * k;
  const void* act;
  const void* sfb;
  int ld;
  if (gateup) {
    a.N = F;
    a.K = H;
    a.proj = 0;
    a.row_scale = ws.sx;
    a.out = (float*)ws.h;
    act = ws.xs4;
    sfb = ws.xsf4;
    ld = ws.ldx;
  } else {
    a.N = H;
    a.K = F;
    a.proj = 2;
    a.row_scale = ws.sh;
    a.out = ws.o;
    act = ws.hs4;
    sfb = ws.hsf4;
    ld = ws.ldh;
  }
  CUtensorMap mb, ms;
  if (!encode_bytes_map(&mb, act, R, a.K / 2, 128, true) || !encode_bytes_map(&ms, sfb, R, ld, 16, false))
    return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kF4Smem);
  if (err != cudaSuccess) return err;
  launch_chained(expert_gemm_fp4_kernel, dim3(fp4_sm_count()), dim3(kF4Threads), kF4Smem, stream, mb, ms, a);
  return cudaGetLastError();
}

}  // namespace moe

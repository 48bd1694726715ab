// Dequant-fused grouped expert GEMM on warp-level tensor cores (mma.sync
// m16n8k16, fp32 accumulate).  The packed weights of one expert are streamed
// once per (128-row weight tile, chunk of token rows), unpacked in registers,
// written to shared memory as 16-bit operands and multiplied against the
// chunk's activation rows (the pages' packed-linear operator: MoE
// mixed-precision page sec. 2.3 / 3.5; SwiGLU epilogue fused as in its
// sec. 3.6 "fused linear + activation").
//
// Orientation: MMA rows = weight output rows n (A operand, [n][k] in smem),
// MMA columns = token rows (B operand, [token][k] in smem), so one dequantized
// weight tile serves every token of the chunk.
#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kNT = 128;       // weight rows per CTA
constexpr int kKT = 128;       // inputs per main-loop step (one packed tile)
constexpr int kLds = kKT + 8;  // padded smem row (elements) -> conflict-free ldmatrix

template <typename T>
struct MmaType;
template <>
struct MmaType<__half> {
  __device__ static __forceinline__ void mma(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  }
  __device__ static __forceinline__ __half from_float(float v) { return __float2half_rn(v); }
};
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x2(uint32_t* r, const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r[0]), "=r"(r[1]) : "r"(a));
}

// Codes of one thread for one main-loop step: two groups (kg = 2*half, 2*half+1)
// of its weight row, up to 4 words each, plus the scales.
struct Frag {
  uint32_t w[2][4];
  uint32_t sc;  // int: two fp16 scales (lo = first group); NVFP4: four e4m3 bytes
};

__device__ __forceinline__ void load_frag(Frag& f, const uint32_t* __restrict__ codes,
                                          const uint8_t* __restrict__ scales, int fmt, int n, int kt,
                                          int half, int K) {
  const int wpg = fmt_words(fmt);
#pragma unroll
  for (int gi = 0; gi < 2; ++gi) {
    const int kg = 2 * half + gi;
    const uint64_t base = word_index(n, kt * kKT + kg * 32, K, wpg, 0);
#pragma unroll
    for (int w = 0; w < 4; ++w) f.w[gi][w] = (w < wpg) ? __ldg(codes + base + (uint64_t)w * 128u) : 0u;
  }
  const int g0 = kt * 4 + 2 * half;  // first group index (32 inputs) of this thread
  if (fmt == MOE_FMT_NVFP4) {
    const int G16 = K / 16;
    uint32_t s = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) s |= (uint32_t)__ldg(scales + scale_index(n, 2 * g0 + b, G16)) << (8 * b);
    f.sc = s;
  } else {
    const uint16_t* s16 = reinterpret_cast<const uint16_t*>(scales);
    const int G = K / 32;
    f.sc = (uint32_t)__ldg(s16 + scale_index(n, g0, G)) | ((uint32_t)__ldg(s16 + scale_index(n, g0 + 1, G)) << 16);
  }
}

// Unpacked 16-bit values of code i (0..31) of group gi.
template <typename T>
__device__ __forceinline__ float code_value(const Frag& f, int fmt, int gi, int i) {
  if (fmt == MOE_FMT_NVFP4) {
    const uint32_t c = (f.w[gi][i >> 3] >> (4 * (i & 7))) & 15u;
    const uint32_t sb = (f.sc >> (8 * (2 * gi + (i >> 4)))) & 255u;
    return e2m1_value(c) * e4m3_value(sb);  // exact in fp16 (<= 6 significant bits, within range)
  }
  const float s = __half2float(__ushort_as_half((uint16_t)(f.sc >> (16 * gi))));
  // code i of a pair-interleaved word: pair i/2 at the low (even i) or high (odd i) half-word
  int q;
  if (fmt == MOE_FMT_INT4) {
    q = (int)((f.w[gi][i >> 3] >> ((i & 1) * 16 + ((i & 7) >> 1) * 4)) & 15u) - 8;
  } else if (fmt == MOE_FMT_INT2) {
    q = (int)((f.w[gi][i >> 4] >> ((i & 1) * 16 + ((i & 15) >> 1) * 2)) & 3u) - 2;
  } else {
    const uint32_t lo = (f.w[gi][i >> 4] >> ((i & 1) * 16 + ((i & 15) >> 1) * 2)) & 3u;
    const uint32_t hi = (f.w[gi][2] >> ((i & 1) * 16 + (i >> 1))) & 1u;
    q = (int)(lo | (hi << 2)) - 4;
  }
  return s * (float)q;  // exact in fp32; rounded once to the 16-bit operand type
}

template <typename T>
__device__ __forceinline__ void store_frag(const Frag& f, int fmt, T* row /* smem row of kLds */, int half) {
#pragma unroll
  for (int gi = 0; gi < 2; ++gi) {
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      uint4 v;
      T* t = reinterpret_cast<T*>(&v);
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = MmaType<T>::from_float(code_value<T>(f, fmt, gi, c8 * 8 + j));
      *reinterpret_cast<uint4*>(row + (2 * half + gi) * 32 + c8 * 8) = v;
    }
  }
}

}  // namespace

struct GemmArgs {
  const uint8_t* packed;
  int E, H, F;
  int N, K;
  int proj;             // 0: gate+up (SwiGLU epilogue), 2: down
  const void* act;      // [rows][K] 16-bit activations in sorted row order
  const int32_t* chunks;
  const int32_t* chunk_count;
  const float* row_scale;  // NVFP4: gate/up -> sx per token, down -> sh per row; else null
  const int32_t* perm;     // sorted row -> entry t*k+j
  int topk;
  void* out;            // gate/up: h ([rows][F], fp16 int / fp32 NVFP4); down: o fp32 [rows][H]
};

// MT = token rows per chunk (16 or 64).  256 threads = 8 warps: warp_n (0..3)
// takes 32 weight rows, warp_m (0..1) takes MT/2 tokens.
template <typename T, int MT, bool GATEUP>
__global__ void __launch_bounds__(256) expert_gemm_mma_kernel(GemmArgs a) {
  constexpr int NMAT = GATEUP ? 2 : 1;
  constexpr int NT8 = MT / 16;  // n8 tiles per warp
  extern __shared__ __align__(16) uint8_t smem_raw[];
  T* sA = reinterpret_cast<T*>(smem_raw);            // [NMAT][kNT][kLds]
  T* sB = sA + NMAT * kNT * kLds;                    // [MT][kLds]

  const int n_tiles = a.N / kNT;
  const int chunk = blockIdx.x / n_tiles;
  const int ntile = blockIdx.x % n_tiles;
  if (chunk >= *a.chunk_count) return;
  const int e = a.chunks[3 * chunk], row0 = a.chunks[3 * chunk + 1], rows = a.chunks[3 * chunk + 2];

  const LayerHdr L = hdr_view(a.packed, a.E, a.H, a.F);
  const uint32_t* codes[NMAT];
  const uint8_t* scales[NMAT];
  int fmt[NMAT];
  float tsc[NMAT];
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    const int i = e * 3 + a.proj + m;
    fmt[m] = L.fmt[i];
    codes[m] = reinterpret_cast<const uint32_t*>(L.base + L.code_off[i]);
    scales[m] = L.base + L.scale_off[i];
    tsc[m] = (fmt[m] == MOE_FMT_NVFP4) ? L.tscale[i] : 1.0f;
  }

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nl = tid & 127, half = tid >> 7;
  const int n = ntile * kNT + nl;
  const int warp_n = warp & 3, warp_m = warp >> 2;
  const T* act = reinterpret_cast<const T*>(a.act);

  float acc[NMAT][2][NT8][4];
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < NT8; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][i][j][c] = 0.0f;

  constexpr int BCH = MT * (kKT / 8) / 256;  // 16-byte activation chunks per thread per step
  Frag fr[NMAT];
  uint4 bv[BCH];
  const int ksteps = a.K / kKT;

  auto load_step = [&](int kt) {
#pragma unroll
    for (int m = 0; m < NMAT; ++m) load_frag(fr[m], codes[m], scales[m], fmt[m], n, kt, half, a.K);
#pragma unroll
    for (int c = 0; c < BCH; ++c) {
      const int id = tid + 256 * c;
      const int r = id / (kKT / 8), c8 = id % (kKT / 8);
      bv[c] = (r < rows) ? __ldg(reinterpret_cast<const uint4*>(act + (size_t)(row0 + r) * a.K + kt * kKT) + c8)
                         : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto store_step = [&]() {
#pragma unroll
    for (int m = 0; m < NMAT; ++m) store_frag<T>(fr[m], fmt[m], sA + (m * kNT + nl) * kLds, half);
#pragma unroll
    for (int c = 0; c < BCH; ++c) {
      const int id = tid + 256 * c;
      const int r = id / (kKT / 8), c8 = id % (kKT / 8);
      *reinterpret_cast<uint4*>(sB + r * kLds + c8 * 8) = bv[c];
    }
  };

  load_step(0);
  for (int kt = 0; kt < ksteps; ++kt) {
    store_step();
    __syncthreads();
    if (kt + 1 < ksteps) load_step(kt + 1);  // next step's global loads overlap the MMAs
#pragma unroll
    for (int ks = 0; ks < kKT / 16; ++ks) {
      uint32_t bf[NT8][2];
      if (NT8 == 1) {
        const int r = warp_m * (MT / 2) + (lane & 7);
        ldsm_x2(bf[0], sB + r * kLds + ks * 16 + ((lane >> 3) & 1) * 8);
      } else {
#pragma unroll
        for (int j = 0; j < NT8; j += 2) {
          const int r = warp_m * (MT / 2) + j * 8 + (lane & 7) + ((lane >> 4) << 3);
          uint32_t t4[4];
          ldsm_x4(t4, sB + r * kLds + ks * 16 + ((lane >> 3) & 1) * 8);
          bf[j][0] = t4[0];
          bf[j][1] = t4[1];
          bf[j + 1][0] = t4[2];
          bf[j + 1][1] = t4[3];
        }
      }
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint32_t af[4];
          const int r = warp_n * 32 + i * 16 + (lane & 15);
          ldsm_x4(af, sA + (m * kNT + r) * kLds + ks * 16 + (lane >> 4) * 8);
#pragma unroll
          for (int j = 0; j < NT8; ++j) MmaType<T>::mma(acc[m][i][j], af, bf[j]);
        }
      }
    }
    __syncthreads();
  }

  // Epilogue.  acc[m][i][j][c]: weight row warp_n*32 + i*16 + lane/4 (+8 for c >= 2),
  // token warp_m*MT/2 + j*8 + 2*(lane%4) (+1 for odd c).
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < NT8; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int nn = ntile * kNT + warp_n * 32 + i * 16 + (lane >> 2) + ((c >> 1) << 3);
        const int tok = warp_m * (MT / 2) + j * 8 + 2 * (lane & 3) + (c & 1);
        if (tok >= rows) continue;
        const int r = row0 + tok;
        if (GATEUP) {
          float g = acc[0][i][j][c], u = acc[NMAT - 1][i][j][c];
          if (a.row_scale) {  // NVFP4: per-token activation scale and per-matrix weight scales
            const float sx = a.row_scale[a.perm[r] / a.topk];
            g *= sx * tsc[0];
            u *= sx * tsc[NMAT - 1];
          }
          const float h = g / (1.0f + __expf(-g)) * u;
          if (a.row_scale) reinterpret_cast<float*>(a.out)[(size_t)r * a.N + nn] = h;
          else reinterpret_cast<__half*>(a.out)[(size_t)r * a.N + nn] = __float2half_rn(h);
        } else {
          float o = acc[0][i][j][c];
          if (a.row_scale) o *= a.row_scale[r] * tsc[0];
          reinterpret_cast<float*>(a.out)[(size_t)r * a.N + nn] = o;
        }
      }
}

template <typename T, int MT, bool GATEUP>
static cudaError_t launch_one(const GemmArgs& a, int max_chunks, cudaStream_t stream) {
  constexpr int NMAT = GATEUP ? 2 : 1;
  const size_t smem = (size_t)(NMAT * kNT + MT) * kLds * sizeof(T);
  auto kern = expert_gemm_mma_kernel<T, MT, GATEUP>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long long grid = (long long)max_chunks * (a.N / kNT);
  kern<<<(unsigned)grid, 256, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_expert_gemm_mma(const uint8_t* packed, int E, int H, int F, int k, bool fp4, bool gateup,
                                   int chunk_rows, int max_chunks, const Workspace& ws, cudaStream_t stream) {
  GemmArgs g{};
  g.packed = packed;
  g.E = E;
  g.H = H;
  g.F = F;
  g.chunks = ws.chunks;
  g.chunk_count = ws.chunk_count;
  g.perm = ws.perm;
  g.topk = k;
  if (gateup) {  // gate + up -> h
    g.N = F;
    g.K = H;
    g.proj = 0;
    g.act = ws.xs;
    g.row_scale = fp4 ? ws.sx : nullptr;
    g.out = ws.h;
    return chunk_rows == 16 ? launch_one<__half, 16, true>(g, max_chunks, stream)
                            : launch_one<__half, 64, true>(g, max_chunks, stream);
  }
  // down -> o
  g.N = H;
  g.K = F;
  g.proj = 2;
  g.act = fp4 ? ws.hb : ws.h;
  g.row_scale = fp4 ? ws.sh : nullptr;
  g.out = ws.o;
  return chunk_rows == 16 ? launch_one<__half, 16, false>(g, max_chunks, stream)
                          : launch_one<__half, 64, false>(g, max_chunks, stream);
}

}  // namespace moe

/*
 * moe.h -- C ABI of the B200 (sm_100a) quantized Mixture-of-Experts FFN layer.
 *
 * Three calls:
 *   moe_pack           quantizes fp32 expert weights into the packed layer buffer
 *                      (optionally keeping each matrix's largest weights in an
 *                      fp16 side list);
 *   moe_layer_forward  runs the layer: fp32 router -> top-k with a softmax over
 *                      the chosen k -> permutation of tokens by expert ->
 *                      per-expert SwiGLU FFN on dequantized weights -> weighted
 *                      combine;
 *   moe_layer_forward_noalloc  the same with a workspace inside the library.
 *
 * Where the method comes from (web pages; section numbers as printed there):
 *  - "quantized MoE LLM inference" (cloud.baidu.com article 9434801), expert
 *    routing section: logits = router(x); top-k indices; weights = softmax of
 *    the chosen logits; output = weighted sum of the chosen experts.
 *  - "MoE混合精度量化实战：门控保精度+专家激进压缩" (MoE mixed-precision
 *    quantization in practice): sec. 2.1 keeps the gate/router unquantized and
 *    quantizes expert-input activations per token with a live scale;
 *    sec. 2.3 and 3.5 pack each expert in 128-column blocks, each block
 *    quantized on its own, concatenated into one stream read by a custom
 *    packed-linear kernel; sec. 3.3 gives the 4-bit code range [-8, 7].
 *  - AlphaQ MoE quantization stack (mhpn.cn news 995352), sec. 2.2 and 4.2:
 *    bit widths chosen per expert and per projection (gate 3-bit, middle 2-bit,
 *    output 4-bit), group size 32.
 *  - "Expert-aware quantisation: near-Q4 quality at near-Q2 size?": frequently
 *    routed ("hot") experts at 4-bit, the rest ("cold") at 2-bit, and below
 *    2 bits for the coldest (the 1-bit sign code here).
 *  - The same mixed-precision page, sec. 4.2, tip 2: each expert's top 0.05% of
 *    weights by |w| kept in fp16 beside the quantized rest (MOE_FMT_OUTLIERS).
 *  - The NVFP4 remarks of the MoE inference page: e2m1 weights with e4m3 block
 *    scales; with MOE_ACT_NVFP4 the activations take the same format and prefill
 *    runs the tensor core's block-scaled FP4 MMA.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless marked HOST.  The caller owns all
 *    memory; the library allocates no device or pinned memory and keeps no
 *    state between calls except a per-process cache of device properties.
 *    Two exceptions belong to moe_layer_forward_noalloc alone: its fixed
 *    scratch array (a __device__ array that every GPU loading the library
 *    holds) and a per-device cache of that array's address (see there).
 *  - Calls are asynchronous on `stream`; nothing is synchronized inside.
 *  - Errors are reported by the return code only.  Arguments are validated
 *    before anything is launched, so a call that returns an error other than
 *    MOE_ERR_CUDA has launched nothing.
 *  - Device-side failures (a bounded wait that gave up, an fp16 range
 *    overflow) are written as a moe_status value to moe_debug.status when that
 *    pointer is given (the caller zeroes it and reads it after synchronizing).
 *    They happen after the call has returned, so its return code cannot carry
 *    them: without moe_debug.status a call that met one still returns MOE_OK
 *    and its y is undefined.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,        /* null pointer, out-of-range count or index */
  MOE_ERR_ALIGN = 2,      /* a pointer misses its required alignment */
  MOE_ERR_SHAPE = 3,      /* H or F not a multiple of 128, E > 256, k > min(E, 8), ... */
  MOE_ERR_WORKSPACE = 4,  /* workspace or output buffer too small */
  MOE_ERR_FORMAT = 5,     /* unknown format code, NVFP4 mixed with integer formats,
                             or a packed buffer whose header disagrees */
  MOE_ERR_CUDA = 6,       /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 7,    /* device-side bounded wait gave up (status word only) */
  MOE_ERR_UNSUPPORTED_DEVICE = 8, /* current device is not compute capability 10.0 */
  MOE_ERR_RANGE = 9       /* integer-format layer: a SwiGLU output h reached the fp16 limit
                             (|h| >= 65520 rounds to inf); status word only */
} moe_status;

/* Weight formats, chosen per expert and per projection. */
enum {
  MOE_FMT_INT1 = 1,   /* sign codes {-1,+1},      fp16 scale per 32 inputs (mean |w|): the
                         sub-2-bit cold tier of the expert-aware quantisation page */
  MOE_FMT_INT2 = 2,   /* symmetric codes {-1,0,1}, fp16 scale per 32 inputs */
  MOE_FMT_INT3 = 3,   /* symmetric codes [-3,3],   fp16 scale per 32 inputs */
  MOE_FMT_INT4 = 4,   /* symmetric codes [-7,7],   fp16 scale per 32 inputs */
  MOE_FMT_NVFP4 = 16, /* e2m1 codes, e4m3 scale per 16 inputs, fp32 scale per matrix */
  MOE_FMT_OUTLIERS = 0x80  /* flag OR'ed onto a format code: the matrix keeps its top 0.05% of
                              weights by |w| (floor(N*K*5/10000), ties to the lower row-major
                              index) in an fp16 side list; they are zeroed before the group
                              quantization and their residual w - dequant(w) is added back in the
                              expert GEMMs (MoE mixed-precision page sec. 4.2, tip 2).  Integer
                              and NVFP4 matrices with FP8 activations. */
};

/*
 * Packed layer buffer (written by moe_pack; little-endian; read by the kernels).
 *
 * Header, 16384 bytes:
 *   [0]     u32 magic 0x51454F4D        [4]  u32 version 1
 *   [8]     i32 E   [12] i32 H   [16] i32 F
 *   [20]    u32 flags           bit 0: the layer has an outlier section (else 0)
 *   [24]    u64 out_sec         byte offset of the outlier section (0 if none)
 *   [32]    u8  fmt[768]        base formats (without MOE_FMT_OUTLIERS) of (expert e,
 *                               projection p) at e*3+p, p = 0 gate [F x H], 1 up [F x H],
 *                               2 down [H x F]; entries past E*3 are zero
 *   [800]   u64 code_off[768]   byte offset of each matrix's codes
 *   [6944]  u64 scale_off[768]  byte offset of each matrix's scales
 *   [13088] f32 tscale[768]     NVFP4 per-matrix scale (0 for integer formats)
 *   [16160..16384) zero
 * Sections follow from byte 16384 in (expert, projection) order, codes then
 * scales, each starting on a 256-byte boundary.  Sizes for an N x K matrix:
 * integer b-bit codes N*K*b/8 bytes, scales N*K/16 bytes (fp16 per 32);
 * NVFP4 codes N*K/2 bytes, scales N*K/16 bytes (e4m3 per 16).
 *
 * Quantization of one N x K matrix (N outputs, K inputs, row-major fp32):
 *   integer b-bit (qmax = 2^(b-1)-1; the code -2^(b-1) is not used):
 *     per row n and group g of 32 consecutive inputs: amax = max|w|;
 *     s = fp16 round-to-nearest-even of the fp32 quotient amax/qmax, saturated
 *     to 65504; q = clamp(rint(w/s), -qmax, qmax) with an IEEE fp32 division
 *     and round-half-even (s == 0 gives q = 0).  Dequantized weight = s*q.
 *   1-bit sign code (the sub-2-bit cold tier): per row and group of 32,
 *     s = fp16 round-to-nearest-even of (fp32 sum of |w| in input order)/32,
 *     saturated to 65504 (the least-squares scale of a sign code); q = +1 for
 *     w >= 0, else -1.  Dequantized weight = s*q.
 *   NVFP4: sT = amax(matrix)/2688 in fp32 (1 if the matrix is all zero);
 *     per row and block of 16 inputs: sb = e4m3(blockmax/(6*sT)) (round to
 *     nearest even, saturate to 448); v = e2m1(w/(sb*sT)) (nearest even,
 *     saturate to 6; sb == 0 gives v = 0).  Dequantized weight = e2m1(v)*sb*sT.
 * Code layout: tiles of 128 outputs x 128 inputs, tile order output-block
 * major, input-block minor.  Inside a tile, u32 words ordered
 * [kg 0..3][word 0..b-1][n 0..127] (kg = group of 32 inputs inside the tile,
 * b = 1, 2, 3, 4 words per group; NVFP4 uses 4).  Stored integer code
 * u = q+2^(b-1); 1-bit: u = (q+1)/2.
 * Inside an integer word the two codes of each pair (2j, 2j+1) sit 16 bits
 * apart (even code in the low half-word), so one mask of a shifted word
 * yields both:
 *   4-bit: codes 8w..8w+7 in word w; code 8w+2j at bits 4j..4j+3, code
 *          8w+2j+1 at bits 16+4j..16+4j+3 (j = 0..3)
 *   1-bit: codes 0..31 in word 0; code 2j at bit j, code 2j+1 at bit 16+j
 *          (j = 0..15)
 *   2-bit: codes 16w..16w+15 in word w; code 16w+2j at bits 2j..2j+1, code
 *          16w+2j+1 at bits 16+2j..17+2j (j = 0..7)
 *   3-bit: words 0-1 hold the low two bits of u as for 2-bit; word 2 holds
 *          bit 2 of u: of pair m = 4c+j (c, j = 0..3), code 2m at bit
 *          P = 8*(c/2) + c%2 + 2j and code 2m+1 at bit 16+P
 *   NVFP4: codes 8w..8w+7 in word w, code 8w+i at bits 4i..4i+3.
 * Scale layout: [N/128][K/gs][128] (gs = 32 integer, 16 NVFP4).
 *
 * Outlier section (present when any fmt code carries MOE_FMT_OUTLIERS), at the
 * first 256-byte boundary after the last expert section:
 *   u64 side_off[768]       byte offset of each matrix's side list (0 if none)
 *   u32 scratch[64 + 65536] selection state of moe_pack (contents unspecified)
 * then, from the next 256-byte boundary, one side list per opted-in matrix in
 * (expert, projection) order, each on a 256-byte boundary:
 *   u32 row_ptr[N+1]        row n's entries are [row_ptr[n], row_ptr[n+1])
 *   u32 entry[n_out]        column | (fp16 residual bits << 16), in (row, column)
 *                           order; n_out = floor(N*K*5/10000)
 * The residual is w - dequant at that position, taken in double and rounded
 * once to fp16: w itself for every format with a zero code, w - s for the
 * 1-bit sign code (a zeroed weight reads +s).  The layer computes with
 * dequant(codes) + residual.  The quantization above then sees the matrix with
 * its outliers set to 0 (group scales, NVFP4 sT and block scales included).
 */

/*
 * moe_pack -- quantize and pack fp32 expert weights (the pages' expert packing,
 * MoE mixed-precision page sec. 2.3/3.5; bit widths per expert/projection as on
 * the AlphaQ page sec. 4.2).
 *
 * Size query: out == NULL -> *bytes_out = total size of the layer buffer; no
 *   device work.  code_off / scale_off (HOST, [E*3], nullable) receive the
 *   section offsets in both modes.
 * Pack: writes the header and the sections of experts [e0, e0+ne) into `out`
 *   (DEVICE, 256-byte aligned, out_bytes >= the queried size), so a layer too
 *   large to stage in fp32 can be packed a few experts at a time.
 *   W: DEVICE fp32 [ne][3][H*F] -- gate [F][H], up [F][H], down [H][F],
 *   row-major, 16-byte aligned.  fmt: HOST u8 [E*3], a format code per matrix,
 *   optionally OR'ed with MOE_FMT_OUTLIERS.  moe_layer_forward must be given the
 *   same codes (flags included) as moe_pack.
 * Shapes: 1 <= E <= 256; H, F multiples of 128 (up to 32768).
 * Errors: MOE_ERR_ARG (null W/fmt/bytes_out, bad e0/ne), MOE_ERR_SHAPE,
 *   MOE_ERR_FORMAT, MOE_ERR_ALIGN, MOE_ERR_WORKSPACE (out_bytes too small),
 *   MOE_ERR_UNSUPPORTED_DEVICE, MOE_ERR_CUDA.
 */
MOE_API moe_status moe_pack(const float* W, int32_t e0, int32_t ne, int32_t E, int32_t H, int32_t F,
                    const uint8_t* fmt, void* out, uint64_t out_bytes, uint64_t* bytes_out,
                    uint64_t* code_off, uint64_t* scale_off, cudaStream_t stream);

/* Activation formats of an NVFP4 layer's expert GEMMs (moe_weights.act). */
enum {
  MOE_ACT_FP8 = 0,    /* per-token dynamic FP8: x per token and the SwiGLU output h per row as
                         e4m3 codes with scale amax/448 (MoE mixed-precision page, sec. 2.1) */
  MOE_ACT_NVFP4 = 1   /* NVFP4 activations: x per token and h per row take the weights' NVFP4
                         rule with the row as the tensor (s = amax/2688 in fp32, 1 for an
                         all-zero row; e4m3 block scale per 16 = e4m3(blockmax/(6*s)); e2m1
                         codes = e2m1(a/(sb*s)), 0 where sb = 0).  Prefill batches then run the
                         block-scaled FP4 tensor-core MMA (tcgen05.mma kind::mxf4nvf4) on the
                         codes and block scales of both operands, with s and the weights'
                         tensor scale applied to the sums. */
};

/* A packed layer as moe_layer_forward reads it. */
typedef struct {
  int32_t E, H, F;
  const uint8_t* fmt;   /* HOST [E*3]: must equal the fmt the buffer was packed with */
  const void* packed;   /* DEVICE, 256-byte aligned, written by moe_pack */
  uint64_t packed_bytes;
  int32_t act;          /* MOE_ACT_*: activation format of an NVFP4 layer; 0 for integer layers
                           (MOE_ERR_FORMAT otherwise) */
} moe_weights;

/* Optional outputs of moe_layer_forward; every pointer is DEVICE and nullable. */
typedef struct {
  int32_t* topk_idx;  /* [T*k] chosen experts, descending logit (ties: lower index) */
  float* topk_w;      /* [T*k] softmax weights over the chosen k */
  int32_t* perm;      /* [T*k] row r of the expert-sorted order holds entry t*k+j */
  int32_t* inv;       /* [T*k] entry t*k+j -> its row */
  int32_t* counts;    /* [E]   rows per expert */
  uint8_t* xq;        /* [T*H] NVFP4 layers: e4m3 codes of x */
  float* sx;          /* [T]   NVFP4 layers: per-token scale of x (amax/448) */
  uint8_t* hq;        /* [T*k*F] NVFP4 layers: e4m3 codes of the SwiGLU output, sorted rows */
  float* sh;          /* [T*k] NVFP4 layers: per-row scale of the SwiGLU output */
  int32_t* status;    /* [1]   device-side error code (moe_status), 0 if none */
  cudaEvent_t* stage_events; /* HOST [MOE_STAGE_EVENTS] or NULL: recorded on `stream` before
                                router+top-k, permutation, activation gather/quantization,
                                gate/up GEMM, h quantization (NVFP4), down GEMM, combine,
                                and after combine, so stage times can be read back */
  uint64_t* trace;    /* [MOE_TRACE_WORDS] or NULL: diagnostics of the gate/up expert GEMM:
                         clock64 stamps taken by CTA 0, MOE_TRACE_EVENTS rows of
                         MOE_TRACE_STAGES entries.  Zero it before the call.
                         tcgen05 GEMM (many rows per expert), per pipeline stage: row 0
                         producer got a free stage, 1 producer issued its copies, 2 dequant
                         warp 0 saw the stage land, 3 dequant warp 0 released it, 4 MMA lane
                         saw it ready, 5 MMA issued and committed it; per work item: row 6
                         epilogue start, row 7 its end.
                         Decode GEMV (few rows per expert), per weight tile: row 0 producer got
                         a free stage, 1 producer issued its copies, 2 consumer warp 0 found it
                         landed, 3 consumer warp 0 released it; per work item: row 4 producer
                         loaded the following item, 6 consumers started it, 7 finished it. */
  uint32_t test_withhold; /* test hook, 0 in normal use: nonzero makes the copy warps of the expert
                             GEMMs issue no loads, so their consumers' bounded waits run out.  The
                             call then writes MOE_ERR_TIMEOUT to *status; the outputs are undefined
                             and the context stays usable. */
  uint32_t wait_cycles;   /* budget of the expert GEMMs' waits on their pipelines, in clock cycles;
                             0: the default (~1-2 s).  Waits for copies still in flight at exit keep
                             the default. */
  uint8_t* xsb;       /* [T*H/16] MOE_ACT_NVFP4: e4m3 block scales of x (xq then holds one e2m1 code
                         per byte, sx the row scales amax/2688) */
  uint8_t* hsb;       /* [T*k*F/16] MOE_ACT_NVFP4: e4m3 block scales of h, sorted rows (hq: one e2m1
                         code per byte; sh: row scales) */
} moe_debug;

#define MOE_TRACE_EVENTS 8
#define MOE_TRACE_STAGES 1024
#define MOE_TRACE_WORDS (MOE_TRACE_EVENTS * MOE_TRACE_STAGES)

#define MOE_STAGE_EVENTS 8

/*
 * moe_layer_forward -- y = MoE(x).
 *
 * x: DEVICE bf16 [T][H], 16-byte aligned.  router_w: DEVICE fp32 [E][H]
 *   (16-byte aligned); router_b: DEVICE fp32 [E] or NULL.  k: 1..min(E, 8).
 * y: DEVICE bf16 [T][H] (16-byte aligned), fully overwritten.
 * ws: DEVICE workspace, 256-byte aligned; ws == NULL -> *ws_bytes_out = the
 *   size needed for (T, k, weights) and nothing runs.
 * Steps (all on `stream`):
 *   1. logits[t][e] = sum_h x[t][h]*Wr[e][h] (+ b[e]) accumulated in fp32
 *      (the router stays unquantized: MoE mixed-precision page sec. 2.1); for
 *      many tokens each fp32 weight is split exactly into three bf16 terms so
 *      the tensor cores form exact products, summed in fp32 chunks of 64
 *      inputs with Kahan-compensated chunk sums;
 *   2. top-k (ties to the lower expert index; NaN ranks lowest), then
 *      w = softmax over the k chosen logits (expert-routing section of the
 *      quantized-MoE-inference page);
 *   3. counts per expert, exclusive offsets and a stable permutation (rows of
 *      one expert in ascending token order);
 *   4. NVFP4 layers only: per-token dynamic FP8 e4m3 codes of x with scale
 *      amax/448 (MoE mixed-precision page sec. 2.1), or with act =
 *      MOE_ACT_NVFP4 per-token NVFP4 codes and block scales;
 *   5. per expert: h = silu(Wg x) * (Wu x) with fp32 accumulation on
 *      dequantized weights (integer formats: fp16 operands, weights rounded
 *      once to fp16 as s*q; NVFP4: exact fp16 operands, scales applied after
 *      the sum; NVFP4 activations in prefill: the block-scaled FP4 MMA on the
 *      codes); NVFP4 layers then quantize each h row to e4m3 (amax/448), or
 *      to NVFP4 with act = MOE_ACT_NVFP4;
 *   6. o = Wd h per row; y[t] = bf16( sum_j w[t][j] * o[row(t,j)] ) summed in
 *      fp32 in ascending j.
 * Integer-format layers run their expert GEMMs on fp16 operands.  A token
 * whose max |x| reaches 2^15 is scaled by a power of two 2^-e (exact) before
 * its fp16 conversion and its gate/up sums by 2^e after, so every finite bf16
 * x is accepted.  The SwiGLU output h is stored in fp16: an |h| that rounds
 * beyond 65504 writes MOE_ERR_RANGE to moe_debug.status (y is then not
 * finite).  NVFP4 layers scale x and h per row and have no such limit.
 * Layers must be all-NVFP4 or all-integer (MOE_ERR_FORMAT).  Matrices packed
 * with MOE_FMT_OUTLIERS add their side lists' residuals to the GEMM sums in
 * the epilogues (fp32, the row's activations as the GEMM reads them); with
 * MOE_ACT_NVFP4 activations such a layer is rejected (MOE_ERR_FORMAT).
 * Errors: MOE_ERR_ARG, MOE_ERR_ALIGN, MOE_ERR_SHAPE, MOE_ERR_FORMAT,
 *   MOE_ERR_WORKSPACE, MOE_ERR_UNSUPPORTED_DEVICE, MOE_ERR_CUDA.
 */
MOE_API moe_status moe_layer_forward(const void* x, int32_t T, const float* router_w, const float* router_b,
                             const moe_weights* w, int32_t k, void* y, void* ws, uint64_t ws_bytes,
                             uint64_t* ws_bytes_out, const moe_debug* dbg, cudaStream_t stream);

/*
 * moe_layer_forward_noalloc -- moe_layer_forward for callers that cannot
 * allocate device memory: code running inside a CUDA graph or an allocator
 * callback, embedded runtimes without cudaMalloc, or hosts whose memory pool
 * must not grow.  (The method on the pages has no counterpart; this is a
 * calling convenience of this library.)
 *
 * The workspace is a fixed array of MOE_NOALLOC_SCRATCH_BYTES (32 MiB) inside
 * this library (a file-scope __device__ array, so every GPU that loads the
 * library holds it until the process exits).  The call allocates nothing and
 * calls no allocating CUDA or library routine; the caller still provides x,
 * the router weights, the packed layer, y and (optionally) dbg, exactly as for
 * moe_layer_forward.  Batches whose workspace (the ws_bytes_out query of
 * moe_layer_forward) exceeds the array are rejected with MOE_ERR_WORKSPACE
 * before anything runs; decode-sized batches of the five reference layers
 * fit (the largest, 64 tokens of the 12288 x 14336 layer, needs ~13 MiB).
 *
 * The first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (with that device current) and caches it; make that
 * first call before any stream capture.  The cached address belongs to the
 * device's current context: a cudaDeviceReset (or any other teardown of the
 * primary context) while the library is in use leaves it stale, so do not
 * reset a device between calls of this entry point.  Every call shares the
 * one array and leaves its contents behind, so calls that overlap on the GPU
 * (other streams, other host threads) race on it: serialize them.  Nothing in
 * the array needs to start at zero: every byte the forward reads is written
 * earlier in the same call.  The array also holds the status word used when
 * dbg or dbg->status is NULL, which the caller cannot read: pass
 * moe_debug.status to see device-side errors (MOE_ERR_TIMEOUT, MOE_ERR_RANGE).
 * Errors: as moe_layer_forward.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (32ull << 20)
MOE_API moe_status moe_layer_forward_noalloc(const void* x, int32_t T, const float* router_w,
                                             const float* router_b, const moe_weights* w, int32_t k, void* y,
                                             const moe_debug* dbg, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */

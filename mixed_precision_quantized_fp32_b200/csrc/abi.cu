// Host side of the C ABI declared in include/moe.h: argument validation,
// workspace carving and the launch sequence of the layer forward.
#include <cstring>

#include "moe_common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kMaxDev = 64;
int g_dev_ok[kMaxDev];  // 0 unknown, 1 sm_100, -1 other (per-process property cache)

moe_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return MOE_ERR_UNSUPPORTED_DEVICE;
  if (g_dev_ok[dev] == 0) {
    // the library ships sm_100a code only, which runs on compute capability 10.0 alone
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_dev_ok[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED_DEVICE;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

bool shape_ok(int E, int H, int F) {
  return E >= 1 && E <= kMaxE && H >= 128 && F >= 128 && H % 128 == 0 && F % 128 == 0 && H <= 32768 &&
         F <= 32768;
}

// Layer kind: 0 = all integer, 1 = all NVFP4, -1 = unknown code or a mix.
// fmt: base formats.
int layer_kind(int E, const uint8_t* fmt) {
  int n_fp4 = 0;
  for (int i = 0; i < 3 * E; ++i) {
    if (!fmt_known(fmt[i])) return -1;
    n_fp4 += fmt[i] == MOE_FMT_NVFP4;
  }
  if (n_fp4 == 0) return 0;
  return n_fp4 == 3 * E ? 1 : -1;
}

struct Plan {
  int chunk_rows;  // rows per work chunk of one expert
  int max_chunks;  // upper bound on the number of chunks
  bool tc;         // tcgen05 expert GEMMs (many rows per expert) or warp-MMA (few rows per expert)
};

// Few rows per expert (decode): chunks of 8 rows on the streaming GEMV (warp
// MMA); an expert with more rows gets several chunks, which read the same weight
// tiles close in time (the second read hits L2).  Many rows per expert
// (prefill): 256-row chunks on the tcgen05 kernel (128 on the block-scaled FP4
// kernel of NVFP4 activations).
Plan make_plan(int T, int k, int E, bool act4) {
  Plan p;
  const long long R = (long long)T * k;
  const long long active = R < E ? R : E;
  const long long avg = active > 0 ? (R + active - 1) / active : 0;
  p.tc = avg > 32 && R >= 256;
  p.chunk_rows = p.tc ? (act4 ? kFp4ChunkRows : kTcChunkRows) : 8;
  p.max_chunks = (int)(E + (R + p.chunk_rows - 1) / p.chunk_rows);
  return p;
}

// Carve the workspace; with base == nullptr only the size is computed.
uint64_t carve(uint8_t* base, int T, int k, int E, int H, int F, bool fp4, bool act4, const Plan& plan,
               Workspace* w) {
  const uint64_t R = (uint64_t)T * k;
  const uint64_t nblk = (R + 1023) / 1024;
  uint64_t pos = 0;
  auto take = [&](uint64_t bytes) -> void* {
    void* p = base ? (void*)(base + pos) : nullptr;
    pos = up256(pos + bytes);
    return p;
  };
  Workspace ws{};
  const int rparts = router_parts(T, H, E);
  ws.logits = (float*)take((uint64_t)(rparts > 1 ? rparts : 1) * T * E * 4);
  if (rparts > 0) ws.wsplit = (__nv_bfloat16*)take((uint64_t)3 * E * H * 2);
  ws.idx = (int32_t*)take(R * 4);
  ws.wts = (float*)take(R * 4);
  ws.counts = (int32_t*)take((uint64_t)E * 4);
  ws.offsets = (int32_t*)take((uint64_t)(E + 1) * 4);
  ws.blk_hist = (int32_t*)take(nblk * E * 4);
  ws.rank = (int32_t*)take(R * 4);
  ws.perm = (int32_t*)take(R * 4);
  ws.inv = (int32_t*)take(R * 4);
  ws.chunks = (int32_t*)take((uint64_t)plan.max_chunks * 3 * 4);
  ws.chunk_count = (int32_t*)take(4);
  ws.status = (int32_t*)take(4);
  if (fp4) {
    ws.xq = (uint8_t*)take((uint64_t)T * H);
    ws.sx = (float*)take((uint64_t)T * 4);
  }
  if (!fp4) ws.xinv = (float*)take(R * 4);
  if (act4) {
    // NVFP4 activations: block scales of x per token; prefill gathers codes + scales,
    // decode gathers fp16 block values
    ws.ldx = (H / 16 + 15) / 16 * 16;
    ws.ldh = (F / 16 + 15) / 16 * 16;
    ws.xsf = (uint8_t*)take((uint64_t)T * ws.ldx);
    if (plan.tc) {
      ws.xs4 = (uint8_t*)take(R * H / 2);
      ws.xsf4 = (uint8_t*)take(R * ws.ldx);
      ws.hs4 = (uint8_t*)take(R * F / 2);
      ws.hsf4 = (uint8_t*)take(R * ws.ldh);
    } else {
      ws.xs = take(R * H * 2);
      ws.hb = take(R * F * 2);
    }
    ws.h = take(R * F * 4);
    ws.sh = (float*)take(R * 4);
  } else {
    ws.xs = take(R * H * 2);
    ws.h = take(R * F * (fp4 ? 4 : 2));
    if (fp4) {
      ws.hb = take(R * F * 2);
      ws.hq = (uint8_t*)take(R * F);
      ws.sh = (float*)take(R * 4);
    }
  }
  ws.o = (float*)take(R * H * 4);
  if (!plan.tc) {
    const int pg = gemv_split((long long)R, E, F, H, 2), pd = gemv_split((long long)R, E, H, F, 1);
    const uint64_t part_g = pg > 1 ? (uint64_t)pg * R * 2 * F : 0, part_d = pd > 1 ? (uint64_t)pd * R * H : 0;
    const uint64_t part = part_g > part_d ? part_g : part_d;
    if (part) ws.part = (float*)take(part * 4);
    ws.counter_len = 2;  // work counters of the gate/up and down GEMVs
    ws.counters = (int32_t*)take((uint64_t)ws.counter_len * 4);
    if (!fp4) {
      ws.xsum = (float*)take(R * (H / 32) * 4);
      ws.hsum = (float*)take(R * (F / 32) * 4);
    }
  }
  if (w) *w = ws;
  return pos;
}

// The caller's format codes split into base formats (what the kernels decode) and
// whether any matrix keeps an outlier side list.  Returns false on an unknown flag.
bool split_fmt(int E, const uint8_t* fmt, uint8_t* base, bool* any_out) {
  *any_out = false;
  for (int i = 0; i < 3 * E; ++i) {
    if (fmt[i] & ~(MOE_FMT_OUTLIERS | 0x1F)) return false;
    base[i] = (uint8_t)fmt_base(fmt[i]);
    *any_out |= fmt_outliers(fmt[i]);
  }
  return true;
}

// Full layout: expert sections (base formats) then the outlier section.
bool full_layout(int E, int H, int F, const uint8_t* fmt, uint64_t* co, uint64_t* so, uint64_t* side,
                 uint64_t* out_sec, uint64_t* total) {
  uint8_t base[3 * kMaxE];
  bool any = false;
  if (!split_fmt(E, fmt, base, &any)) return false;
  uint64_t end = 0;
  if (!layer_layout(E, H, F, base, co, so, &end)) return false;
  *out_sec = outlier_layout(E, H, F, fmt, end, side, total);
  return true;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_pack(const float* W, int32_t e0, int32_t ne, int32_t E, int32_t H, int32_t F,
                               const uint8_t* fmt, void* out, uint64_t out_bytes, uint64_t* bytes_out,
                               uint64_t* code_off, uint64_t* scale_off, cudaStream_t stream) {
  if (!fmt) return MOE_ERR_ARG;
  if (!shape_ok(E, H, F)) return MOE_ERR_SHAPE;
  uint64_t co[3 * kMaxE], so[3 * kMaxE], side[3 * kMaxE], total = 0, out_sec = 0;
  if (!full_layout(E, H, F, fmt, co, so, side, &out_sec, &total)) return MOE_ERR_FORMAT;
  if (code_off) std::memcpy(code_off, co, sizeof(uint64_t) * 3 * E);
  if (scale_off) std::memcpy(scale_off, so, sizeof(uint64_t) * 3 * E);
  if (bytes_out) *bytes_out = total;
  if (!out) return bytes_out ? MOE_OK : MOE_ERR_ARG;
  if (!W) return MOE_ERR_ARG;
  if (e0 < 0 || ne < 0 || e0 > E || ne > E - e0) return MOE_ERR_ARG;
  if (!aligned(out, 256) || !aligned(W, 16)) return MOE_ERR_ALIGN;
  if (out_bytes < total) return MOE_ERR_WORKSPACE;
  const moe_status ds = check_device();
  if (ds != MOE_OK) return ds;
  if (launch_pack(W, e0, ne, E, H, F, fmt, (uint8_t*)out, co, so, out_sec, side, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

extern "C" moe_status moe_layer_forward(const void* x, int32_t T, const float* router_w, const float* router_b,
                                        const moe_weights* w, int32_t k, void* y, void* ws, uint64_t ws_bytes,
                                        uint64_t* ws_bytes_out, const moe_debug* dbg, cudaStream_t stream) {
  if (!w || !w->fmt) return MOE_ERR_ARG;
  const int E = w->E, H = w->H, F = w->F;
  if (!shape_ok(E, H, F)) return MOE_ERR_SHAPE;
  if (T < 0 || k < 1 || k > kMaxK || k > E) return MOE_ERR_SHAPE;
  if ((long long)T * k > (1LL << 20)) return MOE_ERR_SHAPE;
  uint8_t fmt[3 * kMaxE];  // base formats
  bool outliers = false;
  if (!split_fmt(E, w->fmt, fmt, &outliers)) return MOE_ERR_FORMAT;
  const int kind = layer_kind(E, fmt);
  if (kind < 0) return MOE_ERR_FORMAT;
  const bool fp4 = kind == 1;
  if (w->act != MOE_ACT_FP8 && w->act != MOE_ACT_NVFP4) return MOE_ERR_ARG;
  if (w->act == MOE_ACT_NVFP4 && !fp4) return MOE_ERR_FORMAT;  // NVFP4 activations need an NVFP4 layer
  if (w->act == MOE_ACT_NVFP4 && outliers) return MOE_ERR_FORMAT;  // side lists: FP8 activations only
  const bool act4 = w->act == MOE_ACT_NVFP4;
  const Plan plan = make_plan(T, k, E, act4);
  const uint64_t need = carve(nullptr, T, k, E, H, F, fp4, act4, plan, nullptr);
  if (!ws) {
    if (!ws_bytes_out) return MOE_ERR_ARG;
    *ws_bytes_out = need;
    return MOE_OK;
  }
  if (ws_bytes_out) *ws_bytes_out = need;
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !y || !w->packed) return MOE_ERR_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(router_w, 16) || !aligned(w->packed, 256) ||
      !aligned(ws, 256))
    return MOE_ERR_ALIGN;
  uint64_t co[3 * kMaxE], so[3 * kMaxE], side[3 * kMaxE], total = 0, out_sec = 0;
  if (!full_layout(E, H, F, w->fmt, co, so, side, &out_sec, &total)) return MOE_ERR_FORMAT;
  if (w->packed_bytes < total) return MOE_ERR_WORKSPACE;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  const moe_status ds = check_device();
  if (ds != MOE_OK) return ds;

  Workspace wsp;
  carve((uint8_t*)ws, T, k, E, H, F, fp4, act4, plan, &wsp);
  moe_debug d{};
  if (dbg) d = *dbg;
  const __nv_bfloat16* xb = (const __nv_bfloat16*)x;

  cudaEvent_t* ev = d.stage_events;
  auto mark = [&](int i) -> bool { return !ev || cudaEventRecord(ev[i], stream) == cudaSuccess; };
  const uint8_t* packed = (const uint8_t*)w->packed;

  if (!mark(0)) return MOE_ERR_CUDA;
  if (launch_router_topk(xb, router_w, router_b, T, H, E, k, wsp, d.topk_idx, d.topk_w, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(1)) return MOE_ERR_CUDA;
  if (launch_permute(T, k, E, plan.chunk_rows, wsp, d.counts, d.perm, d.inv, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (!mark(2)) return MOE_ERR_CUDA;
  if (act4) {
    if (launch_gather_nvfp4(xb, T, H, k, plan.tc, wsp, d.xq, d.xsb, d.sx, stream) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (launch_gather(xb, T, H, k, fp4, wsp, d.xq, d.sx, stream) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  if (!mark(3)) return MOE_ERR_CUDA;
  int32_t* status = d.status ? d.status : wsp.status;
  auto gemm = [&](bool gateup) -> cudaError_t {
    const GemmHooks hooks{d.test_withhold, d.wait_cycles};
    if (act4 && plan.tc)
      return launch_expert_gemm_fp4(packed, E, H, F, T, k, gateup, wsp, status, d.trace, hooks, stream);
    return plan.tc ? launch_expert_gemm_tc(packed, fmt, E, H, F, T, k, fp4, gateup, wsp, status, d.trace, hooks,
                                           outliers, stream)
                   : launch_expert_gemv(packed, w->packed_bytes, fmt, E, H, F, T * k, k, fp4, gateup,
                                        plan.max_chunks, plan.chunk_rows, wsp, status, gateup ? d.trace : nullptr,
                                        hooks, outliers, stream);
  };
  if (gemm(true) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(4)) return MOE_ERR_CUDA;
  if (act4) {
    if (launch_act_quant_h_nvfp4(T * k, F, plan.tc, wsp, d.hq, d.hsb, d.sh, stream) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (fp4 && launch_act_quant_h(T * k, F, wsp, d.hq, d.sh, stream) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  if (!mark(5)) return MOE_ERR_CUDA;
  if (gemm(false) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(6)) return MOE_ERR_CUDA;
  if (launch_combine(T, k, H, wsp, (__nv_bfloat16*)y, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (!mark(7)) return MOE_ERR_CUDA;
  return MOE_OK;
}

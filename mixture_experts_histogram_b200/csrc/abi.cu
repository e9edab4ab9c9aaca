// The C ABI (include/moe.h): argument checks, the workspace layout, TMA
// descriptors, and the launch sequence of one layer forward.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "moe.h"
#include "ptx.cuh"

namespace moe {

namespace {

// CTAs the router aims for when it splits K for small token counts (B200: 148 SMs).
constexpr int kRouterTargetCtas = 148;

// Expert-GEMM variant. AUTO runs GEMM1 (gate/up) on 2-SM pairs when the
// routed groups average at least kPairMinRows rows (prefill: each weight tile
// then crosses L2 -> SM once per 256 rows; 1.46 vs 1.57 ms at T = 8192) and
// on single CTAs otherwise (decode: a 256-row tile would load twice the
// activation rows for one or two valid ones). GEMM2 (down) runs on single CTAs,
// which measured faster at every size (0.91 vs 0.98 ms at T = 8192).
int g_gemm_variant = MOE_GEMM_AUTO;
constexpr int64_t kPairMinRows = 128;
constexpr int64_t kSwapMinRows = 1;
constexpr int64_t kSwapMaxRows = 16;
// FP8 down GEMM: staged TMA stores of y when its groups average this many rows
// and its K (the intermediate size) is at most this deep.
constexpr int64_t kStoreYMinRows = 128;
constexpr int kStoreYMaxInter = 4096;

// K pieces of the down GEMM over R rows. Its tiles (M tiles x ceil(H/256) N
// tiles) number at most (min(G, R) + R/128) x ceil(H/256); when even that bound
// fills less than half of the GPU (the dense FFN at decode: 16 tiles), each
// tile's K range is split so that about one item runs per SM, every piece at
// least 4 K stages deep, and the pieces' fp32 sums are added afterwards in
// piece order. A function of the configuration and R only (it also sizes the
// workspace); NVFP4 does not split.
int down_k_split(const moe_config& c, int64_t R) {
  if (c.wdtype == MOE_WDTYPE_NVFP4 || R <= 0) return 1;
  const int64_t groups = c.n_experts + c.n_shared;
  const int64_t items = ((groups < R ? groups : R) + R / kTileM) * ceil_div(c.hidden, 256);
  if (2 * items > kRouterTargetCtas) return 1;
  const int64_t stages = c.inter / (c.wdtype == MOE_WDTYPE_FP8_E4M3 ? 128 : 64);
  int64_t ks = kRouterTargetCtas / items;
  if (ks > stages / 4) ks = stages / 4;
  if (ks > 16) ks = 16;
  return ks < 2 ? 1 : (int)ks;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D tensor map over a row-major [outer, inner] array with a 128B-swizzled box.
bool map_2d(CUtensorMap* m, const void* base, bool fp8, uint64_t inner, uint64_t outer, uint32_t box_inner,
            uint32_t box_outer) {
  const int es = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * es};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint8 tensor map without swizzle (NVFP4 codes and scales): rows of
// `inner` bytes, boxes of box_inner bytes x box_outer rows.
bool map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
            uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_config(const moe_config* c, int64_t T) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (c->n_shared < 0 || c->n_shared > 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->wdtype != MOE_WDTYPE_BF16 && c->wdtype != MOE_WDTYPE_FP8_E4M3 && c->wdtype != MOE_WDTYPE_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 || c->inter % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  // NVFP4: the scale tensors' rows (K/16 bytes) must be whole 16-byte TMA strides.
  if (c->wdtype == MOE_WDTYPE_NVFP4 && (c->hidden % 256 || c->inter % 256)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_experts > kMaxExperts || c->top_k > kMaxTopK || c->top_k > c->n_experts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)(c->top_k + c->n_shared) * T >= ((int64_t)1 << 31) - 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)c->n_experts * c->hidden >= ((int64_t)1 << 31) || (int64_t)c->n_experts * c->inter >= ((int64_t)1 << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

int check_weights(const moe_config* c, const moe_weights* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const bool nv = c->wdtype == MOE_WDTYPE_NVFP4;
  const void* need[] = {w->router_w, w->w1, w->w3, w->w2};
  for (const void* p : need) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned(p, 16)) return MOE_ERR_MISALIGNED;
  }
  if ((fp8 || nv) && (!w->s1 || !w->s3 || !w->s2)) return MOE_ERR_INVALID_ARG;
  if (nv && (!w->g1 || !w->g3 || !w->g2)) return MOE_ERR_INVALID_ARG;
  if (nv && (!aligned(w->s1, 16) || !aligned(w->s3, 16) || !aligned(w->s2, 16))) return MOE_ERR_MISALIGNED;
  if (c->n_shared) {
    const void* sh[] = {w->sw1, w->sw3, w->sw2};
    for (const void* p : sh) {
      if (!p) return MOE_ERR_INVALID_ARG;
      if (!aligned(p, 16)) return MOE_ERR_MISALIGNED;
    }
    if ((fp8 || nv) && (!w->ss1 || !w->ss3 || !w->ss2)) return MOE_ERR_INVALID_ARG;
    if (nv && (!w->sg1 || !w->sg3 || !w->sg2)) return MOE_ERR_INVALID_ARG;
    if (nv && (!aligned(w->ss1, 16) || !aligned(w->ss3, 16) || !aligned(w->ss2, 16))) return MOE_ERR_MISALIGNED;
  }
  return MOE_OK;
}

#define CUDA_TRY(expr)                            \
  do {                                            \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// ---- per-kernel profiling ----
constexpr int kProfKernels = 9;
const char* const kProfNames[kProfKernels] = {"router_gemm", "router_topk", "histogram", "scan", "scatter",
                                              "gather",      "gemm1_gate_up_swiglu", "gemm2_down", "combine"};
std::mutex g_prof_mu;
bool g_prof = false;
bool g_prof_ready = false;
int g_prof_recorded = 0;
cudaEvent_t g_ev[kProfKernels + 1];

struct Prof {
  bool on;
  cudaStream_t s;
  int n = 0;
  explicit Prof(cudaStream_t st) : s(st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    on = g_prof;
    if (on && !g_prof_ready) {
      for (auto& e : g_ev) cudaEventCreate(&e);
      g_prof_ready = true;
    }
    if (on) cudaEventRecord(g_ev[0], s);
  }
  void mark() {
    if (on && n < kProfKernels) cudaEventRecord(g_ev[++n], s);
  }
  ~Prof() {
    if (on) g_prof_recorded = n;
  }
};

void router_shape(int E, int* nbox, int* box_rows) {
  const int ep = (int)round_up(E, 16);
  if (ep <= 256) {
    *nbox = 1;
    *box_rows = ep;
  } else {
    *nbox = 2;
    *box_rows = (int)round_up(ceil_div(ep, 2), 16);
  }
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

// Router: logits GEMM + top-k. Writes idx/gate (and optionally logits).
int run_route(const moe_config* c, const WsLayout& L, int64_t T, const void* x, const void* router_w,
              const float* bias, int32_t* idx, float* gate, float* logits, uint8_t* ws, cudaStream_t s, Prof& prof) {
  if (!get_encoder()) return MOE_ERR_CUDA;
  RouterParams rp{};
  rp.T = (int32_t)T;
  rp.H = c->hidden;
  rp.E = c->n_experts;
  router_shape(c->n_experts, &rp.nbox, &rp.box_rows);
  rp.kstages = c->hidden / 64;
  rp.ksplit = (int32_t)L.ksplit;
  rp.partial = reinterpret_cast<float*>(ws + L.logits_part);
  rp.status = reinterpret_cast<int*>(ws + L.status);
  CUtensorMap tx, tw;
  if (!map_2d(&tx, x, false, c->hidden, T, 64, kTileM)) return MOE_ERR_CUDA;
  if (!map_2d(&tw, router_w, false, c->hidden, c->n_experts, 64, rp.box_rows)) return MOE_ERR_CUDA;
  if (rp.ksplit == 1) {
    // One CTA holds each token tile's whole K sum: the top-k runs in its epilogue.
    rp.fused = 1;
    rp.k = c->top_k;
    rp.bias = bias;
    rp.idx = idx;
    rp.gate = gate;
    rp.logits = logits;
    CUDA_TRY(launch_router_gemm(rp, tx, tw, s));
    prof.mark();
    prof.mark();  // no separate top-k kernel
    return MOE_OK;
  }
  CUDA_TRY(launch_router_gemm(rp, tx, tw, s));
  prof.mark();
  TopkParams tp{};
  tp.T = (int32_t)T;
  tp.E = c->n_experts;
  tp.k = c->top_k;
  tp.ksplit = rp.ksplit;
  tp.partial = rp.partial;
  tp.bias = bias;
  tp.idx = idx;
  tp.gate = gate;
  tp.logits = logits;
  CUDA_TRY(launch_topk(tp, s));
  prof.mark();
  return MOE_OK;
}

PermuteParams permute_params(const moe_config* c, const WsLayout& L, int64_t T, const int32_t* idx,
                             const float* gate, uint8_t* ws) {
  PermuteParams pp{};
  pp.T = (int32_t)T;
  pp.E = c->n_experts;
  pp.k = c->top_k;
  pp.S = c->n_shared;
  pp.G = c->n_experts + c->n_shared;
  pp.e0 = 0;
  pp.E_all = c->n_experts;
  pp.sh_t0 = 0;
  pp.sh_t1 = (int32_t)T;
  pp.chunks = (int32_t)L.chunks;
  pp.idx = idx;
  pp.gate = gate;
  pp.chunk_base = reinterpret_cast<int32_t*>(ws + L.chunk_base);
  pp.counts = reinterpret_cast<int32_t*>(ws + L.counts);
  pp.offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  pp.mt_prefix = reinterpret_cast<int32_t*>(ws + L.mt_prefix);
  pp.mp_prefix = reinterpret_cast<int32_t*>(ws + L.mp_prefix);
  pp.perm = reinterpret_cast<int32_t*>(ws + L.perm);
  pp.pos = reinterpret_cast<int32_t*>(ws + L.pos);
  pp.row_gate = gate ? reinterpret_cast<float*>(ws + L.row_gate) : nullptr;
  pp.status = reinterpret_cast<int*>(ws + L.status);
  return pp;
}

// One 256-token chunk (decode): histogram, scan and scatter in one launch; its
// time is reported under "histogram" and the other two marks read zero.
int run_permute(const PermuteParams& pp, cudaStream_t s, Prof& prof) {
  if (pp.chunks == 1) {
    CUDA_TRY(launch_permute_one_chunk(pp, s));
    prof.mark();
    prof.mark();
    prof.mark();
    return MOE_OK;
  }
  CUDA_TRY(launch_histogram(pp, s));
  prof.mark();
  CUDA_TRY(launch_scan(pp, s));
  prof.mark();
  CUDA_TRY(launch_scatter(pp, s));
  prof.mark();
  return MOE_OK;
}

// Process-wide test hooks of the expert GEMMs (moe_debug_inject).
uint64_t g_wait_ns = kWaitLimitNs;
int g_inject = 0;

// Kernel of one expert GEMM: single CTAs, 2-SM pairs, or (FP8) the swapped-
// operand kernel for decode-sized groups. Under AUTO, FP8 layers whose routed
// groups average kSwapMinRows to kSwapMaxRows rows run both GEMMs swapped
// (T = 64: GEMM1 0.580 -> 0.563 ms, GEMM2 0.302 -> 0.282; T = 512 about equal;
// at T <= 8 the single-CTA kernel was 5-8% faster); otherwise GEMM1 runs on
// pairs when the groups average at least kPairMinRows rows and GEMM2 on
// single CTAs.
enum GemmKind { kSingle = 0, kPair = 1, kSwap = 2 };

GemmKind gemm_kind(bool gate_up, int64_t routed_rows, int n_experts, int wdtype) {
  const bool fp8 = wdtype == MOE_WDTYPE_FP8_E4M3;
  const bool nvfp4 = wdtype == MOE_WDTYPE_NVFP4;
  switch (g_gemm_variant) {
    case MOE_GEMM_SINGLE: return kSingle;
    case MOE_GEMM_PAIR: return nvfp4 ? kSingle : kPair;
    case MOE_GEMM_SWAP: return (fp8 || nvfp4) ? kSwap : kSingle;
    default: break;
  }
  if (nvfp4) return routed_rows <= kSwapMaxRows * (int64_t)n_experts ? kSwap : kSingle;
  if (fp8 && routed_rows >= kSwapMinRows * (int64_t)n_experts && routed_rows <= kSwapMaxRows * (int64_t)n_experts)
    return kSwap;
  return (gate_up && routed_rows >= kPairMinRows * (int64_t)n_experts) ? kPair : kSingle;
}

bool amaps(AMaps* a, const void* base, bool fp8, uint64_t inner, uint64_t rows) {
  const uint32_t box_k = fp8 ? 128 : 64;
  return map_2d(&a->rows128, base, fp8, inner, rows, box_k, 128) &&
         map_2d(&a->rows64, base, fp8, inner, rows, box_k, 64) && map_2d(&a->rows32, base, fp8, inner, rows, box_k, 32);
}

// The grouped gate/up GEMM (GEMM1) over R rows of A [R, H] grouped by `offsets`
// (tile prefixes mt / mp for single CTAs / pairs). FP8: a_scale_t [H/128,
// rows_pad]; out = h codes [R, I] with out_scale_t [I/128, rows_pad]. BF16: out
// = h [R, I] bf16. raw: out = fp32 [R, 2I] gate and up sums (no SwiGLU).
int run_gate_up(const moe_config* c, const WsLayout& L, int64_t R, const void* a, const float* a_scale_t,
                const int32_t* offsets, const int32_t* mt, const int32_t* mp, GemmKind kind, const moe_weights* w,
                void* out, float* out_scale_t, bool raw, int* status, cudaStream_t s) {
  const bool pair = kind == kPair;
  if (!get_encoder()) return MOE_ERR_CUDA;
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const int H = c->hidden, I = c->inter, E = c->n_experts, S = c->n_shared;
  const uint32_t box_k = fp8 ? 128 : 64;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  AMaps ma;
  if (c->wdtype == MOE_WDTYPE_NVFP4) {
    // W4A16: bf16 activations; codes [E I, H/2] and scales [E I, H/16] per matrix.
    NvMaps nm;
    bool ok = amaps(&ma, a, false, H, R) && map_u8(&nm.code0, w->w1, H / 2, (uint64_t)E * I, 32, 128) &&
              map_u8(&nm.code1, w->w3, H / 2, (uint64_t)E * I, 32, 128) &&
              map_u8(&nm.scale0, w->s1, H / 16, (uint64_t)E * I, 16, 128) &&
              map_u8(&nm.scale1, w->s3, H / 16, (uint64_t)E * I, 16, 128);
    if (S) {
      ok = ok && map_u8(&nm.scode0, w->sw1, H / 2, I, 32, 128) && map_u8(&nm.scode1, w->sw3, H / 2, I, 32, 128) &&
           map_u8(&nm.sscale0, w->ss1, H / 16, I, 16, 128) && map_u8(&nm.sscale1, w->ss3, H / 16, I, 16, 128);
    } else {
      nm.scode0 = nm.code0;
      nm.scode1 = nm.code1;
      nm.sscale0 = nm.scale0;
      nm.sscale1 = nm.scale1;
    }
    if (!ok) return MOE_ERR_CUDA;
    GemmParams g{};
  g.k_split = 1;
    g.mt_prefix = mt;
    g.offsets = offsets;
    g.G = E + S;
    g.E = E;
    g.K = H;
    g.N = I;
    g.n_tiles = I / 128;
    g.n_fastest = 0;
    g.R = (int32_t)R;
    g.rows_pad = L.rows_pad;
    g.b_scale0 = w->g1;
    g.b_scale1 = w->g3;
    g.bs_scale0 = w->sg1;
    g.bs_scale1 = w->sg3;
    g.out = out;
    g.status = status;
    g.wait_ns = g_wait_ns;
    g.raw_out = raw ? 1 : 0;
    g.inject = g_inject;
    if (kind == kSwap) CUDA_TRY(launch_nvfp4_swap(g, true, sms, ma, nm, s));
    else CUDA_TRY(launch_nvfp4_gemm(g, true, sms, ma, nm, s));
    return MOE_OK;
  }
  CUtensorMap w1, w3, sw1, sw3;
  bool ok = amaps(&ma, a, fp8, H, R) && map_2d(&w1, w->w1, fp8, H, (uint64_t)E * I, box_k, 128) &&
            map_2d(&w3, w->w3, fp8, H, (uint64_t)E * I, box_k, 128);
  if (S) {
    ok = ok && map_2d(&sw1, w->sw1, fp8, H, I, box_k, 128) && map_2d(&sw3, w->sw3, fp8, H, I, box_k, 128);
  } else {
    sw1 = w1;
    sw3 = w3;
  }
  if (!ok) return MOE_ERR_CUDA;
  GemmParams g{};
  g.k_split = 1;
  g.mt_prefix = pair ? mp : mt;
  g.offsets = offsets;
  g.G = E + S;
  g.E = E;
  g.K = H;
  g.N = I;
  g.n_tiles = I / 128;
  g.n_fastest = 0;
  g.R = (int32_t)R;
  g.rows_pad = L.rows_pad;
  g.a_scale = fp8 ? a_scale_t : nullptr;
  g.b_scale0 = w->s1;
  g.b_scale1 = w->s3;
  g.bs_scale0 = w->ss1;
  g.bs_scale1 = w->ss3;
  g.out = out;
  g.out_scale = fp8 ? out_scale_t : nullptr;
  g.row_gate = nullptr;
  g.status = status;
  g.wait_ns = g_wait_ns;
  g.raw_out = raw ? 1 : 0;
  g.inject = g_inject;
  if (kind == kSwap && fp8) CUDA_TRY(launch_gemm_swap(g, true, sms, ma, w1, w3, sw1, sw3, s));
  else CUDA_TRY(launch_gemm1(g, fp8, pair, sms, ma, w1, w3, sw1, sw3, s));
  return MOE_OK;
}

// The grouped down GEMM (GEMM2): y [R, H] bf16 = row_gate[r] * (A W2_g^T) for
// A [R, I] (FP8: codes with a_scale_t [I/128, rows_pad]); row_gate may be null (1).
int run_down(const moe_config* c, const WsLayout& L, int64_t R, const void* a, const float* a_scale_t,
             const int32_t* offsets, const int32_t* mt, const int32_t* mp, GemmKind kind, const moe_weights* w,
             const float* row_gate, void* y, uint8_t* ws, int* status, cudaStream_t s) {
  const bool pair = kind == kPair;
  if (!get_encoder()) return MOE_ERR_CUDA;
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const int H = c->hidden, I = c->inter, E = c->n_experts, S = c->n_shared;
  const uint32_t box_k = fp8 ? 128 : 64;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  AMaps ma;
  if (c->wdtype == MOE_WDTYPE_NVFP4) {
    NvMaps nm;
    bool ok = amaps(&ma, a, false, I, R) && map_u8(&nm.code0, w->w2, I / 2, (uint64_t)E * H, 32, 256) &&
              map_u8(&nm.scale0, w->s2, I / 16, (uint64_t)E * H, 16, 256);
    if (S) {
      ok = ok && map_u8(&nm.scode0, w->sw2, I / 2, H, 32, 256) && map_u8(&nm.sscale0, w->ss2, I / 16, H, 16, 256);
    } else {
      nm.scode0 = nm.code0;
      nm.sscale0 = nm.scale0;
    }
    nm.code1 = nm.code0;
    nm.scode1 = nm.scode0;
    nm.scale1 = nm.scale0;
    nm.sscale1 = nm.sscale0;
    if (!ok) return MOE_ERR_CUDA;
    GemmParams g{};
  g.k_split = 1;
    g.mt_prefix = mt;
    g.offsets = offsets;
    g.G = E + S;
    g.E = E;
    g.K = I;
    g.N = H;
    g.n_tiles = (int32_t)ceil_div(H, 256);
    g.n_fastest = 1;
    g.R = (int32_t)R;
    g.rows_pad = L.rows_pad;
    g.b_scale0 = w->g2;
    g.b_scale1 = w->g2;
    g.bs_scale0 = w->sg2;
    g.bs_scale1 = w->sg2;
    g.out = y;
    g.row_gate = row_gate;
    g.status = status;
    g.wait_ns = g_wait_ns;
    g.inject = g_inject;
    if (kind == kSwap) CUDA_TRY(launch_nvfp4_swap(g, false, sms, ma, nm, s));
    else CUDA_TRY(launch_nvfp4_gemm(g, false, sms, ma, nm, s));
    return MOE_OK;
  }
  CUtensorMap w2, w2h, sw2, sw2h;
  bool ok = amaps(&ma, a, fp8, I, R) && map_2d(&w2, w->w2, fp8, I, (uint64_t)E * H, box_k, 256) &&
            map_2d(&w2h, w->w2, fp8, I, (uint64_t)E * H, box_k, 128);
  if (S) {
    ok = ok && map_2d(&sw2, w->sw2, fp8, I, H, box_k, 256) && map_2d(&sw2h, w->sw2, fp8, I, H, box_k, 128);
  } else {
    sw2 = w2;
    sw2h = w2h;
  }
  if (!ok) return MOE_ERR_CUDA;
  GemmParams g{};
  g.k_split = 1;
  g.mt_prefix = pair ? mp : mt;
  g.offsets = offsets;
  g.G = E + S;
  g.E = E;
  g.K = I;
  g.N = H;
  g.n_tiles = (int32_t)ceil_div(H, 256);
  g.n_fastest = 1;
  g.R = (int32_t)R;
  g.rows_pad = L.rows_pad;
  g.a_scale = fp8 ? a_scale_t : nullptr;
  g.b_scale0 = w->s2;
  g.b_scale1 = w->s2;
  g.bs_scale0 = w->ss2;
  g.bs_scale1 = w->ss2;
  g.out = y;
  g.out_scale = nullptr;
  g.row_gate = row_gate;
  g.status = status;
  g.wait_ns = g_wait_ns;
  g.raw_out = 0;
  g.inject = g_inject;
  g.k_split = down_k_split(*c, L.R);
  if (g.k_split > 1) g.part = reinterpret_cast<float*>(ws + L.part);
  if (kind == kSwap && fp8) {
    CUDA_TRY(launch_gemm_swap(g, false, sms, ma, w2, w2h, sw2, sw2h, s));
  } else {
    // FP8 groups of a tile or more on average, with a short K loop per tile: the
    // y tiles leave through shared memory and TMA stores (T = 8192: 0.90 -> 0.84
    // ms). The one fewer pipeline stage this costs made smaller layers (T = 8:
    // 0.074 -> 0.078 ms) and the dense FFN's 13,824-deep K loop (0.459 -> 0.472)
    // slower.
    CUtensorMap ym;
    const bool store_y =
        fp8 && g.k_split == 1 && R >= kStoreYMinRows * (int64_t)g.G && c->inter <= kStoreYMaxInter;
    if (store_y && !map_2d(&ym, y, false, H, (uint64_t)R, 64, 32)) return MOE_ERR_CUDA;
    CUDA_TRY(launch_gemm2(g, fp8, pair, sms, ma, w2, w2h, sw2, sw2h, store_y ? &ym : nullptr, s));
  }
  if (g.k_split > 1)
    CUDA_TRY(launch_split_reduce(g.part, g.k_split, R, H, offsets + g.G, row_gate, status, y, s));
  return MOE_OK;
}

// gather + GEMM1 + GEMM2 for a permutation already in the workspace; y [R, H] bf16.
// routed_rows: the routed rows this call expects (k T on one GPU), which
// decides whether the gate/up GEMM runs on 2-SM pairs.
int run_experts(const moe_config* c, const WsLayout& L, int64_t T, const void* x, const moe_weights* w,
                const int32_t* pos, void* y, uint8_t* ws, cudaStream_t s, Prof& prof, int64_t routed_rows) {
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const int S = c->n_shared;
  const int64_t R = L.R;
  GatherParams gp{};
  gp.T = (int32_t)T;
  gp.H = c->hidden;
  gp.S = c->top_k + S;
  gp.rows_pad = L.rows_pad;
  gp.x = static_cast<const uint16_t*>(x);
  gp.pos = pos;
  gp.xp = ws + L.xp;
  gp.sxp = fp8 ? reinterpret_cast<float*>(ws + L.sxp) : nullptr;
  gp.scale_row_major = 0;
  CUDA_TRY(launch_gather(gp, fp8, s));
  prof.mark();

  const int32_t* offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  const int32_t* mt = reinterpret_cast<const int32_t*>(ws + L.mt_prefix);
  const int32_t* mp = reinterpret_cast<const int32_t*>(ws + L.mp_prefix);
  int* status = reinterpret_cast<int*>(ws + L.status);
  const GemmKind k1 = gemm_kind(true, routed_rows, c->n_experts, c->wdtype);
  const GemmKind k2 = gemm_kind(false, routed_rows, c->n_experts, c->wdtype);
  int rc = run_gate_up(c, L, R, ws + L.xp, reinterpret_cast<const float*>(ws + L.sxp), offsets, mt, mp, k1, w,
                       ws + L.h, reinterpret_cast<float*>(ws + L.sh), false, status, s);
  if (rc != MOE_OK) return rc;
  prof.mark();
  rc = run_down(c, L, R, ws + L.h, reinterpret_cast<const float*>(ws + L.sh), offsets, mt, mp, k2, w,
                reinterpret_cast<const float*>(ws + L.row_gate), y, ws, status, s);
  if (rc != MOE_OK) return rc;
  prof.mark();
  return MOE_OK;
}

int run_combine(const moe_config* c, int64_t T, const void* y, const int32_t* pos, void* out, cudaStream_t s,
                Prof& prof) {
  CombineParams cp{};
  cp.T = (int32_t)T;
  cp.H = c->hidden;
  cp.S = c->top_k + c->n_shared;
  cp.y = static_cast<const uint16_t*>(y);
  cp.pos = pos;
  cp.out = static_cast<uint16_t*>(out);
  CUDA_TRY(launch_combine(cp, s));
  prof.mark();
  return MOE_OK;
}

int check_ws(const moe_config* c, int64_t T, void* ws, size_t ws_bytes, WsLayout* L) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_MISALIGNED;
  *L = ws_layout(*c, T, kRouterTargetCtas);
  if (ws_bytes < L->total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

}  // namespace

std::atomic<uint64_t> g_launches{0};

cudaError_t counted_launch(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

WsLayout ws_layout(const moe_config& c, int64_t T, int target_ctas) {
  WsLayout L{};
  const int S = c.n_shared, k = c.top_k, E = c.n_experts, G = E + S;
  const bool fp8 = c.wdtype == MOE_WDTYPE_FP8_E4M3;
  const int64_t es = fp8 ? 1 : 2;
  L.T = T;
  L.R = (int64_t)(k + S) * T;
  L.rows_pad = round_up(L.R, kTileM) + 2 * kTileM;  // a 256-row pair tile may start at the last row
  L.chunks = ceil_div(T > 0 ? T : 1, kHistChunk);
  const int64_t m_tiles = ceil_div(T > 0 ? T : 1, kTileM);
  int64_t ks = target_ctas / m_tiles;
  const int64_t kmax = c.hidden / 64 < 16 ? c.hidden / 64 : 16;
  L.ksplit = ks < 1 ? 1 : (ks > kmax ? kmax : ks);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (size_t)round_up((int64_t)(off + (bytes ? bytes : 1)), 1024);
    return o;
  };
  L.status = take(kStatusBytes);  // status word, first-timeout record, debug counters
  L.idx = take((size_t)T * k * 4);
  L.gate = take((size_t)T * k * 4);
  L.logits_part = take((size_t)L.ksplit * T * E * 4);
  L.chunk_base = take((size_t)E * L.chunks * 4);
  L.counts = take((size_t)G * 4);
  L.offsets = take((size_t)(G + 1) * 4);
  L.mt_prefix = take((size_t)(G + 1) * 4);
  L.mp_prefix = take((size_t)(G + 1) * 4);
  L.perm = take((size_t)L.R * 4);
  L.pos = take((size_t)T * (k + S) * 4);
  L.row_gate = take((size_t)L.R * 4);
  L.xp = take((size_t)L.R * c.hidden * es);
  L.sxp = take(fp8 ? (size_t)(c.hidden / 128) * L.rows_pad * 4 : 0);
  L.h = take((size_t)L.R * c.inter * es);
  L.sh = take(fp8 ? (size_t)(c.inter / 128) * L.rows_pad * 4 : 0);
  L.y = take((size_t)L.R * c.hidden * 2);
  const int k2 = down_k_split(c, L.R);
  L.part = take(k2 > 1 ? (size_t)k2 * L.R * c.hidden * 4 : 0);
  L.x_stage = take((size_t)T * c.hidden * 2);
  L.out_stage = take((size_t)T * c.hidden * 2);
  L.total = off;
  return L;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_workspace_bytes(const moe_config* cfg, int64_t T, size_t* bytes) {
  const int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = ws_layout(*cfg, T, kRouterTargetCtas).total;
  return MOE_OK;
}

int moe_forward(const moe_config* cfg, int64_t T, const void* x, const moe_weights* w, void* out, int32_t* topk_idx,
                float* topk_w, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if ((rc = check_weights(cfg, w)) != MOE_OK) return rc;
  if (!x || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return MOE_ERR_MISALIGNED;
  if ((topk_idx == nullptr) != (topk_w == nullptr)) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  Prof prof(s);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(ws + L.idx);
  float* gate = topk_w ? topk_w : reinterpret_cast<float*>(ws + L.gate);
  if ((rc = run_route(cfg, L, T, x, w->router_w, w->router_bias, idx, gate, nullptr, ws, s, prof)) != MOE_OK) return rc;
  const PermuteParams pp = permute_params(cfg, L, T, idx, gate, ws);
  if ((rc = run_permute(pp, s, prof)) != MOE_OK) return rc;
  if ((rc = run_experts(cfg, L, T, x, w, pp.pos, ws + L.y, ws, s, prof, (int64_t)cfg->top_k * T)) != MOE_OK) return rc;
  return run_combine(cfg, T, ws + L.y, pp.pos, out, s, prof);
}

int moe_forward_host_async(const moe_config* cfg, int64_t T, const void* x_host, const moe_weights* w,
                           void* out_host, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t bytes = (size_t)T * cfg->hidden * 2;
  CUDA_TRY(cudaMemcpyAsync(ws + L.x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
  rc = moe_forward(cfg, T, ws + L.x_stage, w, ws + L.out_stage, nullptr, nullptr, workspace, workspace_bytes, stream);
  if (rc != MOE_OK) return rc;
  CUDA_TRY(cudaMemcpyAsync(out_host, ws + L.out_stage, bytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

int moe_forward_host(const moe_config* cfg, int64_t T, const void* x_host, const moe_weights* w, void* out_host,
                     void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  const int rc = moe_forward_host_async(cfg, T, x_host, w, out_host, workspace, workspace_bytes, stream);
  if (rc != MOE_OK || T == 0) return rc;
  CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

int moe_forward_ep_partial(const moe_config* cfg, int64_t T, const void* x, const moe_weights* w, int32_t e0,
                           int32_t e1, int64_t shared_t0, int64_t shared_t1, float* partial, int32_t* topk_idx,
                           float* topk_w, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (e0 < 0 || e1 <= e0 || e1 > cfg->n_experts) return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared && (shared_t0 < 0 || shared_t1 < shared_t0 || shared_t1 > T)) return MOE_ERR_INVALID_ARG;
  moe_config lc = *cfg;  // this rank's routed experts only
  lc.n_experts = e1 - e0;
  if ((rc = check_weights(&lc, w)) != MOE_OK) return rc;
  if (!x || !partial) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(partial, 16)) return MOE_ERR_MISALIGNED;
  if ((topk_idx == nullptr) != (topk_w == nullptr)) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  Prof prof(s);
  prof.on = false;
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(ws + L.idx);
  float* gate = topk_w ? topk_w : reinterpret_cast<float*>(ws + L.gate);
  if ((rc = run_route(cfg, L, T, x, w->router_w, w->router_bias, idx, gate, nullptr, ws, s, prof)) != MOE_OK) return rc;
  PermuteParams pp = permute_params(&lc, L, T, idx, gate, ws);
  pp.e0 = e0;
  pp.E_all = cfg->n_experts;
  pp.sh_t0 = cfg->n_shared ? (int32_t)shared_t0 : 0;
  pp.sh_t1 = cfg->n_shared ? (int32_t)shared_t1 : 0;
  if ((rc = run_permute(pp, s, prof)) != MOE_OK) return rc;
  // The gate/up GEMM's variant follows the rows a routed group gets on average.
  const int64_t routed_rows = (int64_t)cfg->top_k * T * lc.n_experts / cfg->n_experts;
  if ((rc = run_experts(&lc, L, T, x, w, pp.pos, ws + L.y, ws, s, prof, routed_rows)) != MOE_OK) return rc;
  CUDA_TRY(launch_ep_partial(T, cfg->hidden, cfg->top_k + cfg->n_shared, ws + L.y, pp.pos, partial, s));
  return MOE_OK;
}

int moe_route(const moe_config* cfg, int64_t T, const void* x, const void* router_w, const float* router_bias,
              int32_t* topk_idx, float* topk_w, float* logits, void* workspace, size_t workspace_bytes,
              moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (!x || !router_w || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16)) return MOE_ERR_MISALIGNED;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  Prof prof(s);
  prof.on = false;
  return run_route(cfg, L, T, x, router_w, router_bias, topk_idx, topk_w, logits, ws, s, prof);
}

int moe_quantize_act(int64_t T, int32_t hidden, const void* x, uint8_t* q, float* s, moe_stream_t stream) {
  if (T < 0 || hidden <= 0 || hidden % 128 || !x || !q || !s) return MOE_ERR_INVALID_ARG;
  if (T > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return MOE_ERR_MISALIGNED;
  if (T == 0) return MOE_OK;
  GatherParams gp{};
  gp.T = (int32_t)T;
  gp.H = hidden;
  gp.S = 1;
  gp.rows_pad = T;
  gp.x = static_cast<const uint16_t*>(x);
  gp.pos = nullptr;
  gp.xp = q;
  gp.sxp = s;
  gp.scale_row_major = 1;
  CUDA_TRY(launch_gather(gp, true, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

int moe_permute(const moe_config* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* pos, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (!topk_idx || !counts || !offsets || !perm || !pos) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  if (T == 0) {
    const int G = cfg->n_experts + cfg->n_shared;
    CUDA_TRY(cudaMemsetAsync(counts, 0, (size_t)G * 4, s));
    CUDA_TRY(cudaMemsetAsync(offsets, 0, (size_t)(G + 1) * 4, s));
    return MOE_OK;
  }
  PermuteParams pp = permute_params(cfg, L, T, topk_idx, nullptr, ws);
  pp.counts = counts;
  pp.offsets = offsets;
  pp.perm = perm;
  pp.pos = pos;
  Prof prof(s);
  prof.on = false;
  return run_permute(pp, s, prof);
}

int moe_experts(const moe_config* cfg, int64_t T, const void* x, const int32_t* topk_idx, const float* topk_w,
                const moe_weights* w, void* y, int32_t* pos, void* workspace, size_t workspace_bytes,
                moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if ((rc = check_weights(cfg, w)) != MOE_OK) return rc;
  if (!x || !topk_idx || !topk_w || !y || !pos) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return MOE_ERR_MISALIGNED;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  Prof prof(s);
  prof.on = false;
  PermuteParams pp = permute_params(cfg, L, T, topk_idx, topk_w, ws);
  pp.pos = pos;
  if ((rc = run_permute(pp, s, prof)) != MOE_OK) return rc;
  return run_experts(cfg, L, T, x, w, pos, y, ws, s, prof, (int64_t)cfg->top_k * T);
}

int moe_combine(const moe_config* cfg, int64_t T, const void* y, const int32_t* pos, void* out, moe_stream_t stream) {
  int rc = check_config(cfg, T);
  if (rc != MOE_OK) return rc;
  if (!y || !pos || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16)) return MOE_ERR_MISALIGNED;
  if (T == 0) return MOE_OK;
  Prof prof(reinterpret_cast<cudaStream_t>(stream));
  prof.on = false;
  return run_combine(cfg, T, y, pos, out, reinterpret_cast<cudaStream_t>(stream), prof);
}

int moe_grouped_gemm(const moe_config* cfg, int stage, int64_t R, const int32_t* offsets, const void* a,
                     const float* a_scale, const moe_weights* w, const float* row_gate, void* out, float* out_scale,
                     void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_config(cfg, 0);
  if (rc != MOE_OK) return rc;
  if ((rc = check_weights(cfg, w)) != MOE_OK) return rc;
  if (stage != MOE_STAGE_GATE_UP && stage != MOE_STAGE_GATE_UP_RAW && stage != MOE_STAGE_DOWN)
    return MOE_ERR_INVALID_ARG;
  if (R < 0 || !offsets || !a || !out) return MOE_ERR_INVALID_ARG;
  if (R >= ((int64_t)1 << 31) - 512) return MOE_ERR_UNSUPPORTED_SHAPE;
  const bool fp8 = cfg->wdtype == MOE_WDTYPE_FP8_E4M3;
  if (fp8 && !a_scale) return MOE_ERR_INVALID_ARG;
  if (fp8 && stage == MOE_STAGE_GATE_UP && !out_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(out, 16) || !aligned(offsets, 4)) return MOE_ERR_MISALIGNED;
  // The workspace of moe_forward for ceil(R / (top_k + n_shared)) tokens holds
  // every scratch buffer this needs.
  const int64_t T = ceil_div(R, cfg->top_k + cfg->n_shared);
  if ((rc = check_config(cfg, T)) != MOE_OK) return rc;
  WsLayout L;
  if ((rc = check_ws(cfg, T, workspace, workspace_bytes, &L)) != MOE_OK) return rc;
  if (R == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status);
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusBytes, s));
  const int G = cfg->n_experts + cfg->n_shared;
  int32_t* mt = reinterpret_cast<int32_t*>(ws + L.mt_prefix);
  int32_t* mp = reinterpret_cast<int32_t*>(ws + L.mp_prefix);
  CUDA_TRY(launch_tile_prefix(offsets, G, (int32_t)R, mt, mp, status, s));
  if (stage == MOE_STAGE_DOWN) {
    float* a_t = reinterpret_cast<float*>(ws + L.sh);
    if (fp8) CUDA_TRY(launch_scale_transpose(a_scale, a_t, R, cfg->inter / 128, L.rows_pad, true, s));
    return run_down(cfg, L, R, a, a_t, offsets, mt, mp, gemm_kind(false, R, G, cfg->wdtype), w, row_gate, out, ws,
                    status, s);
  }
  float* a_t = reinterpret_cast<float*>(ws + L.sxp);
  float* o_t = reinterpret_cast<float*>(ws + L.sh);
  if (fp8) CUDA_TRY(launch_scale_transpose(a_scale, a_t, R, cfg->hidden / 128, L.rows_pad, true, s));
  const bool raw = stage == MOE_STAGE_GATE_UP_RAW;
  rc = run_gate_up(cfg, L, R, a, a_t, offsets, mt, mp, gemm_kind(true, R, G, cfg->wdtype), w, out, o_t, raw, status,
                   s);
  if (rc != MOE_OK) return rc;
  if (fp8 && !raw) CUDA_TRY(launch_scale_transpose(o_t, out_scale, R, cfg->inter / 128, L.rows_pad, false, s));
  return MOE_OK;
}

int moe_read_status_detail(const void* workspace, moe_stream_t stream, int* detail) {
  if (!workspace || !detail) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v[4] = {0, 0, 0, 0};
  CUDA_TRY(cudaMemcpyAsync(v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaStreamSynchronize(s));
  for (int i = 0; i < 4; ++i) detail[i] = v[i];
  return MOE_OK;
}

int moe_debug_inject(int what, uint64_t wait_limit_ns) {
  if (what != MOE_INJECT_NONE && what != MOE_INJECT_GEMM_NO_LOADS) return MOE_ERR_INVALID_ARG;
  g_inject = what;
  g_wait_ns = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
  return MOE_OK;
}

int moe_read_status(const void* workspace, moe_stream_t stream, int* device_status) {
  if (!workspace || !device_status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  CUDA_TRY(cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaStreamSynchronize(s));
  *device_status = v;
  return MOE_OK;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_BAD_INDEX: return "expert index out of range (pair skipped)";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_MISALIGNED: return "misaligned buffer";
    default: return "unknown status";
  }
}

int moe_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof = enable != 0;
  g_prof_recorded = 0;
  return MOE_OK;
}

int moe_profile_read(float* ms, int n, int* n_out) {
  if (!ms || !n_out) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  const int m = g_prof_recorded;
  *n_out = m;
  if (m == 0) return MOE_OK;
  CUDA_TRY(cudaEventSynchronize(g_ev[m]));
  for (int i = 0; i < m && i < n; ++i) CUDA_TRY(cudaEventElapsedTime(&ms[i], g_ev[i], g_ev[i + 1]));
  return MOE_OK;
}

const char* moe_profile_kernel_name(int i) { return (i >= 0 && i < kProfKernels) ? kProfNames[i] : ""; }

int moe_set_gemm_variant(int variant) {
  if (variant != MOE_GEMM_AUTO && variant != MOE_GEMM_SINGLE && variant != MOE_GEMM_PAIR && variant != MOE_GEMM_SWAP)
    return MOE_ERR_INVALID_ARG;
  g_gemm_variant = variant;
  return MOE_OK;
}

int moe_launch_count(uint64_t* n) {
  if (!n) return MOE_ERR_INVALID_ARG;
  *n = g_launches.load(std::memory_order_relaxed);
  return MOE_OK;
}

int moe_device_sm_count(int* sms) {
  if (!sms) return MOE_ERR_INVALID_ARG;
  const int n = sm_count();
  if (n <= 0) return MOE_ERR_CUDA;
  *sms = n;
  return MOE_OK;
}

}  // extern "C"

// The C ABI (include/moe.h): argument checks, the workspace layout, TMA
// descriptors, and the launch sequence of one layer forward.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "moe.h"

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

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_config(const moe_config* c, int64_t T) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (c->n_shared < 0 || c->n_shared > 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->wdtype != MOE_WDTYPE_BF16 && c->wdtype != MOE_WDTYPE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 || c->inter % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_experts > kMaxExperts || c->top_k > kMaxTopK || c->top_k > c->n_experts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)(c->top_k + c->n_shared) * T >= ((int64_t)1 << 31) - 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)c->n_experts * c->hidden >= ((int64_t)1 << 31) || (int64_t)c->n_experts * c->inter >= ((int64_t)1 << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

int check_weights(const moe_config* c, const moe_weights* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const void* need[] = {w->router_w, w->w1, w->w3, w->w2};
  for (const void* p : need) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned(p, 16)) return MOE_ERR_MISALIGNED;
  }
  if (fp8 && (!w->s1 || !w->s3 || !w->s2)) return MOE_ERR_INVALID_ARG;
  if (c->n_shared) {
    const void* sh[] = {w->sw1, w->sw3, w->sw2};
    for (const void* p : sh) {
      if (!p) return MOE_ERR_INVALID_ARG;
      if (!aligned(p, 16)) return MOE_ERR_MISALIGNED;
    }
    if (fp8 && (!w->ss1 || !w->ss3 || !w->ss2)) return MOE_ERR_INVALID_ARG;
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

struct Maps {
  CUtensorMap x, wr, w1, w3, sw1, sw3, w2, sw2, w2h, sw2h;  // w2h/sw2h: 128-row boxes
  AMaps xp, h;                                           // GEMM1 / GEMM2 activations
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

// gather + GEMM1 + GEMM2 for a permutation already in the workspace; y [R, H] bf16.
int run_experts(const moe_config* c, const WsLayout& L, int64_t T, const void* x, const moe_weights* w,
                const int32_t* pos, void* y, uint8_t* ws, cudaStream_t s, Prof& prof) {
  if (!get_encoder()) return MOE_ERR_CUDA;
  const bool fp8 = c->wdtype == MOE_WDTYPE_FP8_E4M3;
  const int H = c->hidden, I = c->inter, E = c->n_experts, S = c->n_shared;
  const int es = fp8 ? 1 : 2;
  const uint32_t box_k = 128 / es;
  const int64_t R = L.R;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  const bool pair = g_gemm_variant == MOE_GEMM_PAIR;  // GEMM2 (and the maps it shares)
  const bool pair1 = pair || (g_gemm_variant == MOE_GEMM_AUTO && (int64_t)c->top_k * T >= kPairMinRows * E);

  GatherParams gp{};
  gp.T = (int32_t)T;
  gp.H = H;
  gp.S = c->top_k + S;
  gp.rows_pad = L.rows_pad;
  gp.x = static_cast<const uint16_t*>(x);
  gp.pos = pos;
  gp.xp = ws + L.xp;
  gp.sxp = fp8 ? reinterpret_cast<float*>(ws + L.sxp) : nullptr;
  gp.scale_row_major = 0;
  CUDA_TRY(launch_gather(gp, fp8, s));
  prof.mark();

  Maps m;
  auto amaps = [&](AMaps* a, const void* base, uint64_t inner) {
    return map_2d(&a->rows128, base, fp8, inner, R, box_k, 128) && map_2d(&a->rows64, base, fp8, inner, R, box_k, 64) &&
           map_2d(&a->rows32, base, fp8, inner, R, box_k, 32);
  };
  bool ok = amaps(&m.xp, ws + L.xp, H) && amaps(&m.h, ws + L.h, I) &&
            map_2d(&m.w1, w->w1, fp8, H, (uint64_t)E * I, box_k, 128) &&
            map_2d(&m.w3, w->w3, fp8, H, (uint64_t)E * I, box_k, 128) &&
            map_2d(&m.w2, w->w2, fp8, I, (uint64_t)E * H, box_k, 256) &&
            map_2d(&m.w2h, w->w2, fp8, I, (uint64_t)E * H, box_k, 128);
  if (S) {
    ok = ok && map_2d(&m.sw1, w->sw1, fp8, H, I, box_k, 128) && map_2d(&m.sw3, w->sw3, fp8, H, I, box_k, 128) &&
         map_2d(&m.sw2, w->sw2, fp8, I, H, box_k, 256) && map_2d(&m.sw2h, w->sw2, fp8, I, H, box_k, 128);
  } else {
    m.sw1 = m.w1;
    m.sw3 = m.w3;
    m.sw2 = m.w2;
    m.sw2h = m.w2h;
  }
  if (!ok) return MOE_ERR_CUDA;

  GemmParams g1{};
  g1.mt_prefix = reinterpret_cast<const int32_t*>(ws + (pair1 ? L.mp_prefix : L.mt_prefix));
  g1.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  g1.G = E + S;
  g1.E = E;
  g1.K = H;
  g1.N = I;
  g1.n_tiles = I / 128;
  g1.n_fastest = 0;
  g1.R = (int32_t)R;
  g1.rows_pad = L.rows_pad;
  g1.a_scale = fp8 ? reinterpret_cast<const float*>(ws + L.sxp) : nullptr;
  g1.b_scale0 = w->s1;
  g1.b_scale1 = w->s3;
  g1.bs_scale0 = w->ss1;
  g1.bs_scale1 = w->ss3;
  g1.out = ws + L.h;
  g1.out_scale = fp8 ? reinterpret_cast<float*>(ws + L.sh) : nullptr;
  g1.row_gate = nullptr;
  g1.status = reinterpret_cast<int*>(ws + L.status);
  CUDA_TRY(launch_gemm1(g1, fp8, pair1, sms, m.xp, m.w1, m.w3, m.sw1, m.sw3, s));
  prof.mark();

  GemmParams g2 = g1;
  g2.mt_prefix = reinterpret_cast<const int32_t*>(ws + (pair ? L.mp_prefix : L.mt_prefix));
  g2.K = I;
  g2.N = H;
  g2.n_tiles = (int32_t)ceil_div(H, 256);
  g2.n_fastest = 1;
  g2.a_scale = fp8 ? reinterpret_cast<const float*>(ws + L.sh) : nullptr;
  g2.b_scale0 = w->s2;
  g2.b_scale1 = w->s2;
  g2.bs_scale0 = w->ss2;
  g2.bs_scale1 = w->ss2;
  g2.out = y;
  g2.out_scale = nullptr;
  g2.row_gate = reinterpret_cast<const float*>(ws + L.row_gate);
  CUDA_TRY(launch_gemm2(g2, fp8, pair, sms, m.h, m.w2, m.w2h, m.sw2, m.sw2h, s));
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
  L.status = take(16384);  // status word, first-timeout record, debug counters
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
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16384, s));
  Prof prof(s);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(ws + L.idx);
  float* gate = topk_w ? topk_w : reinterpret_cast<float*>(ws + L.gate);
  if ((rc = run_route(cfg, L, T, x, w->router_w, w->router_bias, idx, gate, nullptr, ws, s, prof)) != MOE_OK) return rc;
  const PermuteParams pp = permute_params(cfg, L, T, idx, gate, ws);
  if ((rc = run_permute(pp, s, prof)) != MOE_OK) return rc;
  if ((rc = run_experts(cfg, L, T, x, w, pp.pos, ws + L.y, ws, s, prof)) != MOE_OK) return rc;
  return run_combine(cfg, T, ws + L.y, pp.pos, out, s, prof);
}

int moe_forward_host(const moe_config* cfg, int64_t T, const void* x_host, const moe_weights* w, void* out_host,
                     void* workspace, size_t workspace_bytes, moe_stream_t stream) {
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
  CUDA_TRY(cudaStreamSynchronize(s));
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
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16384, s));
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
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16384, s));
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
  CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16384, s));
  Prof prof(s);
  prof.on = false;
  PermuteParams pp = permute_params(cfg, L, T, topk_idx, topk_w, ws);
  pp.pos = pos;
  if ((rc = run_permute(pp, s, prof)) != MOE_OK) return rc;
  return run_experts(cfg, L, T, x, w, pos, y, ws, s, prof);
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
  if (variant != MOE_GEMM_AUTO && variant != MOE_GEMM_SINGLE && variant != MOE_GEMM_PAIR) return MOE_ERR_INVALID_ARG;
  g_gemm_variant = variant;
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

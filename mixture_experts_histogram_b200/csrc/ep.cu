// Expert parallelism: one rank's share of the layer, and the rank-ordered sum
// of the ranks' partial outputs.
//
// The pages deploy the layer at TP = EP = 8 (StepFun "Step-5 minimal
// inference" README, deployment section: 44 of the 352 routed experts on each
// of 8 GPUs, tokens replicated over the group) and add the ranks' partial
// results in rank order with FP32 accumulation (same README, "Long-output
// stability"). Here:
//   - every rank routes every token over all E experts (the same kernels on
//     the same inputs give the same routing on every rank);
//   - rank r computes its routed experts [e0, e1) and the shared expert for its
//     own slice of tokens [t0, t1) (the shared expert is replicated and its
//     rows split by token, so every rank does about the same work);
//   - its partial output p_r[t] = sum over its (token, slot) rows of the
//     gate-weighted expert rows, in fp32 in slot order (no bf16 rounding);
//   - out[t] = bf16(p_0[t] + p_1[t] + ... + p_{R-1}[t]), fp32 in rank order
//     (moe_ep_reduce), over whichever token range the caller reduces (all
//     tokens for an all-reduce, the rank's slice for a reduce-scatter).
// The partial buffers that moe_ep_reduce reads may be this GPU's memory (the
// partials gathered by a collective) or peers' memory mapped into this
// device's address space (plain loads over NVLink).
#include <cuda_bf16.h>

#include "common.cuh"
#include "moe.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxRanks = 16;

struct ReduceParams {
  const float* part[kMaxRanks];
  int32_t n_ranks, H;
  int64_t t0;
  uint16_t* out;
};

// One CTA per token: p[t] = sum over slots j (in order) of y[pos[t, j]],
// rows with pos < 0 left out (another rank's experts or shared slice).
template <int kMaxSlots>
__global__ void __launch_bounds__(kThreads) ep_partial_kernel(int32_t H, int32_t S, const uint16_t* __restrict__ y,
                                                              const int32_t* __restrict__ pos,
                                                              float* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = blockIdx.x;
  int32_t rows[kMaxSlots];
#pragma unroll
  for (int j = 0; j < kMaxSlots; ++j) rows[j] = j < S ? pos[t * S + j] : -1;
  const int nvec = H / 8;
  for (int c = threadIdx.x; c < nvec; c += kThreads) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxSlots; ++j) {
      if (rows[j] < 0) continue;
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(y + (int64_t)rows[j] * H) + c);
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
    float4* o = reinterpret_cast<float4*>(part + t * H) + 2 * c;
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// One CTA per token of [t0, t0 + gridDim.x): the ranks' fp32 partials added in
// rank order, rounded once to bf16. Each thread owns 8 columns per step; the
// loads of every rank are issued before the sum.
__global__ void __launch_bounds__(kThreads) ep_reduce_kernel(const ReduceParams p) {
  const int64_t t = p.t0 + blockIdx.x;
  const int nvec = p.H / 8;
  for (int c = threadIdx.x; c < nvec; c += kThreads) {
    float4 v[kMaxRanks][2];
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r) {
      if (r < p.n_ranks) {
        const float4* src = reinterpret_cast<const float4*>(p.part[r] + t * p.H) + 2 * c;
        v[r][0] = __ldcs(src);
        v[r][1] = __ldcs(src + 1);
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r) {
      if (r < p.n_ranks) {
        acc[0] += v[r][0].x;
        acc[1] += v[r][0].y;
        acc[2] += v[r][0].z;
        acc[3] += v[r][0].w;
        acc[4] += v[r][1].x;
        acc[5] += v[r][1].y;
        acc[6] += v[r][1].z;
        acc[7] += v[r][1].w;
      }
    }
    uint4 o;
    __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) ob[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    reinterpret_cast<uint4*>(p.out + t * p.H)[c] = o;
  }
}

}  // namespace

cudaError_t launch_ep_partial(int64_t T, int32_t H, int32_t S, const void* y, const int32_t* pos, float* part,
                              cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const uint16_t* yy = static_cast<const uint16_t*>(y);
  if (S <= 9) return launch_pdl(ep_partial_kernel<9>, dim3((unsigned)T), dim3(kThreads), 0, s, 1, H, S, yy, pos, part);
  return launch_pdl(ep_partial_kernel<kMaxTopK + 1>, dim3((unsigned)T), dim3(kThreads), 0, s, 1, H, S, yy, pos, part);
}

}  // namespace moe

using namespace moe;

extern "C" int moe_ep_reduce(int32_t n_ranks, const float* const* partials, int64_t T, int32_t hidden, int64_t t0,
                             int64_t t1, void* out, moe_stream_t stream) {
  if (n_ranks < 1 || !partials || !out || T < 0 || hidden <= 0 || hidden % 128) return MOE_ERR_INVALID_ARG;
  if (n_ranks > kMaxRanks) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (t0 < 0 || t1 < t0 || t1 > T) return MOE_ERR_INVALID_ARG;
  if (t1 - t0 > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(out) & 15) return MOE_ERR_MISALIGNED;
  ReduceParams p{};
  for (int r = 0; r < n_ranks; ++r) {
    if (!partials[r]) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(partials[r]) & 15) return MOE_ERR_MISALIGNED;
    p.part[r] = partials[r];
  }
  if (t1 == t0) return MOE_OK;
  p.n_ranks = n_ranks;
  p.H = hidden;
  p.t0 = t0;
  p.out = static_cast<uint16_t*>(out);
  ep_reduce_kernel<<<(unsigned)(t1 - t0), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return counted_launch(cudaGetLastError()) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

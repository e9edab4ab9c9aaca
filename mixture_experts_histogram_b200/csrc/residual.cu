// The steps on either side of the MoE layer on the fp32 residual stream
// (NeMo "Step-5-Preview" page, "Full-Depth H100 Benchmark" table: FP32 norms
// and residuals; "Attention and Precision": FP32 residual stream).
//
// rmsnorm: x[t] = bf16(r[t] / sqrt(mean(r[t]^2) + eps) * w), everything in fp32
//   (IEEE sqrt and division), one rounding to bf16: the layer's input.
// combine + residual: r_out[t] = r[t] + sum_j y[pos[t, j]], the layer's expert
//   rows summed in fp32 in slot order (routed slots, then the shared expert)
//   and added to the residual in fp32, with no bf16 rounding of the layer output.
#include <cuda_bf16.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) s += red[i];  // every thread, same order
  return s;
}

// One CTA per token; each thread owns float4 pieces of the row.
__global__ void __launch_bounds__(kThreads) rmsnorm_kernel(int32_t H, const float* __restrict__ r,
                                                           const float* __restrict__ w, float eps,
                                                           uint16_t* __restrict__ x) {
  __shared__ float red[kThreads / 32];
  const int64_t t = blockIdx.x;
  const int nvec = H / 4;
  const float4* row = reinterpret_cast<const float4*>(r + t * H);
  float ss = 0.0f;
  for (int c = threadIdx.x; c < nvec; c += kThreads) {
    const float4 v = row[c];
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
  }
  const float total = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(total / (float)H + eps);
  const float4* wv = reinterpret_cast<const float4*>(w);
  uint2* out = reinterpret_cast<uint2*>(x + t * H);
  for (int c = threadIdx.x; c < nvec; c += kThreads) {
    const float4 v = row[c], g = wv[c];
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * inv * g.x, v.y * inv * g.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * inv * g.z, v.w * inv * g.w);
    out[c] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
  }
}

// One CTA per token; each thread owns 8 columns per step: the token's expert
// rows (bf16, 16-byte loads) summed in fp32 in slot order, then added to the
// residual (fp32). r_out may be r.
template <int kMaxSlots>
__global__ void __launch_bounds__(kThreads) combine_residual_kernel(int32_t H, int32_t S, const uint16_t* y,
                                                                    const int32_t* pos, const float* r,
                                                                    float* r_out) {
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
      const uint4 v = reinterpret_cast<const uint4*>(y + (int64_t)rows[j] * H)[c];
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
    const float4* rr = reinterpret_cast<const float4*>(r + t * H) + 2 * c;
    float4* ro = reinterpret_cast<float4*>(r_out + t * H) + 2 * c;
    const float4 a = rr[0], b = rr[1];
    ro[0] = make_float4(a.x + acc[0], a.y + acc[1], a.z + acc[2], a.w + acc[3]);
    ro[1] = make_float4(b.x + acc[4], b.y + acc[5], b.z + acc[6], b.w + acc[7]);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_rmsnorm(int64_t T, int32_t hidden, const float* residual, const float* weight, float eps,
                           void* x_bf16, moe_stream_t stream) {
  if (T < 0 || hidden <= 0 || hidden % 128 || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (T > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!residual || !weight || !x_bf16) return MOE_ERR_INVALID_ARG;
  if (!aligned16(residual) || !aligned16(weight) || !aligned16(x_bf16)) return MOE_ERR_MISALIGNED;
  rmsnorm_kernel<<<(unsigned)T, kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      hidden, residual, weight, eps, static_cast<uint16_t*>(x_bf16));
  return counted_launch(cudaGetLastError()) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_combine_residual(const moe_config* cfg, int64_t T, const void* y, const int32_t* pos,
                                    const float* residual, float* residual_out, moe_stream_t stream) {
  if (!cfg || T < 0) return MOE_ERR_INVALID_ARG;
  if (cfg->hidden <= 0 || cfg->hidden % 128 || cfg->top_k <= 0 || cfg->n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (cfg->top_k > kMaxTopK || cfg->n_shared > 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!y || !pos || !residual || !residual_out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(residual) || !aligned16(residual_out)) return MOE_ERR_MISALIGNED;
  const int S = cfg->top_k + cfg->n_shared;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (S <= 9)
    combine_residual_kernel<9><<<(unsigned)T, kThreads, 0, s>>>(cfg->hidden, S, static_cast<const uint16_t*>(y), pos,
                                                               residual, residual_out);
  else
    combine_residual_kernel<kMaxTopK + 1><<<(unsigned)T, kThreads, 0, s>>>(
        cfg->hidden, S, static_cast<const uint16_t*>(y), pos, residual, residual_out);
  return counted_launch(cudaGetLastError()) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

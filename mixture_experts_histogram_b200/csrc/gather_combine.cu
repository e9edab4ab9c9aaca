// Row movement around the expert GEMMs.
//
// gather: copies each token's activation row into the k+S expert rows it
// feeds (pos[t, j]), so every expert group's rows are contiguous for the
// GEMM's TMA loads. With FP8 expert storage it also quantises the row on the
// way, per 1x128 block: scale = blockmax/448 (IEEE fp32 division), codes =
// E4M3(x / scale) rounded to nearest even with saturation; an all-zero block
// gets scale 1 and zero codes (block-scaled FP8 of the StepFun "Step-5 minimal
// inference" README). Scales go to a [H/128, rows] array so a GEMM tile's 128
// row scales for one K block are contiguous.
//
// combine: out[t] = sum over slots j of y[pos[t, j]] (gate already applied by
// the down-projection epilogue), in fp32 in slot order (routed slots, then the
// shared expert), rounded once to bf16; 16-byte loads and stores (README,
// "Long-output stability": fixed-order fp32 accumulation of partial results).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) gather_bf16_kernel(const GatherParams p) {
  const int64_t t = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(p.x + t * p.H);
  const int nvec = p.H / 8;
  for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
    const uint4 v = src[c];
    for (int j = 0; j < p.S; ++j) {
      const int64_t row = p.pos ? p.pos[t * p.S + j] : t;
      if (row >= 0) reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.xp) + row * p.H)[c] = v;
    }
  }
}

// One warp per 128-element block; each lane quantises 4 consecutive values.
__global__ void __launch_bounds__(256) gather_fp8_kernel(const GatherParams p) {
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nblk = p.H / 128;
  for (int kb = warp; kb < nblk; kb += 8) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p.x + t * p.H + kb * 128 + lane * 4);
    const __nv_bfloat162 b01 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 b23 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 f01 = __bfloat1622float2(b01), f23 = __bfloat1622float2(b23);
    float amax = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float s = 1.0f;
    uint32_t codes = 0;
    if (amax > 0.0f) {
      s = __fdiv_rn(amax, 448.0f);
      const float2 q01 = make_float2(__fdiv_rn(f01.x, s), __fdiv_rn(f01.y, s));
      const float2 q23 = make_float2(__fdiv_rn(f23.x, s), __fdiv_rn(f23.y, s));
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(q01, __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(q23, __NV_SATFINITE, __NV_E4M3);
      codes = lo | (hi << 16);
    }
    for (int j = 0; j < p.S; ++j) {
      const int64_t row = p.pos ? p.pos[t * p.S + j] : t;
      if (row < 0) continue;
      *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(p.xp) + row * p.H + kb * 128 + lane * 4) = codes;
      if (lane == 0) {
        if (p.scale_row_major) p.sxp[row * nblk + kb] = s;
        else p.sxp[(int64_t)kb * p.rows_pad + row] = s;
      }
    }
  }
}

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  const int64_t t = blockIdx.x;
  const int nvec = p.H / 8;
  for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < p.S; ++j) {
      const int64_t r = p.pos[t * p.S + j];
      if (r < 0) continue;
      const uint4 v = reinterpret_cast<const uint4*>(p.y + r * p.H)[c];
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
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

cudaError_t launch_gather(const GatherParams& p, bool fp8, cudaStream_t s) {
  if (p.T == 0) return cudaSuccess;
  if (fp8) gather_fp8_kernel<<<(unsigned)p.T, 256, 0, s>>>(p);
  else gather_bf16_kernel<<<(unsigned)p.T, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  if (p.T == 0) return cudaSuccess;
  combine_kernel<<<(unsigned)p.T, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace moe

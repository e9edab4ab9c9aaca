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
  pdl_wait();
  pdl_trigger();
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

// One half-warp per 128-element block: each lane loads 8 bf16 (16 bytes),
// the half-warp reduces the block's amax, and each lane stores its 8 codes
// (8 bytes) to every destination row. Six CTAs' registers per SM leave room
// for the next kernel's CTAs to start under programmatic dependent launch.
template <int kMaxSlots>
__global__ void __launch_bounds__(256, 6) gather_fp8_kernel(const GatherParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int half = lane / 16, hl = lane % 16;
  const int nblk = p.H / 128;
  int32_t rows[kMaxSlots];  // destination rows (< 2^31)
#pragma unroll
  for (int j = 0; j < kMaxSlots; ++j) rows[j] = j < p.S ? (p.pos ? p.pos[t * p.S + j] : (int32_t)t) : -1;
  // Two blocks per half-warp and pass, both loads issued before either is used.
  for (int kb00 = 2 * warp; kb00 < nblk; kb00 += 32) {
    uint4 raws[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int kb = kb00 + 16 * u + half;
      raws[u] = kb < nblk ? __ldcs(reinterpret_cast<const uint4*>(p.x + t * p.H + kb * 128) + hl)
                          : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int kb = kb00 + 16 * u + half;
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raws[u]);
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(b[i]);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      float s = 1.0f;
      uint2 codes = make_uint2(0, 0);
      if (amax > 0.0f) {
        s = __fdiv_rn(amax, 448.0f);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s)),
                                          __NV_SATFINITE, __NV_E4M3);
        codes = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
      }
      if (kb >= nblk) continue;
#pragma unroll
      for (int j = 0; j < kMaxSlots; ++j) {
        const int64_t row = rows[j];
        if (row < 0) continue;
        *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.xp) + row * p.H + kb * 128 + hl * 8) = codes;
        if (hl == 0) {
          if (p.scale_row_major) p.sxp[row * nblk + kb] = s;
          else p.sxp[(int64_t)kb * p.rows_pad + row] = s;
        }
      }
    }
  }
}

// One CTA per token. Each thread owns 8 output columns per step; the token's
// row indices live in registers and every row's 16-byte chunk is loaded before
// the sum, so up to kMaxSlots independent loads are in flight per thread.
template <int kMaxSlots>
__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = blockIdx.x;
  const int nvec = p.H / 8;
  int32_t rows[kMaxSlots];
#pragma unroll
  for (int j = 0; j < kMaxSlots; ++j) rows[j] = j < p.S ? p.pos[t * p.S + j] : -1;
  for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
    uint4 v[kMaxSlots];
#pragma unroll
    for (int j = 0; j < kMaxSlots; ++j)
      if (rows[j] >= 0) v[j] = __ldcs(reinterpret_cast<const uint4*>(p.y + (int64_t)rows[j] * p.H) + c);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxSlots; ++j) {  // slot order: routed slots, then the shared expert
      if (rows[j] < 0) continue;
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
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

// Split-K down GEMM: one CTA per row; each thread sums 8 columns of the k_split
// fp32 piece sums in piece order, applies the row's gate and rounds once.
__global__ void __launch_bounds__(256) split_reduce_kernel(const float* __restrict__ part, int32_t k_split, int64_t R,
                                                           int32_t N, const int32_t* __restrict__ rows_end,
                                                           const float* __restrict__ row_gate,
                                                           const int* __restrict__ status, uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int64_t r = blockIdx.x;
  if (*status != 0) return;
  const int64_t end = *rows_end;
  if (r >= end) return;
  const float g = row_gate ? row_gate[r] : 1.0f;
  for (int c = threadIdx.x; c < N / 8; c += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int kp = 0; kp < k_split; ++kp) {
      const float4* src = reinterpret_cast<const float4*>(part + ((int64_t)kp * R + r) * N) + 2 * c;
      const float4 a = __ldcs(src), b = __ldcs(src + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    uint4 o;
    __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) ob[i] = __floats2bfloat162_rn(acc[2 * i] * g, acc[2 * i + 1] * g);
    reinterpret_cast<uint4*>(y + r * N)[c] = o;
  }
}

// FP8 activation scales between a caller's row-major [R, nb] layout and the
// grouped GEMMs' transposed [nb, rows_pad] one (the stage entry point).
__global__ void __launch_bounds__(256) scale_transpose_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                                              int64_t R, int32_t nb, int64_t rows_pad,
                                                              int32_t to_transposed) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * nb) return;
  const int64_t r = i / nb, kb = i % nb;
  if (to_transposed) dst[kb * rows_pad + r] = src[i];
  else dst[i] = src[kb * rows_pad + r];
}

}  // namespace

cudaError_t launch_scale_transpose(const float* src, float* dst, int64_t R, int32_t nb, int64_t rows_pad,
                                   bool to_transposed, cudaStream_t s) {
  const int64_t n = R * nb;
  if (n == 0) return cudaSuccess;
  scale_transpose_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(src, dst, R, nb, rows_pad, to_transposed ? 1 : 0);
  return counted_launch(cudaGetLastError());
}

cudaError_t launch_split_reduce(const float* part, int32_t k_split, int64_t R, int32_t N, const int32_t* rows_end,
                                const float* row_gate, const int* status, void* y, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  return launch_pdl(split_reduce_kernel, dim3((unsigned)R), dim3(256), 0, s, 1, part, k_split, R, N, rows_end, row_gate,
                    status, static_cast<uint16_t*>(y));
}

cudaError_t launch_gather(const GatherParams& p, bool fp8, cudaStream_t s) {
  if (p.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)p.T), block(256);
  if (fp8 && p.S <= 9) return launch_pdl(gather_fp8_kernel<9>, grid, block, 0, s, 1, p);
  if (fp8) return launch_pdl(gather_fp8_kernel<kMaxTopK + 1>, grid, block, 0, s, 1, p);
  return launch_pdl(gather_bf16_kernel, grid, block, 0, s, 1, p);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  if (p.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)p.T), block(256);
  if (p.S <= 9) return launch_pdl(combine_kernel<9>, grid, block, 0, s, 1, p);
  return launch_pdl(combine_kernel<kMaxTopK + 1>, grid, block, 0, s, 1, p);
}

}  // namespace moe

// Pieces shared by the grouped expert GEMM kernels (FP8/BF16 and NVFP4): the
// work-item decode of the persistent schedule, the SwiGLU arithmetic, the NVFP4
// weight expansion, and the warp-uniform bounded wait.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

struct Item {
  int g, n, row0, end;  // group, N tile, first row of the tile, end of the group's rows
};

// n_fastest: consecutive items walk the N tiles of one row tile (they share A
// rows); otherwise they walk the M tiles of one weight tile (they share B).
__device__ __forceinline__ Item decode_item(int item, int n_tiles, int G, int tile_rows, const int* s_mt,
                                            const int* s_off, bool n_fastest) {
  const int q = item / n_tiles;
  int lo = 0, hi = G;  // s_mt[lo] <= q < s_mt[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mt[mid] <= q) lo = mid;
    else hi = mid;
  }
  Item it;
  it.g = lo;
  const int mtiles = s_mt[lo + 1] - s_mt[lo];
  const int local = item - n_tiles * s_mt[lo];
  it.n = n_fastest ? local % n_tiles : local / mtiles;
  it.row0 = s_off[lo] + (n_fastest ? local / n_tiles : local % mtiles) * tile_rows;
  it.end = s_off[lo + 1];
  return it;
}

// silu(g) * u with silu(g) = g / (1 + e^-g): an exponential and a fast divide.
// The cheaper form (g/2)(1 + tanh(g/2)) through the hardware tanh loses most
// of its relative accuracy to cancellation for negative g and doubled the
// largest per-token error of the layer, so it is not used.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Eight weights of one row: a 32-bit word of E2M1 codes (input 2i in the low
// nibble of byte i) and the E4M3 scale of their 16-input block -> four bf16x2
// words (element 2i in the low half). e2m1 -> f16 and e4m3 -> f16 are exact,
// the f16 product (<= 5 significant bits, magnitude in [2^-10, 2688]) is exact,
// and so is its conversion to bf16.
__device__ __forceinline__ uint4 expand8(uint32_t codes, uint32_t scale_byte) {
  uint32_t s2, p0, p1, p2, p3;
  const uint16_t sb = (uint16_t)(scale_byte * 0x0101u);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(sb));
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(p0), "=r"(p1), "=r"(p2), "=r"(p3)
      : "r"(codes));
  auto to_bf16x2 = [&](uint32_t h2) {
    uint32_t prod, out;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(prod) : "r"(h2), "r"(s2));
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&prod));
    out = pack_bf16x2(f.x, f.y);
    return out;
  };
  return make_uint4(to_bf16x2(p0), to_bf16x2(p1), to_bf16x2(p2), to_bf16x2(p3));
}

// Bounded wait by every lane, with a warp-uniform verdict (keeps the warp
// converged for the .sync.aligned TMEM loads that follow).
template <bool kCluster>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag,
                                          int site, int progress, uint64_t limit_ns) {
  const bool ok = kCluster ? mbar_wait_cluster(bar, parity, status, abort_flag, site, progress, limit_ns)
                           : mbar_wait(bar, parity, status, abort_flag, site, progress, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace moe

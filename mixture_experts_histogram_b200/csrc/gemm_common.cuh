// Pieces shared by the grouped expert GEMM kernels (FP8/BF16 and NVFP4): the
// work-item decode of the persistent schedule, the SwiGLU arithmetic, and the
// warp-uniform bounded wait.
#pragma once

#include <cuda_bf16.h>

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

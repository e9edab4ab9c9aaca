// Token -> expert histogram, its exclusive scan, and the gather indices (the
// "critical MoE primitives" of the StepFun "Step-5 minimal inference" README,
// opening section). Groups 0..E-1 are the routed experts; group E is the
// shared expert, which takes every token (NeMo "Step-5-Preview" page: one
// shared expert, here treated as one more group of the grouped GEMMs).
//
// Row order is fixed and independent of scheduling: groups in index order,
// and inside a group the tokens ascend. Atomics only count; they never decide
// where a row goes:
//   1. histogram: one CTA per 256-token chunk counts its (token, slot) pairs
//      per expert in shared memory -> chunk_base[e][chunk].
//   2. scan: one CTA scans chunk counts per expert (one warp per expert), then
//      the expert totals -> counts, offsets, and the per-group prefixes of
//      128-row tiles and 256-row pair tiles the grouped GEMMs schedule from;
//      chunk_base becomes each chunk's base inside its group.
//   3. scatter: each warp ranks its 32 tokens' pairs in (token, slot) order
//      with __match_any_sync (equal experts in one 32-pair round rank by lane),
//      warps are then offset by an exclusive scan over the CTA's 8 warps, and
//      rows are written: perm[row] = token, pos[token, slot] = row,
//      row_gate[row] = gate.
// With a single chunk (T <= 256, decode) one CTA runs the three steps in one
// launch, with block barriers between them.
#include "common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void histogram_block(const PermuteParams& p, int chunk, int* cnt) {
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t t0 = (int64_t)chunk * kHistChunk;
  const int64_t ntok = min((int64_t)kHistChunk, (int64_t)p.T - t0);
  const int64_t npairs = ntok * p.k;
  const int32_t* idx = p.idx + t0 * p.k;
  for (int64_t i = threadIdx.x; i < npairs; i += blockDim.x) {
    const int eg = idx[i], e = eg - p.e0;
    if (eg < 0 || eg >= p.E_all) latch_status(p.status, MOE_ERR_BAD_INDEX);
    else if (e >= 0 && e < p.E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) p.chunk_base[(int64_t)e * p.chunks + chunk] = cnt[e];
}

__global__ void __launch_bounds__(256) histogram_kernel(const PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[kMaxExperts];
  histogram_block(p, blockIdx.x, cnt);
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

__device__ __forceinline__ void scan_block(const PermuteParams& p, int* cnt_s) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
  // per-expert exclusive scan over chunks (bases relative to the expert's
  // first row). Up to 32 chunks (T <= 8192): a warp loads the counts of 12
  // experts before scanning any, so their load latencies overlap.
  if (p.chunks <= 32) {
    constexpr int kBatch = 12;
    for (int e0 = warp; e0 < p.E; e0 += nwarps * kBatch) {
      int v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int e = e0 + nwarps * j;
        v[j] = (e < p.E && lane < p.chunks) ? p.chunk_base[(int64_t)e * p.chunks + lane] : 0;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int e = e0 + nwarps * j;
        const int incl = warp_inclusive_scan(v[j], lane);
        if (e < p.E && lane < p.chunks) p.chunk_base[(int64_t)e * p.chunks + lane] = incl - v[j];
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (e < p.E && lane == 0) cnt_s[e] = total;
      }
    }
  } else {
    for (int e = warp; e < p.E; e += nwarps) {
      int running = 0;
      int32_t* row = p.chunk_base + (int64_t)e * p.chunks;
      for (int c0 = 0; c0 < p.chunks; c0 += 32) {
        const int c = c0 + lane;
        const int v = c < p.chunks ? row[c] : 0;
        const int incl = warp_inclusive_scan(v, lane);
        if (c < p.chunks) row[c] = running + incl - v;
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) cnt_s[e] = running;
    }
  }
  if (threadIdx.x == 0 && p.S) cnt_s[p.E] = p.sh_t1 - p.sh_t0;
  __syncthreads();
  // offsets and M-tile prefix over the G groups
  if (warp == 0) {
    int run_off = 0, run_mt = 0, run_mp = 0;
    for (int g0 = 0; g0 < p.G; g0 += 32) {
      const int g = g0 + lane;
      const int c = g < p.G ? cnt_s[g] : 0;
      const int mt = (c + kTileM - 1) / kTileM;
      const int mp = (c + 2 * kTileM - 1) / (2 * kTileM);
      const int ic = warp_inclusive_scan(c, lane);
      const int im = warp_inclusive_scan(mt, lane);
      const int ip = warp_inclusive_scan(mp, lane);
      if (g < p.G) {
        p.counts[g] = c;
        p.offsets[g] = run_off + ic - c;
        p.mt_prefix[g] = run_mt + im - mt;
        p.mp_prefix[g] = run_mp + ip - mp;
      }
      run_off += __shfl_sync(0xffffffffu, ic, 31);
      run_mt += __shfl_sync(0xffffffffu, im, 31);
      run_mp += __shfl_sync(0xffffffffu, ip, 31);
    }
    if (lane == 0) {
      p.offsets[p.G] = run_off;
      p.mt_prefix[p.G] = run_mt;
      p.mp_prefix[p.G] = run_mp;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(1024) scan_kernel(const PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt_s[kMaxExperts + 1];
  scan_block(p, cnt_s);
}

// off_s: the G + 1 group offsets in shared memory, filled by the caller before
// the block barrier inside.
__device__ __forceinline__ void scatter_block(const PermuteParams& p, int chunk, int (*wcnt)[kMaxExperts],
                                              const int* off_s) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t tw0 = (int64_t)chunk * kHistChunk + warp * 32;  // this warp's first token
  int rank[kMaxTopK];
  int ekeep[kMaxTopK];
  float gkeep[kMaxTopK];
  // The pairs' experts and gates, all loaded before they are used.
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    ekeep[r] = -1;
    gkeep[r] = 0.0f;
    if (r < p.k) {
      const int pidx = r * 32 + lane;
      const int64_t t = tw0 + pidx / p.k;
      const int j = pidx % p.k;
      if (t < p.T) {
        ekeep[r] = p.idx[t * p.k + j] - p.e0;  // this call's group; others are left out
        if (p.row_gate) gkeep[r] = p.gate[t * p.k + j];
      }
    }
  }
  for (int i = threadIdx.x; i < 8 * kMaxExperts; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();

  // Pass 1: ranks inside the warp, pairs taken in (token, slot) order, 32 per round.
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    rank[r] = 0;
    if (r < p.k) {
      int e = ekeep[r];
      if (e < 0 || e >= p.E || e + p.e0 >= p.E_all) e = -1;
      const int key = e >= 0 ? e : (0x40000000 + lane);  // unmatched sentinel for empty lanes
      const unsigned m = __match_any_sync(0xffffffffu, key);
      const int rk = __popc(m & ((1u << lane) - 1u));
      const int prev = e >= 0 ? wcnt[warp][e] : 0;
      __syncwarp();
      if (e >= 0 && rk == 0) wcnt[warp][e] = prev + __popc(m);
      __syncwarp();
      rank[r] = prev + rk;
      ekeep[r] = e;
    }
  }
  __syncthreads();
  // Pass 2: warp offsets per expert, on top of this chunk's base (the group's
  // first row plus the chunk's base inside the group).
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int run = off_s[e] + p.chunk_base[(int64_t)e * p.chunks + chunk];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int v = wcnt[w][e];
      wcnt[w][e] = run;
      run += v;
    }
  }
  __syncthreads();
  // Pass 3: write the rows.
  const int S = p.S + p.k;
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < p.k) {
      const int pidx = r * 32 + lane;
      const int64_t t = tw0 + pidx / p.k;
      const int j = pidx % p.k;
      if (t < p.T) {
        const int e = ekeep[r];
        if (e >= 0) {
          const int row = wcnt[warp][e] + rank[r];
          p.perm[row] = (int32_t)t;
          p.pos[t * S + j] = row;
          if (p.row_gate) p.row_gate[row] = gkeep[r];
        } else {
          p.pos[t * S + j] = -1;  // a pair left out (another rank's expert, or a bad index)
        }
      }
    }
  }
  // The shared expert's rows: token order, for tokens [sh_t0, sh_t1).
  if (p.S) {
    const int64_t t = (int64_t)chunk * kHistChunk + threadIdx.x;
    if (t < p.T) {
      if (t >= p.sh_t0 && t < p.sh_t1) {
        const int row = off_s[p.E] + (int)(t - p.sh_t0);
        p.perm[row] = (int32_t)t;
        p.pos[t * S + p.k] = row;
        if (p.row_gate) p.row_gate[row] = 1.0f;
      } else {
        p.pos[t * S + p.k] = -1;
      }
    }
  }
}

__global__ void __launch_bounds__(256, 1) scatter_kernel(const PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wcnt[8][kMaxExperts];
  __shared__ int off_s[kMaxExperts + 2];
  for (int g = threadIdx.x; g <= p.G; g += blockDim.x) off_s[g] = p.offsets[g];
  scatter_block(p, blockIdx.x, wcnt, off_s);
}

// T <= 256: the three steps in one CTA. With a single chunk the per-expert
// chunk scan is the identity, so the counts come straight from the shared
// histogram, the block scans them over the groups, and the scatter follows.
__global__ void __launch_bounds__(256, 1) permute_one_chunk_kernel(const PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wcnt[8][kMaxExperts];  // scatter; rows 0-1 first hold the expert counts
  __shared__ int off_s[kMaxExperts + 2];
  __shared__ int wtot[3][8];
  int* cnt = &wcnt[0][0];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int npairs = p.T * p.k;
  for (int i = threadIdx.x; i < npairs; i += blockDim.x) {
    const int eg = p.idx[i], e = eg - p.e0;
    if (eg < 0 || eg >= p.E_all) latch_status(p.status, MOE_ERR_BAD_INDEX);
    else if (e >= 0 && e < p.E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // Exclusive scans over the G groups of their rows, 128-row tiles and 256-row
  // pair tiles: kPer consecutive groups per thread, a warp scan of the
  // threads' sums, then the warps' totals.
  constexpr int kPer = (kMaxExperts + 1 + 255) / 256;
  int c[kPer], mt[kPer], mp[kPer];
  int sc = 0, sm = 0, sp = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int g = threadIdx.x * kPer + u;
    c[u] = g < p.E ? cnt[g] : (g < p.G ? p.sh_t1 - p.sh_t0 : 0);  // group E: the shared expert
    mt[u] = (c[u] + kTileM - 1) / kTileM;
    mp[u] = (c[u] + 2 * kTileM - 1) / (2 * kTileM);
    sc += c[u];
    sm += mt[u];
    sp += mp[u];
  }
  const int ic = warp_inclusive_scan(sc, lane);
  const int im = warp_inclusive_scan(sm, lane);
  const int ip = warp_inclusive_scan(sp, lane);
  if (lane == 31) {
    wtot[0][warp] = ic;
    wtot[1][warp] = im;
    wtot[2][warp] = ip;
  }
  __syncthreads();
  int run_off = ic - sc, run_mt = im - sm, run_mp = ip - sp;
  for (int w = 0; w < warp; ++w) {
    run_off += wtot[0][w];
    run_mt += wtot[1][w];
    run_mp += wtot[2][w];
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int g = threadIdx.x * kPer + u;
    if (g < p.G) {
      p.counts[g] = c[u];
      p.offsets[g] = run_off;
      p.mt_prefix[g] = run_mt;
      p.mp_prefix[g] = run_mp;
      off_s[g] = run_off;
      if (g < p.E) p.chunk_base[g] = 0;  // the one chunk starts at its group's first row
    } else if (g == p.G) {
      p.offsets[g] = run_off;
      p.mt_prefix[g] = run_mt;
      p.mp_prefix[g] = run_mp;
      off_s[g] = run_off;
    }
    run_off += c[u];
    run_mt += mt[u];
    run_mp += mp[u];
  }
  __syncthreads();
  scatter_block(p, 0, wcnt, off_s);
}

// Tile prefixes of caller-given group offsets (the grouped-GEMM stage entry
// point), one warp. The offsets must start at 0, never decrease and end at most
// at R; otherwise MOE_ERR_INVALID_ARG is latched and every group gets zero
// tiles, so the GEMM that follows touches nothing.
__global__ void __launch_bounds__(32) tile_prefix_kernel(const int32_t* offsets, int32_t G, int32_t R, int32_t* mt,
                                                         int32_t* mp, int* status) {
  const int lane = threadIdx.x;
  bool bad = lane == 0 && (offsets[0] != 0 || offsets[G] > R);
  for (int g = lane; g < G; g += 32) bad = bad || offsets[g + 1] < offsets[g];
  bad = __any_sync(0xffffffffu, bad);
  if (bad) latch_status(status, MOE_ERR_INVALID_ARG);
  int run_mt = 0, run_mp = 0;
  for (int g0 = 0; g0 < G; g0 += 32) {
    const int g = g0 + lane;
    const int c = (g < G && !bad) ? offsets[g + 1] - offsets[g] : 0;
    const int t1 = (c + kTileM - 1) / kTileM;
    const int t2 = (c + 2 * kTileM - 1) / (2 * kTileM);
    const int i1 = warp_inclusive_scan(t1, lane);
    const int i2 = warp_inclusive_scan(t2, lane);
    if (g < G) {
      mt[g] = run_mt + i1 - t1;
      mp[g] = run_mp + i2 - t2;
    }
    run_mt += __shfl_sync(0xffffffffu, i1, 31);
    run_mp += __shfl_sync(0xffffffffu, i2, 31);
  }
  if (lane == 0) {
    mt[G] = run_mt;
    mp[G] = run_mp;
  }
}

}  // namespace

cudaError_t launch_tile_prefix(const int32_t* offsets, int32_t G, int32_t R, int32_t* mt, int32_t* mp, int* status,
                               cudaStream_t s) {
  tile_prefix_kernel<<<1, 32, 0, s>>>(offsets, G, R, mt, mp, status);
  return counted_launch(cudaGetLastError());
}

cudaError_t launch_permute_one_chunk(const PermuteParams& p, cudaStream_t s) {
  return launch_pdl(permute_one_chunk_kernel, dim3(1), dim3(256), 0, s, 1, p);
}

cudaError_t launch_histogram(const PermuteParams& p, cudaStream_t s) {
  return launch_pdl(histogram_kernel, dim3((unsigned)p.chunks), dim3(256), 0, s, 1, p);
}

cudaError_t launch_scan(const PermuteParams& p, cudaStream_t s) {
  return launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, 1, p);
}

cudaError_t launch_scatter(const PermuteParams& p, cudaStream_t s) {
  return launch_pdl(scatter_kernel, dim3((unsigned)p.chunks), dim3(256), 0, s, 1, p);
}

}  // namespace moe

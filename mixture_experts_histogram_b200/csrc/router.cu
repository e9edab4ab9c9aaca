// Router: fp32 logits l = x . Wr^T on the tensor cores, then per token the
// top-k selection (ties to the lower expert index) and the softmax gates
// renormalised over the chosen k.
//
// Layer definition: NeMo AutoModel "Step-5-Preview" page, "Model Architecture"
// table (352 routed experts, top-8 routing, a learned router).
//
// Logits GEMM: one CTA per (128-token tile, K split). Warp 0 streams x and Wr
// tiles with TMA into a 3-4 stage ring of 128B-swizzled shared-memory tiles;
// warp 1 issues tcgen05 MMAs (M = 128 tokens, N = up to 2 x 256 experts) into a
// TMEM accumulator; warps 2-5 read the accumulator back (one token row per
// thread, 32 columns at a time), transpose each 32 x 32 block through shared
// memory and store fp32 partial logits as whole 128-byte row segments. Small T is split along K so that the
// 2.9 MB of router weights are streamed by many SMs at once; the top-k kernel
// adds the K-split partials in a fixed order. Without a K split (T >= 148 x 128
// tokens) the selection is fused into this kernel's epilogue instead.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kRouterThreads = 192;
constexpr int kRouterMaxStages = 4;
constexpr int kASmem = kTileM * kStageBytesK;  // 16 KB of x per stage

__host__ __device__ inline int router_b_bytes(const RouterParams& p) { return p.nbox * p.box_rows * kStageBytesK; }

__host__ __device__ inline int router_stages(const RouterParams& p) {
  const int per = kASmem + router_b_bytes(p);
  int st = (200 * 1024) / per;
  return st > kRouterMaxStages ? kRouterMaxStages : st;
}

// The whole K sum of this thread's token row is in TMEM (no K split): the
// token's logits (plus bias) stream through registers 32 columns at a time and
// a sorted list of the kTop largest (the earlier, lower index wins a tie, as a
// later equal value never displaces it) is kept by insertion; then the gates
// are the chosen logits' softmax. Every lane of the warp takes part in the TMEM
// loads; lanes past the last token only skip the writes.
template <int kTop>
__device__ __forceinline__ void fused_topk(const RouterParams& p, uint32_t taddr, int64_t t, int ncols, int lane) {
  float top_v[kTop];
  int top_e[kTop];
#pragma unroll
  for (int j = 0; j < kTop; ++j) {
    top_v[j] = -INFINITY;
    top_e[j] = 0x7fffffff;
  }
  const bool live = t < p.T;
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(taddr + (uint32_t)c0, v);
    tmem_ld_wait(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = c0 + i;
      if (e >= p.E) break;
      float l = __uint_as_float(v[i]);
      if (p.bias) l += __ldg(p.bias + e);
      if (live && p.logits) p.logits[t * p.E + e] = l;
      if (l > top_v[kTop - 1]) {
        float cv = l;
        int ce = e;
#pragma unroll
        for (int j = 0; j < kTop; ++j) {
          const bool sw = cv > top_v[j];
          const float tv = top_v[j];
          const int te = top_e[j];
          top_v[j] = sw ? cv : tv;
          top_e[j] = sw ? ce : te;
          cv = sw ? tv : cv;
          ce = sw ? te : ce;
        }
      }
    }
  }
  if (!live) return;
  float w[kTop], z = 0.0f;
#pragma unroll
  for (int j = 0; j < kTop; ++j) {
    w[j] = j < p.k ? expf(top_v[j] - top_v[0]) : 0.0f;
    z += w[j];
  }
#pragma unroll
  for (int j = 0; j < kTop; ++j) {
    if (j < p.k) {
      p.idx[t * p.k + j] = top_e[j];
      p.gate[t * p.k + j] = w[j] / z;
    }
  }
}

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_gemm_kernel(const RouterParams p, const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = router_stages(p);
  const int bbytes = router_b_bytes(p);
  uint8_t* sA = smem;
  uint8_t* sB = smem + stages * kASmem;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + stages * bbytes);
  uint64_t* empty = full + kRouterMaxStages;
  uint64_t* done = empty + kRouterMaxStages;
  uint64_t* drain = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m_tile = blockIdx.x, split = blockIdx.y;
  const int ks0 = (int)((int64_t)split * p.kstages / p.ksplit);
  const int ks1 = (int)((int64_t)(split + 1) * p.kstages / p.ksplit);
  const int ncols = p.nbox * p.box_rows;
  const uint32_t tmem_cols = ncols <= 32 ? 32 : ncols <= 64 ? 64 : ncols <= 128 ? 128 : ncols <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // x (and the workspace) may come from the previous kernel
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    // ---- TMA producer ----
    int stage = 0;
    uint32_t phase = 0;
    for (int ks = ks0; ks < ks1; ++ks) {
      if (!mbar_wait(&empty[stage], phase ^ 1, p.status, abort_flag)) break;
      mbar_arrive_expect_tx(&full[stage], kASmem + bbytes);
      tma_load_2d(sA + stage * kASmem, &tm_x, &full[stage], ks * 64, m_tile * kTileM);
      for (int b = 0; b < p.nbox; ++b)
        tma_load_2d(sB + stage * bbytes + b * p.box_rows * kStageBytesK, &tm_w, &full[stage], ks * 64,
                    b * p.box_rows);
      if (++stage == stages) { stage = 0; phase ^= 1; }
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    const uint32_t idesc = idesc_mma(1, kTileM, p.box_rows);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int ks = ks0; ks < ks1; ++ks) {
      if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after_sync();
      const uint64_t adesc = sdesc_k_sw128(sA + stage * kASmem);
      for (int kk = 0; kk < 4; ++kk) {
        for (int b = 0; b < p.nbox; ++b) {
          const uint64_t bdesc = sdesc_k_sw128(sB + stage * bbytes + b * p.box_rows * kStageBytesK);
          mma_bf16(tmem + b * p.box_rows, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks > ks0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(&empty[stage]);
      if (++stage == stages) { stage = 0; phase ^= 1; }
    }
    if (ok) mma_commit(done);
    // Drain: every MMA issued so far has completed once this arrives.
    mma_commit(drain);
    mbar_wait(drain, 0, p.status, abort_flag);
  } else if (warp >= 2) {
    // ---- epilogue: one token row per thread ----
    const int q = warp % 4;
    bool ok = mbar_wait(done, 0, p.status, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && p.fused) {
      tc_fence_after_sync();
      if (p.k <= 8) fused_topk<8>(p, tmem + ((uint32_t)(q * 32) << 16), m_tile * kTileM + q * 32 + lane, ncols, lane);
      else fused_topk<kMaxTopK>(p, tmem + ((uint32_t)(q * 32) << 16), m_tile * kTileM + q * 32 + lane, ncols, lane);
    } else if (ok) {
      tc_fence_after_sync();
      // Every MMA has completed (done), so the stage buffers are free: each
      // warp transposes through its own 32 x 33 float block of them.
      float* tr = reinterpret_cast<float*>(smem) + (warp - 2) * 32 * 33;
      const int row0 = m_tile * kTileM + q * 32;  // first token row of this warp
      float* dst0 = p.partial + ((int64_t)split * p.T + row0) * p.E;
      for (int c0 = 0; c0 < ncols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int i = 0; i < 32; ++i) tr[lane * 33 + i] = __uint_as_float(v[i]);
        __syncwarp();
        const int c = c0 + lane;
        for (int r = 0; r < 32 && row0 + r < p.T; ++r)
          if (c < p.E) dst0[(int64_t)r * p.E + c] = tr[r * 33 + lane];
        __syncwarp();
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// One warp per token: sum the K-split partial logits in split order, add the
// bias, pick the top k (largest logit first, ties to the lower index), and
// renormalise their softmax probabilities. kPer: experts per lane (E <= 32
// kPer); kSplitBatch: K splits whose loads are issued together. Both are sized
// to the call so the kernel keeps few registers (more warps in flight).
template <int kPer, int kSplitBatch>
__global__ void __launch_bounds__(256) topk_kernel(const TopkParams p) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  float l[kPer];
  // The loads of a batch of splits are independent and issued together; the
  // splits are added in split order.
  const float* __restrict__ part = p.partial;
#pragma unroll
  for (int i = 0; i < kPer; ++i) l[i] = (lane + 32 * i < p.E) ? 0.0f : -INFINITY;
  for (int s0 = 0; s0 < p.ksplit; s0 += kSplitBatch) {
    float v[kSplitBatch][kPer];
#pragma unroll
    for (int u = 0; u < kSplitBatch; ++u) {
      const float* src = part + ((int64_t)(s0 + u) * p.T + t) * p.E;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        v[u][i] = (s0 + u < p.ksplit && lane + 32 * i < p.E) ? __ldg(src + lane + 32 * i) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kSplitBatch; ++u)
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (s0 + u < p.ksplit) l[i] += v[u][i];
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    if (e < p.E) {
      if (p.bias) l[i] += __ldg(p.bias + e);
      if (p.logits) p.logits[t * p.E + e] = l[i];
    }
  }
  // Selection on 64-bit keys: high word the logit's bits mapped to an unsigned
  // order (larger logit, larger key), low word ~e (equal logits: the lower
  // expert index wins). Each lane keeps the best of its own candidates; a round
  // is one warp max, after which only the winning lane rescans its candidates.
  uint64_t key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    const uint32_t u = __float_as_uint(l[i] == 0.0f ? 0.0f : l[i]);  // -0 ties with +0, as floats do
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    key[i] = e < p.E ? ((uint64_t)ord << 32) | (uint32_t)~(uint32_t)e : 0ull;
  }
  uint64_t best = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) best = key[i] > best ? key[i] : best;
  uint32_t taken = 0;  // bit i: candidate i of this lane already chosen
  float my_v = -INFINITY;
  int my_e = 0;
  for (int j = 0; j < p.k; ++j) {
    uint64_t top = best;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, top, off);
      top = o > top ? o : top;
    }
    const int e = (int)~(uint32_t)top;
    if ((e & 31) == lane) {
      taken |= 1u << (e >> 5);
      best = 0;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const uint64_t kk = (taken >> i) & 1u ? 0ull : key[i];
        best = kk > best ? kk : best;
      }
    }
    if (lane == j) {
      const uint32_t ord = (uint32_t)(top >> 32);
      my_v = __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
      my_e = e;
    }
  }
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  const float w = (lane < p.k) ? expf(my_v - m) : 0.0f;
  float z = w;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  if (lane < p.k) {
    p.idx[t * p.k + lane] = my_e;
    p.gate[t * p.k + lane] = w / z;
  }
}

}  // namespace

cudaError_t launch_router_gemm(const RouterParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_w,
                               cudaStream_t s) {
  const int stages = router_stages(p);
  const size_t smem = 1024 + (size_t)stages * (kASmem + router_b_bytes(p)) + 256;
  cudaError_t e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)ceil_div(p.T, kTileM), (unsigned)p.ksplit);
  return launch_pdl(router_gemm_kernel, grid, dim3(kRouterThreads), smem, s, 1, p, tm_x, tm_w);
}

namespace {
template <int kPer>
cudaError_t launch_topk_per(const TopkParams& p, cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(p.T, 8));
  if (p.ksplit <= 2) return launch_pdl(topk_kernel<kPer, 2>, grid, dim3(256), 0, s, 1, p);
  return launch_pdl(topk_kernel<kPer, 4>, grid, dim3(256), 0, s, 1, p);
}
}  // namespace

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s) {
  static_assert(kMaxExperts <= 16 * 32, "top-k lanes hold at most 16 experts each");
  if (p.E <= 4 * 32) return launch_topk_per<4>(p, s);
  if (p.E <= 8 * 32) return launch_topk_per<8>(p, s);
  if (p.E <= 12 * 32) return launch_topk_per<12>(p, s);
  return launch_topk_per<16>(p, s);
}

}  // namespace moe

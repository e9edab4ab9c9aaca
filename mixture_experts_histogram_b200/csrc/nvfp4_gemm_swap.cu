// Grouped NVFP4 (W4A16) expert GEMMs for decode-sized groups: weights expanded
// into tensor memory as the MMA's A operand.
//
// Same products and the same exact weight expansion as nvfp4_gemm.cu (w =
// e2m1 x e4m3, exact in bf16, times the matrix's fp32 global scale in the
// epilogue). There the expanded 256 x 64 bf16 weight tile of each K stage is
// written to shared memory and read back by a 128-row MMA whose rows are
// mostly empty at decode, so shared-memory traffic (about 100 KB per 9 KB of
// weight bytes) sets the pace. Here the weight rows are the MMA's M side and a
// group's rows its N side (chunks of 32): converter warps expand each thread's
// weight row straight into TMEM (tcgen05.st), where the MMA reads it as the A
// operand (kind::f16, A from TMEM, B = the chunk's bf16 rows from shared
// memory), and shared memory carries only the codes, their scales and the
// chunk's rows.
//
// Work items: (group, 32-row chunk, 256-row weight tile), the chunks of one
// weight tile adjacent.
// Warp roles (one CTA per SM, persistent):
//   warp 0      producer: TMA of the weight codes (256 rows x 32 bytes per
//               64-deep K stage) into a raw ring, of their E4M3 scales (256 rows
//               x 16 bytes, every fourth stage) into a scale ring, and of the
//               chunk's 32 bf16 rows (64 K each) into a row ring.
//   warp 1      TMEM allocation (512 columns) and the single-thread MMA issuer.
//   warps 2-5   epilogue: warp w reads TMEM lane quarter w % 4 of both
//               accumulators (one weight row per thread; GEMM1: its gate and up
//               sums side by side) for the chunk's 32 rows.
//   warps 6-13  converters: warp w expands weight row 32 (w % 4) + lane of the
//               tile's 128-row half (w - 6) / 4 into that lane's TMEM columns
//               (two converter warps per SM sub-partition: the expansion is
//               latency-bound with one).
// TMEM columns: [0, 128) two accumulator buffers of 2 x 32 columns (tile half 0
// rows, then half 1); [128, 128 + 64 kAStages) the A stages, 32 columns per
// half (K elements 2c, 2c + 1 in column c).
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kNsEpiWarps = 4;
constexpr int kNsConvWarps = 8;
constexpr int kNsThreads = 32 * (2 + kNsEpiWarps + kNsConvWarps);
constexpr int kNsTok = 32;                       // rows per chunk (MMA N)
constexpr int kNsRaw = 8;                        // code stages in flight
constexpr int kNsScaleSlots = (kNsRaw + 6) / 4;  // a slot serves 4 stages (see nvfp4_gemm.cu)
constexpr int kNsRowStages = 8;                  // chunk-row stages in flight
constexpr int kNsAStages = 4;                    // expanded weight stages in TMEM
constexpr int kNsCodeBytes = 256 * 32;           // 256 rows x 64 E2M1 codes
constexpr int kNsScaleBytes = 256 * 16;          // 256 rows x 16 E4M3 scales (4 stages)
constexpr int kNsRowBytes = kNsTok * 128;        // 32 rows x 64 bf16
constexpr uint32_t kNsDCols = 128;               // two accumulator buffers of 64 columns
constexpr uint32_t kNsTmemCols = 512;
static_assert(4 * kNsScaleSlots >= kNsRaw + 3, "scale slots too few for the raw ring");
static_assert(kNsDCols + 64 * kNsAStages <= kNsTmemCols, "TMEM budget");
static_assert(kNsRaw <= 16 && kNsAStages <= 8, "ring sizes fit the drain bitmask");

struct NsLayout {
  static constexpr size_t kRows = 0;
  static constexpr size_t kCodes = kRows + (size_t)kNsRowStages * kNsRowBytes;
  static constexpr size_t kScales = kCodes + (size_t)kNsRaw * kNsCodeBytes;
  static constexpr size_t kBars = kScales + (size_t)kNsScaleSlots * kNsScaleBytes;
  static constexpr int kNumBars = 2 * kNsRaw + 2 * kNsRowStages + 2 * kNsAStages + 2 + 2 + 1;
  static constexpr size_t kMisc = kBars + kNumBars * 8;  // tmem slot, abort flag
  static constexpr size_t kMs = kMisc + 16;              // int [G + 1] chunk prefix
  static constexpr size_t kOff = kMs + (kMaxExperts + 2) * 4;
  static constexpr size_t kEnd = kOff + (kMaxExperts + 2) * 4;
  static constexpr size_t kDynamic = kEnd + 1024;
  static_assert(kNsRowBytes % 1024 == 0 && kCodes % 1024 == 0, "swizzled row tiles");
  static_assert(kBars % 8 == 0, "mbarrier alignment");
  static_assert(kDynamic <= 227 * 1024, "shared memory budget");
};

// 14 warps put four on two of the SM's sub-partitions, whose register files
// then allow 128 registers a thread: the bound is declared for 512 threads.
static_assert(kNsThreads <= 512, "register budget");
template <bool kGemm1>
__global__ void __launch_bounds__(512, 1)
    nvfp4_swap_kernel(const GemmParams p, const __grid_constant__ AMaps tm_a, const __grid_constant__ NvMaps tm) {
  using L = NsLayout;
  constexpr uint32_t kIdesc = idesc_mma(1u, 128, kNsTok);  // bf16 x bf16, M = 128, N = 32

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRows = smem + L::kRows;
  uint8_t* sCodes = smem + L::kCodes;
  uint8_t* sScales = smem + L::kScales;
  uint64_t* rfull = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* rempty = rfull + kNsRaw;
  uint64_t* xfull = rempty + kNsRaw;
  uint64_t* xempty = xfull + kNsRowStages;
  uint64_t* afull = xempty + kNsRowStages;
  uint64_t* aempty = afull + kNsAStages;
  uint64_t* tfull = aempty + kNsAStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_ms = reinterpret_cast<int*>(smem + L::kMs);
  int* s_off = reinterpret_cast<int*>(smem + L::kOff);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kNsRaw; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rempty[s], kNsConvWarps);
    }
    for (int s = 0; s < kNsRowStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < kNsAStages; ++s) {
      mbar_init(&afull[s], kNsConvWarps);
      mbar_init(&aempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kNsEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a.rows32);
    tma_prefetch_desc(&tm.code0);
    tma_prefetch_desc(&tm.scale0);
    tma_prefetch_desc(&tm.code1);
    tma_prefetch_desc(&tm.scale1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kNsTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Everything above overlaps the previous kernel's tail; global memory from here.
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= p.G; i += kNsThreads) s_off[i] = p.offsets[i];
  __syncthreads();
  if (warp == 0) {
    // Chunk prefix of the groups (32-row chunks); offsets that do not start at
    // 0, decrease or pass R give no work (the caller's validation latches it).
    bool bad = lane == 0 && (s_off[0] != 0 || s_off[p.G] > p.R);
    for (int g = lane; g < p.G; g += 32) bad = bad || s_off[g + 1] < s_off[g];
    bad = __any_sync(0xffffffffu, bad);
    int run = 0;
    for (int g0 = 0; g0 <= p.G; g0 += 32) {
      const int g = g0 + lane;
      const int c = (g < p.G && !bad) ? (s_off[g + 1] - s_off[g] + kNsTok - 1) / kNsTok : 0;
      int incl = c;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += v;
      }
      if (g <= p.G) s_ms[g] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  const int total = s_ms[p.G] * p.n_tiles;
  const int kstages = p.K / 64;  // 64-deep K stages (K % 256 == 0 for NVFP4)
  const int site0 = 0x3000 | (kGemm1 ? 0x200 : 0);  // wait-site codes recorded with a timeout

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t it_raw = 0, it_row = 0;
      uint32_t issued = 0, issued_phase = 0;  // raw ring bits 0-15, row ring bits 16-23
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok && p.inject != 1; item += gridDim.x) {
        const Item it = decode_item(item, p.n_tiles, p.G, kNsTok, s_ms, s_off, false);
        const bool shared = (it.g == p.E);
        // Weight rows: GEMM1 rows n*128.. of W1 (box 0) and of W3 (box 1); GEMM2
        // rows n*256.. of W2 in one box.
        const int yb = (shared ? 0 : it.g * p.N) + it.n * (kGemm1 ? 128 : 256);
        const CUtensorMap* c0 = shared ? &tm.scode0 : &tm.code0;
        const CUtensorMap* c1 = shared ? &tm.scode1 : &tm.code1;
        const CUtensorMap* s0 = shared ? &tm.sscale0 : &tm.scale0;
        const CUtensorMap* s1 = shared ? &tm.sscale1 : &tm.scale1;
        for (int ks = 0; ks < kstages && ok; ++ks) {
          const uint32_t rs = it_raw % kNsRaw, rph = (it_raw / kNsRaw) & 1u;
          if (!mbar_wait(&rempty[rs], rph ^ 1u, p.status, abort_flag, site0 | 1, item, p.wait_ns)) { ok = false; break; }
          const bool with_scales = (ks & 3) == 0;
          const uint32_t ss = (it_raw / 4) % kNsScaleSlots;
          mbar_arrive_expect_tx(&rfull[rs], kNsCodeBytes + (with_scales ? kNsScaleBytes : 0));
          uint8_t* cdst = sCodes + rs * kNsCodeBytes;
          uint8_t* sdst = sScales + ss * kNsScaleBytes;
          if (kGemm1) {
            tma_load_2d(cdst, c0, &rfull[rs], ks * 32, yb);
            tma_load_2d(cdst + kNsCodeBytes / 2, c1, &rfull[rs], ks * 32, yb);
            if (with_scales) {
              tma_load_2d(sdst, s0, &rfull[rs], (ks / 4) * 16, yb);
              tma_load_2d(sdst + kNsScaleBytes / 2, s1, &rfull[rs], (ks / 4) * 16, yb);
            }
          } else {
            tma_load_2d(cdst, c0, &rfull[rs], ks * 32, yb);
            if (with_scales) tma_load_2d(sdst, s0, &rfull[rs], (ks / 4) * 16, yb);
          }
          issued |= 1u << rs;
          issued_phase = (issued_phase & ~(1u << rs)) | (rph << rs);
          ++it_raw;
          const uint32_t xs = it_row % kNsRowStages, xph = (it_row / kNsRowStages) & 1u;
          if (!mbar_wait(&xempty[xs], xph ^ 1u, p.status, abort_flag, site0 | 2, item, p.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&xfull[xs], (uint32_t)kNsRowBytes);
          tma_load_2d(sRows + xs * kNsRowBytes, &tm_a.rows32, &xfull[xs], ks * 64, it.row0);
          issued |= 1u << (16 + xs);
          issued_phase = (issued_phase & ~(1u << (16 + xs))) | (xph << (16 + xs));
          ++it_row;
        }
      }
      if (!ok) {
        // Let the tensor copies already in flight land before the CTA leaves.
        for (int s = 0; s < 16 + kNsRowStages; ++s) {
          if (!(issued & (1u << s))) continue;
          uint64_t* bar = s < 16 ? &rfull[s] : &xfull[s - 16];
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar, (issued_phase >> s) & 1u) && global_timer_ns() - t0 < 200000000ull) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer --
      uint32_t it_a = 0, it_row = 0, acc_iter = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
        if (!mbar_wait(&tempty[b], tph ^ 1u, p.status, abort_flag, site0 | 3, (int)acc_iter, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d = tmem + b * 64;
        for (int ks = 0; ks < kstages; ++ks) {
          const uint32_t as = it_a % kNsAStages, aph = (it_a / kNsAStages) & 1u;
          const uint32_t xs = it_row % kNsRowStages, xph = (it_row / kNsRowStages) & 1u;
          if (!mbar_wait(&afull[as], aph, p.status, abort_flag, site0 | 4, (int)acc_iter, p.wait_ns) ||
              !mbar_wait(&xfull[xs], xph, p.status, abort_flag, site0 | 5, (int)acc_iter, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a0 = tmem + kNsDCols + as * 64;
          const uint64_t bd = sdesc_k_sw128(sRows + xs * kNsRowBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (ks | kk) ? 1u : 0u;
            mma_bf16_ta(d, a0 + 8 * kk, bd + 2 * kk, kIdesc, acc);
            mma_bf16_ta(d + kNsTok, a0 + 32 + 8 * kk, bd + 2 * kk, kIdesc, acc);
          }
          mma_commit(&aempty[as]);
          mma_commit(&xempty[xs]);
          ++it_a;
          ++it_row;
        }
        if (!ok) break;
        mma_commit(&tfull[b]);
        ++acc_iter;
      }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 200000000ull) {}
    }
  } else if (warp < 2 + kNsEpiWarps) {
    // ---------------------------------------------------------- epilogue --
    const int q = warp % 4;
    const int wrow = 32 * q + lane;  // weight row inside each 128-row half
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t acc_iter = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const Item it = decode_item(item, p.n_tiles, p.G, kNsTok, s_ms, s_off, false);
      const bool shared = (it.g == p.E);
      const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
      if (ok) ok = warp_wait<false>(&tfull[b], tph, p.status, abort_flag, site0 | 6, (int)acc_iter, p.wait_ns);
      tc_fence_after_sync();
      uint32_t v0[kNsTok], v1[kNsTok];
      tmem_ld32(tmem + lane_base + b * 64, v0);
      tmem_ld32(tmem + lane_base + b * 64 + kNsTok, v1);
      tmem_ld_wait(v0);
      tmem_ld_wait(v1);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
      ++acc_iter;
      if (kGemm1) {
        // v0: gate sums (W1 row j), v1: up sums (W3 row j), j = n*128 + wrow.
        const float g1 = shared ? p.bs_scale0[0] : p.b_scale0[it.g];
        const float g3 = shared ? p.bs_scale1[0] : p.b_scale1[it.g];
        const int j = it.n * 128 + wrow;
#pragma unroll
        for (int t = 0; t < kNsTok; ++t) {
          const int64_t row = (int64_t)it.row0 + t;
          if (!ok || row >= it.end) continue;
          const float g = g1 * __uint_as_float(v0[t]), u = g3 * __uint_as_float(v1[t]);
          if (p.raw_out) {
            float* o = static_cast<float*>(p.out) + row * 2 * p.N + j;
            o[0] = g;
            o[p.N] = u;
          } else {
            static_cast<__nv_bfloat16*>(p.out)[row * p.N + j] = __float2bfloat16_rn(silu_mul(g, u));
          }
        }
      } else {
        // v0: output column n*256 + wrow, v1: column n*256 + 128 + wrow.
        const float g2 = shared ? p.bs_scale0[0] : p.b_scale0[it.g];
        const int c0 = it.n * 256 + wrow, c1 = c0 + 128;
#pragma unroll
        for (int t = 0; t < kNsTok; ++t) {
          const int64_t row = (int64_t)it.row0 + t;
          if (!ok || row >= it.end) continue;
          const float gw = (p.row_gate ? p.row_gate[row] : 1.0f) * g2;
          __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.out) + row * p.N;
          if (c0 < p.N) y[c0] = __float2bfloat16_rn(__uint_as_float(v0[t]) * gw);
          if (c1 < p.N) y[c1] = __float2bfloat16_rn(__uint_as_float(v1[t]) * gw);
        }
      }
    }
  } else {
    // --------------------------------------------------------- converters --
    // Thread: weight row wrow of half h (raw row 128 h + wrow), 64 K elements
    // per stage, into TMEM lane wrow.
    const int q = warp % 4;
    const int h = (warp - 2 - kNsEpiWarps) / 4;
    const int wrow = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t it_raw = 0, it_a = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      for (int ks = 0; ks < kstages; ++ks) {
        const uint32_t rs = it_raw % kNsRaw, rph = (it_raw / kNsRaw) & 1u;
        const uint32_t as = it_a % kNsAStages, aph = (it_a / kNsAStages) & 1u;
        if (!warp_wait<false>(&rfull[rs], rph, p.status, abort_flag, site0 | 7, item, p.wait_ns) ||
            !warp_wait<false>(&aempty[as], aph ^ 1u, p.status, abort_flag, site0 | 8, item, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint8_t* codes = sCodes + rs * kNsCodeBytes;
        const uint8_t* scl = sScales + ((it_raw / 4) % kNsScaleSlots) * kNsScaleBytes + (ks & 3) * 4;
        {
          const int rr = 128 * h + wrow;
          const uint4 w0 = *reinterpret_cast<const uint4*>(codes + rr * 32);
          const uint4 w1 = *reinterpret_cast<const uint4*>(codes + rr * 32 + 16);
          const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(scl + rr * 16);
          const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          uint32_t out[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            // Word i holds K elements 8i .. 8i + 7 of this stage; their scale is
            // byte i / 2 (16 elements per scale).
            const uint4 e = expand8(w[i], (sc4 >> (8 * (i / 2))) & 0xFFu);
            out[4 * i] = e.x;
            out[4 * i + 1] = e.y;
            out[4 * i + 2] = e.z;
            out[4 * i + 3] = e.w;
          }
          tmem_st32(tmem + lane_base + kNsDCols + as * 64 + 32 * h, out);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rs]);
          mbar_arrive(&afull[as]);
        }
        ++it_raw;
        ++it_a;
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kNsTmemCols);
  }
}

template <bool kGemm1>
cudaError_t launch_ns(const GemmParams& p, int grid, const AMaps& a, const NvMaps& m, cudaStream_t s) {
  auto kern = nvfp4_swap_kernel<kGemm1>;
  static bool attr_set = false;  // per process; one device's limit serves every B200
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)NsLayout::kDynamic);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kNsThreads), NsLayout::kDynamic, s, 1, p, a, m);
}

}  // namespace

cudaError_t launch_nvfp4_swap(const GemmParams& p, bool gemm1, int grid, const AMaps& tm_a, const NvMaps& tm,
                              cudaStream_t s) {
  return gemm1 ? launch_ns<true>(p, grid, tm_a, tm, s) : launch_ns<false>(p, grid, tm_a, tm, s);
}

}  // namespace moe

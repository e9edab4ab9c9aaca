// Grouped expert GEMMs with NVFP4 expert weights and bf16 activations (W4A16)
// on the 5th-generation tensor cores.
//
// NVFP4 storage (TensorFold PR page, the NVFP4 format its W4A16 linears read):
// E2M1 codes two to a byte (input 2j in the low nibble of byte j) [n, k/2], one
// E4M3 scale per 16 inputs [n, k/16], and an fp32 global scale per matrix that
// multiplies: w = e2m1 x e4m3 x global. Here each routed expert's W1, W3, W2
// (and the shared expert's) is one such matrix, with its own global scale.
//
// The product e2m1 x e4m3 has at most five significant bits and lies in
// [2^-10, 2688], so it is exact in bf16: converter warps expand each stage's
// codes and scales into a bf16 weight tile in shared memory, in the 128-byte
// swizzled K-major layout the MMA reads, and the tile is multiplied on the
// tensor cores (kind::f16, bf16 x bf16 -> fp32 in TMEM) exactly as BF16
// weights would be. The global scale multiplies the fp32 accumulator in the
// epilogue (sum_k x_k (q_k s_k) g = g sum_k x_k q_k s_k).
//
//   GEMM1: h[r, j] = silu(g1 A[r].W1q[j]) * (g3 A[r].W3q[j]), stored bf16
//   GEMM2: y[r, c] = gate[r] * g2 (h[r] . W2q[c]), stored bf16
//
// One CTA per SM, persistent over the same work items as the BF16/FP8 kernel
// (128-row tiles, 256 accumulator columns; GEMM1: 128 gate + 128 up columns).
// Warp roles:
//   warp 0       producer: TMA of the activation tile (into the MMA ring), of
//                the weight codes (256 rows x 32 bytes per 64-deep K stage, into
//                a raw ring) and, every 4 stages, of their scales (256 rows x 16
//                bytes) into a small scale ring.
//   warp 1       TMEM allocation (512 columns) and the single-thread MMA issuer.
//   warps 2-9    epilogue (two column halves x four TMEM lane quarters).
//   warps 10-17  converters: codes x scales -> bf16 weight tile, then a proxy
//                fence and an arrival that hands the stage to the MMA.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kConvWarps = 8;
constexpr int kEpiWarpsNv = 8;
constexpr int kNvThreads = 32 * (2 + kEpiWarpsNv + kConvWarps);
#ifndef MOE_NV_CONV_STAGES
#define MOE_NV_CONV_STAGES 3
#endif
#ifndef MOE_NV_RAW_STAGES
#define MOE_NV_RAW_STAGES 4
#endif
constexpr int kConvStages = MOE_NV_CONV_STAGES;  // A + converted B tiles (the MMA's ring)
constexpr int kRawStages = MOE_NV_RAW_STAGES;    // codes (the converters' ring)
// A scale slot serves 4 stages. The producer refills the slot of scale group
// G at stage 4G after the converters finished stage 4G - kRawStages, so the
// slot's previous group (G - kScaleSlots) must end by then:
// 4 (G - kScaleSlots) + 3 <= 4G - kRawStages.
constexpr int kScaleSlots = (kRawStages + 3 + 3) / 4;
static_assert(4 * kScaleSlots >= kRawStages + 3, "scale slots too few for the raw ring");
static_assert(kRawStages >= 4 && kRawStages <= 24 && kConvStages <= 8, "ring sizes fit the drain bitmask");
constexpr int kABytesNv = kTileM * 128;        // 128 rows x 64 bf16
constexpr int kBRows = 256;
constexpr int kBBytesNv = kBRows * 128;        // 256 rows x 64 bf16
constexpr int kCodeBytes = kBRows * 32;        // 256 rows x 64 E2M1 codes
constexpr int kScaleSlotBytes = kBRows * 16;   // 256 rows x 16 E4M3 scales (4 stages)

struct NvLayout {
  static constexpr size_t kA = 0;
  static constexpr size_t kB = kA + (size_t)kConvStages * kABytesNv;
  static constexpr size_t kCodes = kB + (size_t)kConvStages * kBBytesNv;
  static constexpr size_t kScales = kCodes + (size_t)kRawStages * kCodeBytes;
  static constexpr size_t kBars = kScales + (size_t)kScaleSlots * kScaleSlotBytes;
  static constexpr int kNumBars = 2 * kConvStages + 2 * kRawStages + 2 + 2 + 1;
  static constexpr size_t kMisc = kBars + ((kNumBars * 8 + 127) / 128) * 128;  // tmem slot, abort flag
  static constexpr size_t kMt = kMisc + 64;
  static constexpr size_t kOff = kMt + (kMaxExperts + 2) * 4;
  static constexpr size_t kEnd = kOff + (kMaxExperts + 2) * 4;
  static constexpr size_t kDynamic = kEnd + 1024;
  static_assert(kDynamic <= 227 * 1024, "shared memory budget");
  static_assert(kMisc >= kBars + kNumBars * 8, "mbarriers overlap the misc words");
};

template <bool kGemm1>
__global__ void __launch_bounds__(kNvThreads, 1)
    nvfp4_gemm_kernel(const GemmParams p, const __grid_constant__ AMaps tm_a, const __grid_constant__ NvMaps tm) {
  using L = NvLayout;
  constexpr uint32_t kIdesc = idesc_mma(1u, kTileM, 256);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + L::kA;
  uint8_t* sB = smem + L::kB;
  uint8_t* sCodes = smem + L::kCodes;
  uint8_t* sScales = smem + L::kScales;
  uint64_t* cfull = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* cempty = cfull + kConvStages;
  uint64_t* rfull = cempty + kConvStages;
  uint64_t* rempty = rfull + kRawStages;
  uint64_t* tfull = rempty + kRawStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_mt = reinterpret_cast<int*>(smem + L::kMt);
  int* s_off = reinterpret_cast<int*>(smem + L::kOff);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kConvStages; ++s) {
      mbar_init(&cfull[s], 1 + kConvWarps);  // the producer (A bytes) and every converter warp
      mbar_init(&cempty[s], 1);              // the MMA's commit
    }
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rempty[s], kConvWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarpsNv);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a.rows128);
    tma_prefetch_desc(&tm_a.rows64);
    tma_prefetch_desc(&tm_a.rows32);
    tma_prefetch_desc(&tm.code0);
    tma_prefetch_desc(&tm.scale0);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Everything above overlaps the previous kernel's tail; global memory from here.
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= p.G; i += kNvThreads) {
    s_mt[i] = p.mt_prefix[i];
    s_off[i] = p.offsets[i];
  }
  __syncthreads();
  const int total = s_mt[p.G] * p.n_tiles;
  const int kstages = p.K / 64;
  const int site0 = 0x1000 | (kGemm1 ? 0x200 : 0);  // wait-site codes recorded with a timeout

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t it_raw = 0, it_conv = 0;
      uint32_t issued = 0, issued_phase = 0;  // raw ring (bit s) and MMA ring (bit 24 + s)
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok && p.inject != 1; item += gridDim.x) {
        const Item it = decode_item(item, p.n_tiles, p.G, kTileM, s_mt, s_off, p.n_fastest != 0);
        const bool shared = (it.g == p.E);
        const int v = it.end - it.row0;
        const int a_rows = v <= 32 ? 32 : (v <= 64 ? 64 : 128);
        const CUtensorMap* amap = a_rows == 32 ? &tm_a.rows32 : (a_rows == 64 ? &tm_a.rows64 : &tm_a.rows128);
        // Weight rows: GEMM1 rows n*128.. of W1 (box 0) and of W3 (box 1); GEMM2
        // rows n*256.. of W2 in one box.
        const int yb = (shared ? 0 : it.g * p.N) + it.n * (kGemm1 ? 128 : 256);
        const CUtensorMap* c0 = shared ? &tm.scode0 : &tm.code0;
        const CUtensorMap* c1 = shared ? &tm.scode1 : &tm.code1;
        const CUtensorMap* s0 = shared ? &tm.sscale0 : &tm.scale0;
        const CUtensorMap* s1 = shared ? &tm.sscale1 : &tm.scale1;
        for (int ks = 0; ks < kstages && ok; ++ks) {
          const uint32_t rs = it_raw % kRawStages, rph = (it_raw / kRawStages) & 1u;
          if (!mbar_wait(&rempty[rs], rph ^ 1u, p.status, abort_flag, site0 | 1, item, p.wait_ns)) { ok = false; break; }
          const bool with_scales = (ks & 3) == 0;
          const uint32_t ss = (it_raw / 4) % kScaleSlots;
          mbar_arrive_expect_tx(&rfull[rs], kCodeBytes + (with_scales ? kScaleSlotBytes : 0));
          uint8_t* cdst = sCodes + rs * kCodeBytes;
          uint8_t* sdst = sScales + ss * kScaleSlotBytes;
          if (kGemm1) {
            tma_load_2d(cdst, c0, &rfull[rs], ks * 32, yb);
            tma_load_2d(cdst + kCodeBytes / 2, c1, &rfull[rs], ks * 32, yb);
            if (with_scales) {
              tma_load_2d(sdst, s0, &rfull[rs], (ks / 4) * 16, yb);
              tma_load_2d(sdst + kScaleSlotBytes / 2, s1, &rfull[rs], (ks / 4) * 16, yb);
            }
          } else {
            tma_load_2d(cdst, c0, &rfull[rs], ks * 32, yb);
            if (with_scales) tma_load_2d(sdst, s0, &rfull[rs], (ks / 4) * 16, yb);
          }
          issued |= 1u << rs;
          issued_phase = (issued_phase & ~(1u << rs)) | (rph << rs);
          ++it_raw;
          const uint32_t cs = it_conv % kConvStages, cph = (it_conv / kConvStages) & 1u;
          if (!mbar_wait(&cempty[cs], cph ^ 1u, p.status, abort_flag, site0 | 2, item, p.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&cfull[cs], (uint32_t)a_rows * 128u);
          tma_load_2d(sA + cs * kABytesNv, amap, &cfull[cs], ks * 64, it.row0);
          issued |= 1u << (24 + cs);
          issued_phase = (issued_phase & ~(1u << (24 + cs))) | (cph << (24 + cs));
          ++it_conv;
        }
      }
      if (!ok) {
        // Let the tensor copies already in flight land before the CTA leaves.
        for (int s = 0; s < 24 + kConvStages; ++s) {
          if (!(issued & (1u << s))) continue;
          uint64_t* bar = s < 24 ? &rfull[s] : &cfull[s - 24];
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar, (issued_phase >> s) & 1u) && global_timer_ns() - t0 < 200000000ull) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer --
      uint32_t it_conv = 0, acc_iter = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
        if (!mbar_wait(&tempty[b], tph ^ 1u, p.status, abort_flag, site0 | 3, (int)acc_iter, p.wait_ns)) break;
        tc_fence_after_sync();
        const uint32_t d = tmem + b * 256;
        for (int ks = 0; ks < kstages; ++ks) {
          const uint32_t cs = it_conv % kConvStages, cph = (it_conv / kConvStages) & 1u;
          if (!mbar_wait(&cfull[cs], cph, p.status, abort_flag, site0 | 4, (int)acc_iter, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint64_t ad = sdesc_k_sw128(sA + cs * kABytesNv);
          const uint64_t bd = sdesc_k_sw128(sB + cs * kBBytesNv);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16(d, ad + 2 * kk, bd + 2 * kk, kIdesc, (ks | kk) ? 1u : 0u);
          mma_commit(&cempty[cs]);
          ++it_conv;
        }
        if (!ok) break;
        mma_commit(&tfull[b]);
        ++acc_iter;
      }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 200000000ull) {}
    }
  } else if (warp < 2 + kEpiWarpsNv) {
    // ---------------------------------------------------------- epilogue --
    const int q = warp % 4;
    const int hf = (warp - 2) / 4;
    const int rl = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t acc_iter = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const Item it = decode_item(item, p.n_tiles, p.G, kTileM, s_mt, s_off, p.n_fastest != 0);
      const bool shared = (it.g == p.E);
      const int64_t row = (int64_t)it.row0 + rl;
      const bool row_ok = row < it.end;
      const int col0 = kGemm1 ? it.n * 128 + 64 * hf : it.n * 256 + 128 * hf;
      const bool col_ok = col0 < p.N;
      const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
      if (ok) ok = warp_wait<false>(&tfull[b], tph, p.status, abort_flag, site0 | 6, (int)acc_iter, p.wait_ns);
      tc_fence_after_sync();
      const uint32_t base = tmem + lane_base + b * 256;
      auto release = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
      };
      if (kGemm1) {
        // Global scales of this expert's W1 (gate) and W3 (up).
        const float g1 = shared ? p.bs_scale0[0] : p.b_scale0[it.g];
        const float g3 = shared ? p.bs_scale1[0] : p.b_scale1[it.g];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t g[32], u[32];
          tmem_ld32(base + 64 * hf + 32 * ch, g);
          tmem_ld32(base + 128 + 64 * hf + 32 * ch, u);
          tmem_ld_wait(g);
          tmem_ld_wait(u);
          if (ch == 1) release();
          if (p.raw_out) {
            if (ok && row_ok) {
              float4* dg = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * 2 * p.N + col0 + 32 * ch);
              float4* du = dg + p.N / 4;
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                dg[v] = make_float4(g1 * __uint_as_float(g[4 * v]), g1 * __uint_as_float(g[4 * v + 1]),
                                    g1 * __uint_as_float(g[4 * v + 2]), g1 * __uint_as_float(g[4 * v + 3]));
                du[v] = make_float4(g3 * __uint_as_float(u[4 * v]), g3 * __uint_as_float(u[4 * v + 1]),
                                    g3 * __uint_as_float(u[4 * v + 2]), g3 * __uint_as_float(u[4 * v + 3]));
              }
            }
            continue;
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(silu_mul(g1 * __uint_as_float(g[2 * i]), g3 * __uint_as_float(u[2 * i])),
                                silu_mul(g1 * __uint_as_float(g[2 * i + 1]), g3 * __uint_as_float(u[2 * i + 1])));
          if (ok && row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.N + col0 + 32 * ch);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        const float g2 = shared ? p.bs_scale0[0] : p.b_scale0[it.g];
        const float gw = row_ok ? (p.row_gate ? p.row_gate[row] : 1.0f) * g2 : 0.0f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          tmem_ld32(base + 128 * hf + 32 * ch, v);
          tmem_ld_wait(v);
          if (ch == 3) release();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * gw, __uint_as_float(v[2 * i + 1]) * gw);
          if (ok && row_ok && col_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.N + col0 + 32 * ch);
#pragma unroll
            for (int w = 0; w < 4; ++w) dst[w] = make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
          }
        }
      }
      ++acc_iter;
    }
  } else {
    // --------------------------------------------------------- converters --
    const int cw = warp - 2 - kEpiWarpsNv;   // 0..7
    const int c = lane & 7;                   // 16-byte chunk of a 128-byte row: 8 weights
    const int r0 = (lane >> 3) + 4 * cw;      // this lane's rows: r0 + 32 i
    uint32_t it_raw = 0, it_conv = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      for (int ks = 0; ks < kstages; ++ks) {
        const uint32_t rs = it_raw % kRawStages, rph = (it_raw / kRawStages) & 1u;
        const uint32_t cs = it_conv % kConvStages, cph = (it_conv / kConvStages) & 1u;
        if (!warp_wait<false>(&rfull[rs], rph, p.status, abort_flag, site0 | 7, item, p.wait_ns) ||
            !warp_wait<false>(&cempty[cs], cph ^ 1u, p.status, abort_flag, site0 | 8, item, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint8_t* codes = sCodes + rs * kCodeBytes;
        const uint8_t* scl = sScales + ((it_raw / 4) % kScaleSlots) * kScaleSlotBytes + (ks & 3) * 4 + (c >> 1);
        uint8_t* dst = sB + cs * kBBytesNv;
        // All loads first: the compiler cannot move a load from the code ring
        // above a store into the weight tile (it cannot tell they never alias).
        uint32_t w[kBRows / 32], sc[kBRows / 32];
#pragma unroll
        for (int i = 0; i < kBRows / 32; ++i) {
          const int r = r0 + 32 * i;
          w[i] = *reinterpret_cast<const uint32_t*>(codes + r * 32 + c * 4);
          sc[i] = scl[r * 16];
        }
#pragma unroll
        for (int i = 0; i < kBRows / 32; ++i) {
          const int r = r0 + 32 * i;
          // 128-byte swizzle: chunk c of row r lands at chunk c ^ (r % 8).
          *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = expand8(w[i], sc[i]);
        }
        fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[rs]);
          mbar_arrive(&cfull[cs]);
        }
        ++it_raw;
        ++it_conv;
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

template <bool kGemm1>
cudaError_t launch_nv(const GemmParams& p, int grid, const AMaps& a, const NvMaps& m, cudaStream_t s) {
  auto kern = nvfp4_gemm_kernel<kGemm1>;
  static bool attr_set = false;  // per process; one device's limit serves every B200
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)NvLayout::kDynamic);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kNvThreads), NvLayout::kDynamic, s, 1, p, a, m);
}

}  // namespace

cudaError_t launch_nvfp4_gemm(const GemmParams& p, bool gemm1, int grid, const AMaps& tm_a, const NvMaps& tm,
                              cudaStream_t s) {
  return gemm1 ? launch_nv<true>(p, grid, tm_a, tm, s) : launch_nv<false>(p, grid, tm_a, tm, s);
}

}  // namespace moe

// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The experts are SwiGLU MLPs (NeMo AutoModel "Step-5-Preview" page, "Model
// Architecture": 352 routed experts and one shared expert, intermediate size
// 1,536); expert weights are BF16 or block-scaled FP8 E4M3 (StepFun "Step-5
// minimal inference" README: "block-scaled FP8 expert GEMM"). The shared
// expert is simply group E, after the routed groups.
//
//   GEMM1 (gate/up + SwiGLU):  for each row r of group g and output column j < I
//       h[r, j] = silu(A[r] . W1_g[j]) * (A[r] . W3_g[j])
//     BF16: h stored bf16. FP8: h quantised per 1x128 block (scale = blockmax/448),
//     codes E4M3, scales stored transposed [I/128, rows].
//   GEMM2 (down):  y[r, c] = gate[r] * (h[r] . W2_g[c]), stored bf16.
//
// Accumulator tile per CTA: 128 rows x 256 columns. GEMM1's 256 columns are
// 128 gate columns (W1 rows n0..n0+127) and the matching 128 up columns (W3
// rows n0..n0+127) side by side in one N = 256 MMA, so SwiGLU pairs sit in one
// thread's registers. GEMM2 covers 256 output columns.
//
// Two variants:
//   single (kPair = false): one CTA per tile; each stage holds A (128 rows) and
//     the whole 256-row B tile (48 KB); 4 stages.
//   pair (kPair = true): a cluster of two CTAs on one TPC computes a 256-row
//     tile with 2-SM MMAs (M = 256). Each CTA loads its own 128 A rows and one
//     128-row half of the B tile (32 KB a stage, 6 stages), so every weight
//     tile crosses L2 -> SM once per pair instead of once per 128 rows: a third
//     less L2 traffic per FLOP, for groups with more than ~100 rows.
//
// Persistent CTAs (pairs) walk a static list of work items (group, N tile,
// M tile). GEMM1 keeps the M tiles of one (group, N tile) adjacent, so CTAs
// sharing a weight tile run together; GEMM2 keeps the N tiles of one row tile
// adjacent (its h rows are re-read by 16 N tiles), which measured faster.
// Warp roles:
//   warp 0      producer. Lane 0 issues the TMA loads. In FP8 mode all 32 lanes
//               also cp.async each K block's 128 row scales and two
//               weight-block scales into an 8-slot ring in shared memory.
//   warp 1      allocates 512 TMEM columns; one thread issues the MMAs (in the
//               pair variant only the even CTA of the pair issues them).
//   warps 2-9   epilogue: 2 column halves x 4 TMEM lane quarters; each thread
//               owns one row (TMEM lane) and one half of the tile's columns.
// BF16: the accumulator lives in TMEM for the whole K loop; two 256-column
// buffers let the epilogue of one tile overlap the MMAs of the next.
// FP8: the fp32 block scales are not powers of two, so each 128-deep K block is
// computed into a TMEM partial (two ping-pong buffers) and the epilogue warps
// promote it into register accumulators with sa[row, kb] * sb[nblk, kb].
// FP8 down GEMM with kStoreY: each epilogue warp writes its 32 rows x 128 bf16
// columns of y into shared memory as two 128B-swizzled 32 x 64 boxes and one
// lane stores them with TMA (whole 128-byte lines, asynchronously); the 64 KB
// of staging take one pipeline stage (single: 3 stages, pair: 4).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "gemm_common.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kABytes = kTileM * kStageBytesK;  // 16 KB: 128 rows of A
constexpr int kMaxStages = 6;
constexpr int kMaxGroups = kMaxExperts + 1;
constexpr int kScRing = 8;                      // K blocks of staged FP8 scales
constexpr int kScSlot = 132;                    // floats: 128 row scales + 2 block scales (+ pad)
#ifndef MOE_FP8_CHUNK
#define MOE_FP8_CHUNK 16
#endif
constexpr int kFp8Chunk = MOE_FP8_CHUNK;        // TMEM columns per load when promoting FP8 partials
constexpr int kYBox = 32 * 128;                 // bytes of one y store box: 32 rows x 64 bf16 columns
constexpr int kYWarpBytes = 2 * kYBox;          // an epilogue warp's 32 rows x 128 columns


// kStoreY: the FP8 down GEMM's bf16 y tiles leave through shared memory and TMA
// stores (64 KB of staging, one fewer pipeline stage).
template <bool kPair, bool kStoreY>
struct Cfg {
  static constexpr int kStages = (kPair ? 6 : 4) - (kStoreY ? (kPair ? 2 : 1) : 0);
  static constexpr int kBBytes = (kPair ? 128 : 256) * kStageBytesK;  // this CTA's share of the B tile
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileRows = kPair ? 2 * kTileM : kTileM;      // rows of one work item
  static constexpr size_t kTiles = (size_t)kStages * kStageBytes;
  static constexpr size_t kYStage = kTiles;                           // [kEpiWarps][2 boxes][32][128 B]
  static constexpr size_t kScales = kYStage + (kStoreY ? kEpiWarps * kYWarpBytes : 0);  // float [kScRing][kScSlot]
  static constexpr size_t kBars = kScales + kScRing * kScSlot * 4;    // mbarriers (kNumBars x 8 bytes)
  static constexpr int kNumBars = 2 * kMaxStages + 2 + 2 + 1 + 2 * kScRing;
  static constexpr size_t kMisc = kBars + ((kNumBars * 8 + 127) / 128) * 128;  // tmem slot, abort flag
  static constexpr size_t kAmax = kMisc + 64;                         // float [2][2][128]
  static constexpr size_t kMt = kAmax + 2 * 2 * 128 * 4;              // int [kMaxGroups + 1]
  static constexpr size_t kOff = kMt + (kMaxGroups + 1) * 4;          // int [kMaxGroups + 1]
  static constexpr size_t kEnd = kOff + (kMaxGroups + 1) * 4;
  static constexpr size_t kDynamic = kEnd + 1024;                     // + alignment slack
  static_assert(kMisc >= kBars + kNumBars * 8, "mbarriers overlap the misc words");
  static_assert(kDynamic <= 227 * 1024, "shared memory budget");
  static_assert(kTiles % 1024 == 0, "the y staging boxes need 1024-byte alignment (128-byte swizzle)");
};


// Weight-tile rows of a work item: box 0 starts at row `yb` of `*m0`, box 1 at
// row `yb2` of `*m1`. GEMM1: W1 and W3 rows n0.. (128-row boxes). GEMM2: `*m0`
// maps W2 with 256-row boxes (rows n0..n0+255 in one load), `*m1` the same W2
// with 128-row boxes (the 2-SM variant loads rows n0.. and n0+128.. per CTA).
template <bool kGemm1>
struct BRows {
  const CUtensorMap *m0, *m1;
  int yb, yb2;
  __device__ __forceinline__ BRows(const Item& it, const GemmParams& p, const CUtensorMap* b0, const CUtensorMap* b1,
                                   const CUtensorMap* bs0, const CUtensorMap* bs1) {
    const bool shared = (it.g == p.E);
    yb = (shared ? 0 : it.g * p.N) + it.n * (kGemm1 ? 128 : 256);
    m0 = shared ? bs0 : b0;
    m1 = shared ? bs1 : b1;  // GEMM1: W3; GEMM2: the same W2 with 128-row boxes
    yb2 = kGemm1 ? yb : yb + 128;
  }
};


template <bool kFP8, bool kGemm1, bool kPair, bool kStoreY>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const GemmParams p, const __grid_constant__ AMaps tm_a,
                        const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                        const __grid_constant__ CUtensorMap tm_bs0, const __grid_constant__ CUtensorMap tm_bs1,
                        const __grid_constant__ CUtensorMap tm_y) {
  static_assert(!kStoreY || (kFP8 && !kGemm1), "staged y stores belong to the FP8 down GEMM");
  using C = Cfg<kPair, kStoreY>;
  constexpr int kElemsPerStage = kFP8 ? 128 : 64;  // 128 bytes of K per stage
  constexpr uint32_t kIdesc = idesc_mma(kFP8 ? 0u : 1u, kPair ? 2 * kTileM : kTileM, 256);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * kABytes;
  float* sc = reinterpret_cast<float*>(smem + C::kScales);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBars);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* scfull = drain + 1;
  uint64_t* scempty = scfull + kScRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* amax_x = reinterpret_cast<float*>(smem + C::kAmax);
  int* s_mt = reinterpret_cast<int*>(smem + C::kMt);
  int* s_off = reinterpret_cast<int*>(smem + C::kOff);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = kPair ? cluster_cta_rank() : 0u;  // 0 = the pair's MMA issuer
  const int unit = kPair ? (int)(blockIdx.x / 2) : (int)blockIdx.x;
  const int n_units = kPair ? (int)(gridDim.x / 2) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kPair ? 2 * kEpiWarps : kEpiWarps);  // one arrival per epilogue warp
    }
    for (int j = 0; j < kScRing; ++j) {
      mbar_init(&scfull[j], 32);
      mbar_init(&scempty[j], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a.rows128);
    tma_prefetch_desc(&tm_a.rows64);
    tma_prefetch_desc(&tm_a.rows32);
    tma_prefetch_desc(&tm_b0);
    tma_prefetch_desc(&tm_bs0);
    tma_prefetch_desc(&tm_b1);
    tma_prefetch_desc(&tm_bs1);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  __syncthreads();
  if (kPair) cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Everything above overlaps the previous kernel's tail; global memory from here.
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= p.G; i += kThreads) {
    s_mt[i] = p.mt_prefix[i];
    s_off[i] = p.offsets[i];
  }
  __syncthreads();
  // Work items: (K piece, group, M tile, N tile); k_split > 1 only for the down
  // GEMM when its tiles alone cannot fill the GPU.
  const int base_total = s_mt[p.G] * p.n_tiles;
  const int total = base_total * p.k_split;
  const int kstages = p.K / kElemsPerStage;
  const int nkb = p.K / 128;
  // The item's K piece kp and K stages [ks0, ks1) (FP8: one 128-deep K block per stage).
  auto krange = [&](int item, int& kp, int& ks0, int& ks1) {
    kp = item / base_total;
    ks0 = (int)((int64_t)kstages * kp / p.k_split);
    ks1 = (int)((int64_t)kstages * (kp + 1) / p.k_split);
  };
  // ... and its tile.
  auto piece = [&](int item, int& kp, int& ks0, int& ks1) -> Item {
    krange(item, kp, ks0, ks1);
    return decode_item(item - kp * base_total, p.n_tiles, p.G, C::kTileRows, s_mt, s_off, p.n_fastest != 0);
  };
  const int my_off = kPair ? kTileM * (int)rank : 0;  // this CTA's rows inside a work item
  // Wait-site codes recorded with a timeout: kernel variant, CTA rank, wait.
  const int site0 = (kFP8 ? 0x100 : 0) | (kGemm1 ? 0x200 : 0) | (kPair ? 0x400 : 0) | (int)(rank << 11);
#ifdef MOE_DEBUG_STATE
  int dbg_a = -1, dbg_b = -1, dbg_c = -1;
#define MOE_DBG(a, b, c) (dbg_a = (int)(a), dbg_b = (int)(b), dbg_c = (int)(c))
#else
#define MOE_DBG(a, b, c) ((void)0)
#endif

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    int stage = 0;
    uint32_t phase = 0, sc_iter = 0;
    uint32_t issued = 0;        // bit s: stage s has had a load issued
    uint32_t issued_phase = 0;  // bit s: the phase of that last issue
    bool ok = true;
    // (Test hook: with p.inject == 1 nothing is loaded, so the consumers' first
    // waits run out and the kernel returns MOE_ERR_DEVICE_TIMEOUT with nothing
    // in flight.)
    for (int item = unit; item < total && ok && p.inject != 1; item += n_units) {
      int kp, ks0, ks1;
      const Item it = piece(item, kp, ks0, ks1);
      const bool shared = (it.g == p.E);
      const int my_row0 = it.row0 + my_off;
      const BRows<kGemm1> rows(it, p, &tm_b0, &tm_b1, &tm_bs0, &tm_bs1);
      // A box: the smallest of 32 / 64 / 128 rows that covers this CTA's rows of
      // the group (bytes per stage a_bytes; the pair leader also needs its peer's).
      auto a_rows = [&](int row0) { const int v = it.end - row0; return v <= 32 ? 32 : (v <= 64 ? 64 : 128); };
      const int my_a_rows = a_rows(my_row0);
      const CUtensorMap* amap = my_a_rows == 32 ? &tm_a.rows32 : (my_a_rows == 64 ? &tm_a.rows64 : &tm_a.rows128);
      const uint32_t stage_tx = kPair ? (uint32_t)(a_rows(it.row0) + a_rows(it.row0 + kTileM)) * kStageBytesK +
                                            2u * C::kBBytes
                                      : (uint32_t)my_a_rows * kStageBytesK + C::kBBytes;
      // FP8: where this tile's weight-block scales start (one fp32 per K block).
      const float *sb0 = nullptr, *sb1 = nullptr;
      if (kFP8) {
        const int nblk = p.N / 128;
        if (kGemm1) {
          const int64_t blk = shared ? (int64_t)it.n : (int64_t)it.g * nblk + it.n;
          sb0 = (shared ? p.bs_scale0 : p.b_scale0) + blk * nkb;
          sb1 = (shared ? p.bs_scale1 : p.b_scale1) + blk * nkb;
        } else {
          const int nb0 = 2 * it.n, nb1 = (2 * it.n + 1 < nblk) ? 2 * it.n + 1 : 2 * it.n;
          const float* base = shared ? p.bs_scale0 : p.b_scale0;
          const int64_t g0 = shared ? 0 : (int64_t)it.g * nblk;
          sb0 = base + (g0 + nb0) * nkb;
          sb1 = base + (g0 + nb1) * nkb;
        }
      }
      for (int ks = ks0; ks < ks1; ++ks) {
        bool w = true;
        MOE_DBG(item, ks, sc_iter);
        if (lane == 0) w = mbar_wait(&empty[stage], phase ^ 1, p.status, abort_flag, site0 | 1, item, p.wait_ns);
        if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) { ok = false; break; }
        if (lane == 0) {
          const int kx = ks * kElemsPerStage;
          if (kPair) {
            // Both CTAs' tiles complete on the even CTA's barrier, which expects them all.
            const uint32_t bar0 = map_to_cta(&full[stage], 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], stage_tx);
            tma_load_2d_pair(sA + stage * kABytes, amap, bar0, kx, my_row0);
            // GEMM2's 128-row halves come from the 128-row-box map (passed as the second map).
            tma_load_2d_pair(sB + stage * C::kBBytes, (kGemm1 && rank == 0) ? rows.m0 : rows.m1, bar0, kx,
                             rank ? rows.yb2 : rows.yb);
          } else {
            mbar_arrive_expect_tx(&full[stage], stage_tx);
            tma_load_2d(sA + stage * kABytes, amap, &full[stage], kx, my_row0);
            if (kGemm1) {
              tma_load_2d(sB + stage * C::kBBytes, rows.m0, &full[stage], kx, rows.yb);
              tma_load_2d(sB + stage * C::kBBytes + C::kBBytes / 2, rows.m1, &full[stage], kx, rows.yb2);
            } else {
              // GEMM2's 256 weight rows are contiguous: one 256-row box.
              tma_load_2d(sB + stage * C::kBBytes, rows.m0, &full[stage], kx, rows.yb);
            }
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        }
        if (kFP8) {
          const uint32_t j = sc_iter % kScRing, sph = (sc_iter / kScRing) & 1u;
          if (!warp_wait<false>(&scempty[j], sph ^ 1u, p.status, abort_flag, site0 | 2, item, p.wait_ns)) {
            ok = false;
            break;
          }
          float* slot = sc + j * kScSlot;
          const float* src = p.a_scale + (int64_t)ks * p.rows_pad + my_row0 + lane * 4;
#pragma unroll
          for (int i = 0; i < 4; ++i) cp_async_4(slot + lane * 4 + i, src + i);
          if (lane == 0) {
            cp_async_4(slot + 128, sb0 + ks);
            cp_async_4(slot + 129, sb1 + ks);
          }
          cp_async_arrive(&scfull[j]);
          ++sc_iter;
        }
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    if (kFP8) asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok && lane == 0 && rank == 0) {
      // Let the tensor copies already in flight land before the CTA leaves.
      for (int s = 0; s < C::kStages; ++s) {
        if (!(issued & (1u << s))) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[s], (issued_phase >> s) & 1u) && global_timer_ns() - t0 < 200000000ull) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------ MMA issuer --
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t acc) {
        if (kPair) {
          if (kFP8) mma_e4m3_pair(d, ad, bd, kIdesc, acc);
          else mma_bf16_pair(d, ad, bd, kIdesc, acc);
        } else {
          if (kFP8) mma_e4m3(d, ad, bd, kIdesc, acc);
          else mma_bf16(d, ad, bd, kIdesc, acc);
        }
      };
      auto commit = [&](uint64_t* bar) {
        if (kPair) mma_commit_pair(bar, 0x3);
        else mma_commit(bar);
      };
      auto wait_tempty = [&](uint32_t b, uint32_t par, uint32_t it) {
        return kPair ? mbar_wait_cluster(&tempty[b], par, p.status, abort_flag, site0 | 3, (int)it, p.wait_ns)
                     : mbar_wait(&tempty[b], par, p.status, abort_flag, site0 | 3, (int)it, p.wait_ns);
      };
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      bool ok = true;
      for (int item = unit; item < total && ok; item += n_units) {
        int kp, ks0, ks1;
        krange(item, kp, ks0, ks1);
        if (!kFP8) {
          const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
          if (!wait_tempty(b, tph ^ 1u, acc_iter)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t d = tmem + b * 256;
          for (int ks = ks0; ks < ks1; ++ks) {
            if (!mbar_wait(&full[stage], phase, p.status, abort_flag, site0 | 4, (int)acc_iter, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint64_t ad = sdesc_k_sw128(sA + stage * kABytes);
            const uint64_t bd = sdesc_k_sw128(sB + stage * C::kBBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma(d, ad + 2 * kk, bd + 2 * kk, (ks != ks0 || kk) ? 1u : 0u);
            commit(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
          }
          if (!ok) break;
          commit(&tfull[b]);
          ++acc_iter;
        } else {
          for (int ks = ks0; ks < ks1; ++ks) {
            const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
            MOE_DBG(item, ks, acc_iter);
            if (!wait_tempty(b, tph ^ 1u, acc_iter)) { ok = false; break; }
            if (!mbar_wait(&full[stage], phase, p.status, abort_flag, site0 | 4, (int)acc_iter, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t d = tmem + b * 256;
            const uint64_t ad = sdesc_k_sw128(sA + stage * kABytes);
            const uint64_t bd = sdesc_k_sw128(sB + stage * C::kBBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma(d, ad + 2 * kk, bd + 2 * kk, kk ? 1u : 0u);
            commit(&empty[stage]);
            commit(&tfull[b]);
            ++acc_iter;
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
          }
        }
      }
      // Drain: every MMA issued so far has completed once this arrives.
      if (kPair) mma_commit_pair(drain, 0x1);
      else mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 200000000ull) {}
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp % 4;            // TMEM lane quarter this warp may read
    const int hf = (warp - 2) / 4;     // which half of the tile's columns
    const int rl = q * 32 + lane;      // row inside this CTA's 128 rows
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    // The accumulator is released on the pair's even CTA (or locally).
    auto release_acc = [&](uint32_t b) {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (kPair) mbar_arrive_cluster(map_to_cta(&tempty[b], 0));
        else mbar_arrive(&tempty[b]);
      }
    };
    uint32_t acc_iter = 0, tile_iter = 0, sc_iter = 0;
    bool ok = true;
    for (int item = unit; item < total; item += n_units) {
      int kp, ks0, ks1;
      const Item it = piece(item, kp, ks0, ks1);
      const int64_t row = (int64_t)it.row0 + my_off + rl;
      const bool row_ok = row < it.end;
      // Output columns of this thread: GEMM1 h columns n*128 + 64 hf (+64);
      // GEMM2 y columns n*256 + 128 hf (+128).
      const int col0 = kGemm1 ? it.n * 128 + 64 * hf : it.n * 256 + 128 * hf;
      const bool col_ok = col0 < p.N;
      if (!kFP8) {
        const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
        if (ok) ok = warp_wait<false>(&tfull[b], tph, p.status, abort_flag, site0 | 6, (int)acc_iter, p.wait_ns);
        tc_fence_after_sync();
        const uint32_t base = tmem + lane_base + b * 256;
        if (kGemm1) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t g[32], u[32];
            tmem_ld32(base + 64 * hf + 32 * ch, g);
            tmem_ld32(base + 128 + 64 * hf + 32 * ch, u);
            tmem_ld_wait(g);
            tmem_ld_wait(u);
            if (ch == 1) release_acc(b);
            if (p.raw_out) {
              // The fp32 gate and up sums themselves (stage entry point, tests).
              if (ok && row_ok) {
                float4* dg = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * 2 * p.N + col0 + 32 * ch);
                float4* du = dg + p.N / 4;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                  dg[v] = make_float4(__uint_as_float(g[4 * v]), __uint_as_float(g[4 * v + 1]),
                                      __uint_as_float(g[4 * v + 2]), __uint_as_float(g[4 * v + 3]));
                  du[v] = make_float4(__uint_as_float(u[4 * v]), __uint_as_float(u[4 * v + 1]),
                                      __uint_as_float(u[4 * v + 2]), __uint_as_float(u[4 * v + 3]));
                }
              }
              continue;
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                  silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
            if (ok && row_ok) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.N + col0 + 32 * ch);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        } else {
          const float gw = row_ok ? (p.row_gate ? p.row_gate[row] : 1.0f) : 0.0f;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t v[32];
            tmem_ld32(base + 128 * hf + 32 * ch, v);
            tmem_ld_wait(v);
            if (ch == 3) release_acc(b);
            if (p.part) {
              // Split K: this piece's fp32 sums; the gate and rounding come after the sum.
              if (ok && row_ok && col_ok) {
                float4* dst = reinterpret_cast<float4*>(p.part + ((int64_t)kp * p.R + row) * p.N + col0 + 32 * ch);
#pragma unroll
                for (int w = 0; w < 8; ++w)
                  dst[w] = make_float4(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1]),
                                       __uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3]));
              }
              continue;
            }
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
      } else {
        // FP8: promote each K block's partial with its two block scales.
        float2 acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int kb = ks0; kb < ks1; ++kb) {
          const uint32_t j = sc_iter % kScRing, sph = (sc_iter / kScRing) & 1u;
          MOE_DBG(item, kb, acc_iter);
          if (ok) ok = warp_wait<false>(&scfull[j], sph, p.status, abort_flag, site0 | 5, (int)sc_iter, p.wait_ns);
          const float* slot = sc + j * kScSlot;
          const float a_s = slot[rl];
          const float s0 = slot[128], s1 = slot[129];
          __syncwarp();
          if (lane == 0) mbar_arrive(&scempty[j]);
          ++sc_iter;
          // GEMM1: the first 64 columns are gate columns (s0), the next 64 up columns (s1).
          // GEMM2: the half's 128 columns sit in n-block 2n (hf 0, s0) or 2n+1 (s1).
          const float f0 = a_s * ((kGemm1 || hf == 0) ? s0 : s1);
          const float f1 = kGemm1 ? a_s * s1 : f0;
          const uint32_t b = acc_iter & 1u, tph = (acc_iter >> 1) & 1u;
          if (ok) ok = warp_wait<false>(&tfull[b], tph, p.status, abort_flag, site0 | 6, (int)acc_iter, p.wait_ns);
          tc_fence_after_sync();
          const uint32_t base = tmem + lane_base + b * 256;
          constexpr int kNch = 128 / kFp8Chunk;  // chunks per thread per K block
          auto col_of = [&](int ch) -> uint32_t {
            const int c = ch * kFp8Chunk;
            return kGemm1 ? (c < 64 ? 0u : 128u) + 64 * hf + (c & 63) : 128 * hf + c;
          };
          auto promote = [&](const uint32_t (&v)[kFp8Chunk], int ch) {
            const int c = ch * kFp8Chunk;
            const float f = (kGemm1 && c >= 64) ? f1 : f0;
            const float2 ff = make_float2(f, f);
#pragma unroll
            for (int i = 0; i < kFp8Chunk / 2; ++i)
              acc[c / 2 + i] = fma2(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), ff,
                                    acc[c / 2 + i]);
          };
          if constexpr (kGemm1) {
            // Two load buffers: the next chunk's load is in flight while the
            // current one is promoted (GEMM1: 1.5% faster; GEMM2 measured slower).
            uint32_t va[kFp8Chunk], vb[kFp8Chunk];
            tmem_ld16(base + col_of(0), va);
            tmem_ld_wait(va);
#pragma unroll
            for (int ch = 0; ch < kNch; ch += 2) {
              tmem_ld16(base + col_of(ch + 1), vb);
              promote(va, ch);
              tmem_ld_wait(vb);
              if (ch + 2 < kNch) tmem_ld16(base + col_of(ch + 2), va);
              else release_acc(b);  // every load of this partial has completed
              promote(vb, ch + 1);
              if (ch + 2 < kNch) tmem_ld_wait(va);
            }
          } else {
#pragma unroll
            for (int ch = 0; ch < kNch; ++ch) {
              uint32_t v[kFp8Chunk];
              tmem_ld16(base + col_of(ch), v);
              tmem_ld_wait(v);
              if (ch == kNch - 1) release_acc(b);
              promote(v, ch);
            }
          }
          ++acc_iter;
        }
        if (kGemm1 && p.raw_out) {
          // The fp32 gate and up sums themselves (stage entry point, tests):
          // acc[i] holds gate columns 2i, 2i+1 of this thread, acc[32 + i] the up ones.
          if (ok && row_ok) {
            float4* dg = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * 2 * p.N + col0);
            float4* du = dg + p.N / 4;
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              dg[v] = make_float4(acc[2 * v].x, acc[2 * v].y, acc[2 * v + 1].x, acc[2 * v + 1].y);
              du[v] = make_float4(acc[32 + 2 * v].x, acc[32 + 2 * v].y, acc[33 + 2 * v].x, acc[33 + 2 * v].y);
            }
          }
        } else if (kGemm1) {
          // SwiGLU in place (acc[0..31] gate, acc[32..63] up), then the 1x128 block
          // quantisation of h; the block spans both column halves.
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            acc[i].x = silu_mul(acc[i].x, acc[32 + i].x);
            acc[i].y = silu_mul(acc[i].y, acc[32 + i].y);
            amax = fmaxf(amax, fmaxf(fabsf(acc[i].x), fabsf(acc[i].y)));
          }
          // The two warps that share this row quarter (same q, other column
          // half) exchange their maxima; a 64-thread barrier per pair.
          float* ax = amax_x + (tile_iter & 1u) * 256;
          ax[hf * 128 + rl] = amax;
          named_bar_sync(1 + q, 64);
          amax = fmaxf(amax, ax[(1 - hf) * 128 + rl]);
          const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
          const float inv = amax > 0.0f ? __frcp_rn(s) : 0.0f;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(acc[2 * i].x * inv, acc[2 * i].y * inv),
                                                         __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(
                make_float2(acc[2 * i + 1].x * inv, acc[2 * i + 1].y * inv), __NV_SATFINITE, __NV_E4M3);
            pk[i] = lo | (hi << 16);
          }
          if (ok && row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + row * p.N + col0);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            if (hf == 0) p.out_scale[(int64_t)it.n * p.rows_pad + row] = s;
          }
          ++tile_iter;
        } else if (p.part) {
          // Split K: this piece's fp32 sums; the gate and rounding come after the sum.
          if (ok && row_ok && col_ok) {
            float4* dst = reinterpret_cast<float4*>(p.part + ((int64_t)kp * p.R + row) * p.N + col0);
#pragma unroll
            for (int w = 0; w < 32; ++w)
              dst[w] = make_float4(acc[2 * w].x, acc[2 * w].y, acc[2 * w + 1].x, acc[2 * w + 1].y);
          }
        } else {
          const float gw = row_ok ? (p.row_gate ? p.row_gate[row] : 1.0f) : 0.0f;
          auto packed = [&](int w) {  // y columns col0 + 8w .. +7 of this row, gated, bf16
            const float2 a0 = acc[4 * w], a1 = acc[4 * w + 1], a2 = acc[4 * w + 2], a3 = acc[4 * w + 3];
            return make_uint4(pack_bf16x2(a0.x * gw, a0.y * gw), pack_bf16x2(a1.x * gw, a1.y * gw),
                              pack_bf16x2(a2.x * gw, a2.y * gw), pack_bf16x2(a3.x * gw, a3.y * gw));
          };
          // A warp whose 32 rows all lie inside the group writes them as two
          // 32 x 64 boxes staged in shared memory (128B-swizzled) and stored by
          // TMA, whole 128-byte lines; a thread-per-row store touches 32 lines
          // per instruction. The warp straddling the group's end stores its
          // rows from registers.
          const int64_t wrow0 = (int64_t)it.row0 + my_off + q * 32;
          if (kStoreY && ok && col_ok && wrow0 + 32 <= it.end) {
            uint8_t* ys = smem + C::kYStage + (warp - 2) * kYWarpBytes;
            if (lane == 0) bulk_wait_group_read0();  // the previous tile's boxes have been read
            __syncwarp();
#pragma unroll
            for (int w = 0; w < 16; ++w)
              *reinterpret_cast<uint4*>(ys + (w >> 3) * kYBox + lane * 128 + (((w & 7) ^ (lane & 7)) << 4)) =
                  packed(w);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_y, ys, col0, (int32_t)wrow0);
              tma_store_2d(&tm_y, ys + kYBox, col0 + 64, (int32_t)wrow0);
              bulk_commit_group();
            }
          } else if (ok && row_ok && col_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.N + col0);
#pragma unroll
            for (int w = 0; w < 16; ++w) dst[w] = packed(w);
          }
        }
      }
    }
    if (kStoreY && lane == 0) bulk_wait_group0();  // y boxes written before the CTA leaves
  }
#ifdef MOE_DEBUG_STATE
  // Debug builds: each role's final counters, 16 ints per block from status[64],
  // for the blocks whose counters fit in the workspace's status block.
  constexpr unsigned kDbgBlocks = (unsigned)((kStatusBytes / 4 - 64) / 16);
  static_assert(64 + kDbgBlocks * 16 <= kStatusBytes / 4, "debug counters overrun the status block");
  if (kGemm1 && lane == 0 && blockIdx.x < kDbgBlocks) {
    int* dbg = p.status + 64 + blockIdx.x * 16;
    if (warp == 0) { dbg[0] = dbg_a; dbg[1] = dbg_b; dbg[2] = dbg_c; }
    if (warp == 1) { dbg[3] = dbg_a; dbg[4] = dbg_b; dbg[5] = dbg_c; }
    if (warp == 2) { dbg[6] = dbg_a; dbg[7] = dbg_b; dbg[8] = dbg_c; }
    if (warp == 6) { dbg[9] = dbg_a; dbg[10] = dbg_b; dbg[11] = dbg_c; }
    if (warp == 0) dbg[12] = total;
  }
#endif
  tc_fence_before_sync();
  __syncthreads();
  if (kPair) cluster_sync();  // neither CTA frees the pair's TMEM while the other still reads it
  if (warp == 1) {
    tc_fence_after_sync();
    if (kPair) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

template <bool kFP8, bool kGemm1, bool kPair, bool kStoreY = false>
cudaError_t launch_one(const GemmParams& p, int grid, const AMaps& a, const CUtensorMap& b0,
                       const CUtensorMap& b1, const CUtensorMap& bs0, const CUtensorMap& bs1, const CUtensorMap& y,
                       cudaStream_t s) {
  auto kern = grouped_gemm_kernel<kFP8, kGemm1, kPair, kStoreY>;
  using C = Cfg<kPair, kStoreY>;
  static bool attr_set = false;  // per process; one device's limit serves every B200
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kDynamic);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (!kPair) return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), C::kDynamic, s, 1, p, a, b0, b1, bs0, bs1, y);
  return launch_pdl(kern, dim3((unsigned)(grid & ~1)), dim3(kThreads), C::kDynamic, s, 2, p, a, b0, b1, bs0, bs1, y);
}

}  // namespace

cudaError_t launch_gemm1(const GemmParams& p, bool fp8, bool pair, int grid, const AMaps& tm_a,
                         const CUtensorMap& tm_w1, const CUtensorMap& tm_w3, const CUtensorMap& tm_sw1,
                         const CUtensorMap& tm_sw3, cudaStream_t s) {
  // (The y map is unused by the gate/up GEMM.)
  if (pair)
    return fp8 ? launch_one<true, true, true>(p, grid, tm_a, tm_w1, tm_w3, tm_sw1, tm_sw3, tm_w1, s)
               : launch_one<false, true, true>(p, grid, tm_a, tm_w1, tm_w3, tm_sw1, tm_sw3, tm_w1, s);
  return fp8 ? launch_one<true, true, false>(p, grid, tm_a, tm_w1, tm_w3, tm_sw1, tm_sw3, tm_w1, s)
             : launch_one<false, true, false>(p, grid, tm_a, tm_w1, tm_w3, tm_sw1, tm_sw3, tm_w1, s);
}

cudaError_t launch_gemm2(const GemmParams& p, bool fp8, bool pair, int grid, const AMaps& tm_a,
                         const CUtensorMap& tm_w2, const CUtensorMap& tm_w2h, const CUtensorMap& tm_sw2,
                         const CUtensorMap& tm_sw2h, const CUtensorMap* tm_y, cudaStream_t s) {
  if (fp8 && tm_y) {
    return pair ? launch_one<true, false, true, true>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, *tm_y, s)
                : launch_one<true, false, false, true>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, *tm_y, s);
  }
  const CUtensorMap& unused = tm_w2;
  if (pair)
    return fp8 ? launch_one<true, false, true>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, unused, s)
               : launch_one<false, false, true>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, unused, s);
  return fp8 ? launch_one<true, false, false>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, unused, s)
             : launch_one<false, false, false>(p, grid, tm_a, tm_w2, tm_w2h, tm_sw2, tm_sw2h, unused, s);
}

}  // namespace moe

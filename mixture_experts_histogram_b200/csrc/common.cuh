// Shared declarations of the CUDA library: kernel parameter blocks, the
// workspace layout, and the host-side launch functions of each kernel family.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kTileM = 128;          // rows (tokens) per expert-GEMM tile
constexpr int kStageBytesK = 128;    // K extent of one pipeline stage, in bytes (one 128B swizzle row)
constexpr int kHistChunk = 256;      // tokens per histogram/scatter CTA
constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 16;
// Workspace status block: status word, first-timeout record (site, block,
// progress), and the per-block counters of MOE_DEBUG_STATE builds.
constexpr size_t kStatusBytes = 16384;

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Where each scratch buffer lives inside the caller's workspace (byte offsets
// from its base; every buffer starts on a 1024-byte boundary).
struct WsLayout {
  int64_t T, R, rows_pad, chunks, ksplit;
  size_t status, idx, gate, logits_part, chunk_base, counts, offsets, mt_prefix, mp_prefix;
  size_t perm, pos, row_gate, xp, sxp, h, sh, y, part, x_stage, out_stage, total;
};

WsLayout ws_layout(const moe_config& c, int64_t T, int num_sms);

// ---- router (logits GEMM on tcgen05 + top-k/softmax) ----
struct RouterParams {
  int32_t T, H, E;
  int32_t nbox;         // B boxes per stage (1 or 2)
  int32_t box_rows;     // rows per B box (multiple of 16, <= 256)
  int32_t ksplit;       // K splits (grid.y)
  int32_t kstages;      // total K stages (H / 64)
  float* partial;       // [ksplit, T, E] fp32 (unfused)
  int* status;
  // Fused top-k (ksplit == 1): the epilogue selects and writes idx/gate itself.
  int32_t fused, k;
  const float* bias;    // [E] or null
  int32_t* idx;         // [T, k]
  float* gate;          // [T, k]
  float* logits;        // [T, E] or null
};

struct TopkParams {
  int32_t T, E, k, ksplit;
  const float* partial;     // [ksplit, T, E]
  const float* bias;        // [E] or null
  int32_t* idx;             // [T, k]
  float* gate;              // [T, k]
  float* logits;            // [T, E] or null
};

// ---- histogram / scan / scatter ----
struct PermuteParams {
  int32_t T, E, k, S, G, chunks;
  // Expert parallelism: this call's groups are the routed experts
  // [e0, e0 + E) of the E_all the routing chose from, and the shared expert's
  // rows for tokens [sh_t0, sh_t1). Pairs routed to other experts are left out
  // (pos = -1) without an error; an index outside [0, E_all) latches
  // MOE_ERR_BAD_INDEX. One GPU: e0 = 0, E_all = E, [sh_t0, sh_t1) = [0, T).
  int32_t e0, E_all, sh_t0, sh_t1;
  const int32_t* idx;       // [T, k]
  const float* gate;        // [T, k] or null (row gates then not written)
  int32_t* chunk_base;      // [E, chunks]: per-chunk counts, then absolute row bases
  int32_t* counts;          // [G]
  int32_t* offsets;         // [G + 1]
  int32_t* mt_prefix;       // [G + 1] M-tile prefix (tiles of kTileM rows)
  int32_t* mp_prefix;       // [G + 1] pair-tile prefix (tiles of 2 kTileM rows, 2-SM GEMMs)
  int32_t* perm;            // [S T]
  int32_t* pos;             // [T, S]
  float* row_gate;          // [S T] or null
  int* status;
};

// ---- gather (+ E4M3 quantisation) ----
struct GatherParams {
  int32_t T, H, S;
  int64_t rows_pad;         // row stride of the transposed scale array
  const uint16_t* x;        // [T, H] bf16
  const int32_t* pos;       // [T, S] destination rows (null: row = token, S = 1)
  void* xp;                 // [rows, H] bf16 or E4M3
  float* sxp;               // FP8: scales, [H/128, rows_pad] (transposed) or [T, H/128]
  int32_t scale_row_major;  // 1: scales stored [T, H/128]
};

// ---- grouped expert GEMMs ----
struct GemmParams {
  const int32_t* mt_prefix;  // [G + 1] tile prefix (128-row tiles, or 256-row pair tiles)
  const int32_t* offsets;    // [G + 1]
  int32_t G, E;              // groups, routed experts (group E is the shared expert)
  int32_t K, N;              // reduction length; output width (I for GEMM1, H for GEMM2)
  int32_t n_tiles;           // output tiles per M tile
  int32_t n_fastest;         // item order: 1 = N tiles of a row tile adjacent, 0 = M tiles adjacent
  int32_t R;                 // total rows
  int64_t rows_pad;          // row stride of transposed activation scales
  const float* a_scale;      // FP8: [K/128, rows_pad]
  const float* b_scale0;     // FP8 routed scales (GEMM1: s1, GEMM2: s2)
  const float* b_scale1;     // FP8 routed scales (GEMM1: s3)
  const float* bs_scale0;    // FP8 shared-expert scales
  const float* bs_scale1;
  void* out;                 // GEMM1: h [R, N]; GEMM2: y [R, N] bf16
  float* out_scale;          // GEMM1 FP8: [N/128, rows_pad]
  const float* row_gate;     // GEMM2: [R]
  int* status;
  uint64_t wait_ns;          // limit of every bounded wait (normally 2 s)
  int32_t k_split;           // K pieces per tile (>= 1; > 1 only for GEMM2, with part)
  float* part;               // GEMM2 with k_split > 1: fp32 [k_split, R, N] piece sums, no gate
  int32_t raw_out;           // GEMM1 only: store the fp32 gate/up sums [R, 2N] instead of SwiGLU(h)
  int32_t inject;            // test hook: 1 = the producer issues no loads (the first wait runs out)
};

struct CombineParams {
  int32_t T, H, S;
  const uint16_t* y;         // [S T, H] bf16
  const int32_t* pos;        // [T, S]
  uint16_t* out;             // [T, H] bf16
};

// Counts a kernel launch of this library when `e` is cudaSuccess (read with
// moe_launch_count) and returns `e`. Every launcher returns through it.
cudaError_t counted_launch(cudaError_t e);

// Launches `kern` on `s` with programmatic stream serialization (the kernel
// calls pdl_wait() before its first global-memory access; see ptx.cuh) and, for
// cluster_x > 1, clusters of cluster_x CTAs along x. Counted like every launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = (unsigned)n;
  return counted_launch(cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...));
}

// Host launchers (each returns the launch's cudaError_t).
cudaError_t launch_router_gemm(const RouterParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_w,
                               cudaStream_t s);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
cudaError_t launch_permute_one_chunk(const PermuteParams& p, cudaStream_t s);  // T <= 256
cudaError_t launch_histogram(const PermuteParams& p, cudaStream_t s);
cudaError_t launch_scan(const PermuteParams& p, cudaStream_t s);
cudaError_t launch_scatter(const PermuteParams& p, cudaStream_t s);
cudaError_t launch_gather(const GatherParams& p, bool fp8, cudaStream_t s);
// pair: run the 2-SM (CTA pair, M = 256) variant; p.mt_prefix must then be the
// pair-tile prefix and `grid` even.
// Activation (A) tensor maps of one grouped GEMM: the same rows with 128-, 64-
// and 32-row boxes. A tile loads the smallest box that covers its group's rows
// (decode tiles hold one or two rows; a group's last tile is often short); the
// MMA still reads 128 rows, and the rows past the box only feed output rows that
// are never stored.
struct AMaps {
  CUtensorMap rows128, rows64, rows32;
};

// NVFP4 weight tensor maps of one grouped GEMM (uint8, no swizzle): E2M1
// codes [rows, K/2] with 32-byte boxes (one 64-deep K stage) and E4M3 scales
// [rows, K/16] with 16-byte boxes (four stages). GEMM1: code0/scale0 = W1,
// code1/scale1 = W3 (128-row boxes); GEMM2: code0/scale0 = W2 (256-row boxes).
// The s-prefixed maps are the shared expert's.
struct NvMaps {
  CUtensorMap code0, code1, scode0, scode1, scale0, scale1, sscale0, sscale1;
};

// NVFP4 (W4A16) grouped GEMM, single CTAs: GEMM1 (gate/up + SwiGLU, bf16 h) or
// GEMM2 (down, bf16 y). Global scales: GEMM1 b_scale0/b_scale1 = W1/W3 [E],
// bs_scale0/bs_scale1 = the shared expert's [1]; GEMM2 b_scale0 = W2 [E],
// bs_scale0 = the shared expert's.
cudaError_t launch_nvfp4_gemm(const GemmParams& p, bool gemm1, int grid, const AMaps& tm_a, const NvMaps& tm,
                              cudaStream_t s);

cudaError_t launch_gemm1(const GemmParams& p, bool fp8, bool pair, int grid, const AMaps& tm_a,
                         const CUtensorMap& tm_w1, const CUtensorMap& tm_w3, const CUtensorMap& tm_sw1,
                         const CUtensorMap& tm_sw3, cudaStream_t s);
// tm_w2 / tm_sw2 use 256-row boxes, tm_w2h / tm_sw2h the same tensors with 128-row boxes;
// tm_y (FP8 only; null: per-row stores) maps y [R, N] bf16 with 32-row x 64-column
// 128B-swizzled boxes: the tiles then leave through shared memory and TMA stores.
// The NVFP4 GEMMs for decode-sized groups (nvfp4_gemm_swap.cu): weights expanded
// into TMEM as the MMA's A operand, a group's rows as N in 32-row chunks; maps
// and parameters as for launch_nvfp4_gemm (p.mt_prefix not used).
cudaError_t launch_nvfp4_swap(const GemmParams& p, bool gemm1, int grid, const AMaps& tm_a, const NvMaps& tm,
                              cudaStream_t s);
// The swapped-operand FP8 GEMMs for decode-sized groups (grouped_gemm_swap.cu):
// GEMM1 (gemm1: b0/b1 = W1/W3 with 128-row boxes) or GEMM2 (b0 = W2 with
// 256-row boxes); p.mt_prefix is not used (the kernel derives its 32-row chunks
// from p.offsets); tm_a.rows32 must map the A rows.
cudaError_t launch_gemm_swap(const GemmParams& p, bool gemm1, int grid, const AMaps& tm_a, const CUtensorMap& b0,
                             const CUtensorMap& b1, const CUtensorMap& bs0, const CUtensorMap& bs1, cudaStream_t s);
cudaError_t launch_gemm2(const GemmParams& p, bool fp8, bool pair, int grid, const AMaps& tm_a,
                         const CUtensorMap& tm_w2, const CUtensorMap& tm_w2h, const CUtensorMap& tm_sw2,
                         const CUtensorMap& tm_sw2h, const CUtensorMap* tm_y, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);
// Expert parallelism: a rank's fp32 partial output, the sum of each token's
// expert rows that this rank computed (pos < 0 left out), in slot order.
cudaError_t launch_ep_partial(int64_t T, int32_t H, int32_t S, const void* y, const int32_t* pos, float* part,
                              cudaStream_t s);
// Stage entry point helpers: tile prefixes of caller-given group offsets, and
// FP8 scales between row-major [R, nb] and transposed [nb, rows_pad].
cudaError_t launch_tile_prefix(const int32_t* offsets, int32_t G, int32_t R, int32_t* mt, int32_t* mp, int* status,
                               cudaStream_t s);
// y [R, N] bf16 = row_gate[r] * (sum over pieces kp in order of part[kp, r, :])
// for the rows r < min(*rows_end, R); nothing when *status is set.
cudaError_t launch_split_reduce(const float* part, int32_t k_split, int64_t R, int32_t N, const int32_t* rows_end,
                                const float* row_gate, const int* status, void* y, cudaStream_t s);
cudaError_t launch_scale_transpose(const float* src, float* dst, int64_t R, int32_t nb, int64_t rows_pad,
                                   bool to_transposed, cudaStream_t s);

}  // namespace moe

/*
 * C ABI of the B200 routed Mixture-of-Experts layer forward (sm_100a).
 *
 * The layer (NeMo AutoModel "Step-5-Preview" page, "Model Architecture" table):
 * hidden H = 4,096; a learned router over E = 352 routed experts with top-k = 8
 * routing and one always-on shared expert; every expert a SwiGLU MLP with
 * intermediate size I = 1,536. Expert weights are BF16, or FP8 E4M3 with one
 * fp32 scale per 128x128 block (StepFun "Step-5 minimal inference" README:
 * "block-scaled FP8 expert GEMM"; expert storage follows the checkpoint's
 * quantization_config). The MoE primitives around the expert GEMMs (routing,
 * the token->expert histogram and permutation, the combine) are the same
 * README's "critical MoE primitives".
 *
 * What one call computes, per token t:
 *   l      = x[t] . Wr^T (+ b)                 fp32 logits over the E experts
 *   top-k  = the k largest logits, ties to the lower expert index,
 *            in descending order; g = softmax(l) over the chosen k, renormalised
 *   y_e    = (silu(a W1_e^T) * (a W3_e^T)) W2_e^T   for the k chosen experts
 *            and the shared expert; a = x[t] (BF16 storage) or its 1x128-block
 *            E4M3 quantisation (FP8 storage: scale = blockmax/448)
 *   out[t] = sum_j g_j y_{e_j} + y_shared      summed in fp32 in slot order,
 *                                              rounded once to bf16
 *
 * Conventions for every entry point:
 *  - Layouts are row-major and C-contiguous. Weights are in nn.Linear order
 *    ([out, in], the reduction dimension contiguous):
 *      router_w [E, H] bf16;  w1, w3 [E, I, H];  w2 [E, H, I];
 *      FP8 scales s1, s3 [E, I/128, H/128] fp32;  s2 [E, H/128, I/128] fp32;
 *      the shared expert's sw1, sw3, sw2 (and ss1, ss3, ss2) have the same
 *      layouts with E = 1.
 *  - "Device" pointers are CUDA device memory of the current device; the
 *    caller owns every buffer. The library allocates no device memory per
 *    call: all scratch comes from the caller's workspace (size:
 *    moe_workspace_bytes), except moe_permute_noalloc's fixed 1 MiB
 *    file-scope device array, which every GPU that loads the library holds.
 *  - Calls are asynchronous on `stream` unless stated. Argument errors are
 *    returned synchronously; errors found on the device (a bad expert index,
 *    a timed-out wait) are latched in a status word inside the workspace and
 *    read with moe_read_status.
 *  - Device buffers must be 16-byte aligned (TMA); 256-byte alignment is
 *    recommended. The workspace must be 256-byte aligned.
 *  - Supported shapes: H and I multiples of 128; 1 <= E <= 512;
 *    1 <= top_k <= min(E, 16); n_shared in {0, 1}; 0 <= T, (top_k+n_shared)*T < 2^31.
 *    T == 0 is a no-op that returns MOE_OK.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

/* Expert weight storage. */
enum {
  MOE_WDTYPE_BF16 = 0,     /* bf16 weights, bf16 activations */
  MOE_WDTYPE_FP8_E4M3 = 1, /* E4M3 weights with 128x128 fp32 block scales, E4M3 1x128 activations */
  MOE_WDTYPE_NVFP4 = 2     /* NVFP4 weights, bf16 activations (W4A16; see moe_weights) */
};

/* Status codes (returned, or latched on the device). */
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, bad config or size */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* a shape outside the supported set */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,
  MOE_ERR_CUDA = 4,               /* a CUDA runtime call failed (no device, launch error, ...) */
  MOE_ERR_BAD_INDEX = 5,          /* device: an expert index outside [0, E) was skipped */
  MOE_ERR_DEVICE_TIMEOUT = 6,     /* device: a bounded wait gave up; results are invalid */
  MOE_ERR_MISALIGNED = 7          /* a buffer is not 16-byte (workspace: 256-byte) aligned */
};

typedef struct moe_config {
  int32_t hidden;     /* H */
  int32_t n_experts;  /* E, routed experts */
  int32_t top_k;      /* k */
  int32_t n_shared;   /* 0 or 1 always-on shared expert */
  int32_t inter;      /* I, expert intermediate size */
  int32_t wdtype;     /* MOE_WDTYPE_* */
} moe_config;

/* Device pointers to one layer's weights (see the layouts above). Scale
 * pointers are used only for MOE_WDTYPE_FP8_E4M3 and MOE_WDTYPE_NVFP4;
 * shared-expert pointers only when n_shared == 1. router_bias may be NULL (no
 * bias).
 * MOE_WDTYPE_NVFP4 (TensorFold PR page: the NVFP4 format its W4A16 linears
 * read; a variant the pages describe for another model): every expert matrix
 * [n, k] is stored as E2M1 codes [n, k/2] uint8, two per byte with input 2j in
 * the low nibble of byte j (w1/w3/w2 point to them), E4M3 scales [n, k/16]
 * uint8, one per 16 inputs (s1/s3/s2), and one fp32 global scale per matrix
 * (g1/g3/g2 [E]; the shared expert's sg1/sg3/sg2 [1]); an element is
 * e2m1 x e4m3 x global. Activations and h stay bf16. Needs H and I multiples
 * of 256. */
typedef struct moe_weights {
  const void* router_w;
  const float* router_bias;
  const void* w1;
  const void* w3;
  const void* w2;
  const float* s1;
  const float* s3;
  const float* s2;
  const void* sw1;
  const void* sw3;
  const void* sw2;
  const float* ss1;
  const float* ss3;
  const float* ss2;
  const float* g1; /* NVFP4 global scales [E] */
  const float* g3;
  const float* g2;
  const float* sg1; /* NVFP4 global scales of the shared expert [1] */
  const float* sg3;
  const float* sg2;
} moe_weights;

/* Bytes of workspace that moe_forward (and every stage entry point) needs for
 * T tokens. Host only; touches no device. */
MOE_API int moe_workspace_bytes(const moe_config* cfg, int64_t T, size_t* bytes);

/*
 * The whole layer forward: router + top-k, histogram/scan/permute, grouped
 * expert GEMMs (gate/up with fused SwiGLU, then down), combine.
 *   x        [T, H] bf16, device
 *   out      [T, H] bf16, device (written)
 *   topk_idx [T, k] int32 and topk_w [T, k] fp32, device, optional (NULL): if
 *            given, the routing decision is written there as well.
 */
MOE_API int moe_forward(const moe_config* cfg, int64_t T, const void* x, const moe_weights* w, void* out,
                int32_t* topk_idx, float* topk_w, void* workspace, size_t workspace_bytes,
                moe_stream_t stream);

/*
 * moe_forward from host memory: copies x_host [T, H] bf16 to the device,
 * runs the layer and copies the result into out_host [T, H] bf16; weights and
 * workspace are device memory. Synchronous: returns after out_host is written
 * (pinned host buffers make the copies asynchronous DMA).
 */
MOE_API int moe_forward_host(const moe_config* cfg, int64_t T, const void* x_host, const moe_weights* w,
                     void* out_host, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_forward_host without the final synchronisation: the copy in, the layer
 * and the copy out are queued on `stream` and the call returns. x_host and
 * out_host must stay valid (and should be pinned) until the stream has passed
 * the copy out (cudaStreamSynchronize or an event). A caller that alternates
 * two workspaces and two streams overlaps one step's copies with the other
 * step's kernels; each step still copies its own input in and its output out.
 */
MOE_API int moe_forward_host_async(const moe_config* cfg, int64_t T, const void* x_host, const moe_weights* w,
                                   void* out_host, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---- stage entry points (each a part of moe_forward, for tests and tools) ---- */

/* Router: fp32 logits, top-k selection and renormalised gates.
 * logits [T, E] fp32 (optional): the fp32 logits including the bias. */
MOE_API int moe_route(const moe_config* cfg, int64_t T, const void* x, const void* router_w,
              const float* router_bias, int32_t* topk_idx, float* topk_w, float* logits,
              void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Activation quantisation of x [T, H] bf16 into E4M3 codes q [T, H] and fp32
 * scales s [T, H/128] (one per 1x128 row block, scale = blockmax/448; an
 * all-zero block gets scale 1 and zero codes). */
MOE_API int moe_quantize_act(int64_t T, int32_t hidden, const void* x, uint8_t* q, float* s, moe_stream_t stream);

/* Histogram/scan/permute of a routing decision. Groups 0..E-1 are the routed
 * experts, group E the shared expert (all T tokens) when n_shared == 1.
 *   counts  [E+S] int32    rows per group
 *   offsets [E+S+1] int32  exclusive scan of counts
 *   perm    [(k+S)T] int32 token of each row; rows of a group ascend by token
 *   pos     [T, k+S] int32 row of (token, slot); slot k is the shared row
 * An out-of-range index latches MOE_ERR_BAD_INDEX and its pair is skipped. */
MOE_API int moe_permute(const moe_config* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts,
                int32_t* offsets, int32_t* perm, int32_t* pos, void* workspace, size_t workspace_bytes,
                moe_stream_t stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: a plugin whose host framework owns all device memory, a serving loop
 * that reserved its memory up front, or a latency-critical path that cannot
 * afford an allocation. The pages describe no such entry point; it is a
 * property of this library, not of the layer.
 * Same inputs, outputs and results as moe_permute. Its scratch is a fixed
 * 1 MiB device array inside the library (every GPU that loads the library
 * holds it until the process exits), so E * ceil(T / 256) must not exceed
 * 260,032 (T <= 188,928 tokens at E = 352); larger sizes return
 * MOE_ERR_UNSUPPORTED_SHAPE without touching the device.
 * device_status (optional, device memory, one int) receives the device status
 * (MOE_ERR_BAD_INDEX for skipped pairs); the call zeroes it first. Without it
 * the status word lives in the shared scratch, where no entry point can read
 * it: a caller that needs to detect bad indices must pass device_status.
 * The first call with a given device current looks up the scratch address on
 * that device; make that first call before any stream capture. Every call
 * shares the one scratch array per device: calls whose work overlaps on the
 * GPU (other streams, other threads) race and must be serialised by the
 * caller. The call allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine. */
MOE_API int moe_permute_noalloc(const moe_config* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts,
                                int32_t* offsets, int32_t* perm, int32_t* pos, int* device_status,
                                moe_stream_t stream);

/* Expert MLPs for a given routing: permute, gather (+ quantise), gate/up GEMM
 * with SwiGLU, down GEMM. y [(k+S)T, H] bf16 receives each row's expert output
 * times its gate (1 for shared rows); pos [T, k+S] receives the row of each
 * (token, slot). */
MOE_API int moe_experts(const moe_config* cfg, int64_t T, const void* x, const int32_t* topk_idx,
                const float* topk_w, const moe_weights* w, void* y, int32_t* pos, void* workspace,
                size_t workspace_bytes, moe_stream_t stream);

/* One grouped expert GEMM over rows already grouped by expert (the GEMMs of
 * moe_experts, for tests and tools). Rows [offsets[g], offsets[g+1]) of A belong
 * to group g (routed experts 0..E-1, then the shared expert when n_shared == 1);
 * offsets [E+S+1] int32 (device) must start at 0, never decrease and end at most
 * at R (otherwise MOE_ERR_INVALID_ARG is latched in the workspace status and
 * nothing is computed). Rows past offsets[E+S] are not written.
 *   stage MOE_STAGE_GATE_UP:     A [R, H]; out = h [R, I] = silu(A W1_g^T) * (A W3_g^T),
 *                                bf16 (BF16 storage) or E4M3 codes with out_scale
 *                                [R, I/128] fp32 (FP8: 1x128 blocks, scale = blockmax/448)
 *   stage MOE_STAGE_GATE_UP_RAW: A [R, H]; out = fp32 [R, 2, I]: the gate sums
 *                                A W1_g^T, then the up sums A W3_g^T (no SwiGLU)
 *   stage MOE_STAGE_DOWN:        A [R, I]; out = y [R, H] bf16 = row_gate[r] * (A W2_g^T)
 *                                (row_gate [R] fp32, device; NULL means 1)
 * A is bf16 (BF16 storage) or E4M3 codes with a_scale [R, K/128] fp32 (FP8, K
 * the reduction length). The workspace is moe_workspace_bytes for
 * ceil(R / (top_k + n_shared)) tokens. Device status: moe_read_status. */
enum { MOE_STAGE_GATE_UP = 1, MOE_STAGE_GATE_UP_RAW = 2, MOE_STAGE_DOWN = 3 };
MOE_API int moe_grouped_gemm(const moe_config* cfg, int stage, int64_t R, const int32_t* offsets, const void* a,
                             const float* a_scale, const moe_weights* w, const float* row_gate, void* out,
                             float* out_scale, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Combine: out[t] = sum over slots j < k+S of y[pos[t, j]], fp32 in slot
 * order, rounded once to bf16. y [(k+S)T, H] bf16, pos [T, k+S], out [T, H]. */
MOE_API int moe_combine(const moe_config* cfg, int64_t T, const void* y, const int32_t* pos, void* out,
                moe_stream_t stream);

/* ---- expert parallelism (StepFun "Step-5 minimal inference" README: the
 * deployment at TP = EP = 8 places 44 of the 352 routed experts on each GPU,
 * tokens replicated over the group; "Long-output stability": the ranks'
 * partial results are added in rank order with FP32 accumulation) ---- */

/* One rank's share of the layer. cfg->n_experts is the number of routed
 * experts the router chooses from (all ranks'); this rank computes its routed
 * experts [e0, e1) and, when cfg->n_shared == 1, the shared expert for tokens
 * [shared_t0, shared_t1) (the shared expert is replicated on every rank and
 * its rows divided by token). Every token is routed over all experts:
 *   w->router_w [E, H], w->router_bias [E] or NULL: all experts;
 *   w->w1, w->w3 [e1-e0, I, H], w->w2 [e1-e0, H, I] (+ FP8 scales): this
 *     rank's experts only, expert e0 first; shared-expert weights: whole.
 * partial [T, H] fp32 (device, written): for each token, the sum in slot order
 * of the gate-weighted rows this rank computed (zero where it computed none),
 * not rounded to bf16. Summing the ranks' partials over a partition of the
 * experts and of the shared expert's tokens gives the layer output
 * (moe_ep_reduce). topk_idx / topk_w as for moe_forward. The workspace is
 * moe_workspace_bytes(cfg, T) (the whole layer's). Requires 0 <= e0 < e1 <= E. */
MOE_API int moe_forward_ep_partial(const moe_config* cfg, int64_t T, const void* x, const moe_weights* w,
                                   int32_t e0, int32_t e1, int64_t shared_t0, int64_t shared_t1, float* partial,
                                   int32_t* topk_idx, float* topk_w, void* workspace, size_t workspace_bytes,
                                   moe_stream_t stream);

/* The ranks' partial outputs added in rank order: for t in [t0, t1),
 * out[t] = bf16(partials[0][t] + partials[1][t] + ... + partials[n-1][t]),
 * summed in fp32 in that order and rounded once (nearest even).
 * partials: a host array of n_ranks (1..16) device pointers to [T, H] fp32
 * buffers that this device can read (its own memory, or peers' memory mapped
 * for peer access); out [T, H] bf16 (device; rows outside [t0, t1) untouched).
 * All pointers 16-byte aligned; H a multiple of 128. */
MOE_API int moe_ep_reduce(int32_t n_ranks, const float* const* partials, int64_t T, int32_t hidden, int64_t t0,
                          int64_t t1, void* out, moe_stream_t stream);

/* ---- the fp32 residual stream around the layer ----
 * (NeMo "Step-5-Preview" page, "Full-Depth H100 Benchmark" table: FP32 norms and
 * residuals.) The norm's type is not stated there; these follow the usual
 * decoder reading: RMS normalisation without mean subtraction or bias. */

/* x[t] = bf16(r[t] / sqrt(mean_h(r[t, h]^2) + eps) * weight), computed in fp32
 * (IEEE sqrt and division), rounded once to bf16: the layer's input.
 * residual [T, H] fp32, weight [H] fp32, x_bf16 [T, H] bf16 (device, 16-byte
 * aligned); H a multiple of 128; eps >= 0. */
MOE_API int moe_rmsnorm(int64_t T, int32_t hidden, const float* residual, const float* weight, float eps,
                void* x_bf16, moe_stream_t stream);

/* The combine with the residual add: r_out[t] = r[t] + sum over slots j of
 * y[pos[t, j]], the rows summed in fp32 in slot order and added to r in fp32
 * (no bf16 rounding of the layer output). y and pos as for moe_combine (rows
 * with pos < 0 are skipped); residual, residual_out [T, H] fp32, which may be
 * the same buffer. */
MOE_API int moe_combine_residual(const moe_config* cfg, int64_t T, const void* y, const int32_t* pos,
                const float* residual, float* residual_out, moe_stream_t stream);

/* ---- status and profiling ---- */

/* Synchronises `stream`, then returns the device status latched in the
 * workspace since the last moe_* call that cleared it (every moe_forward,
 * moe_route, moe_permute and moe_experts call clears it first). */
MOE_API int moe_read_status(const void* workspace, moe_stream_t stream, int* device_status);

/* Synchronises `stream`, then copies the workspace's status record:
 * detail[0] = status word (as moe_read_status); for MOE_ERR_DEVICE_TIMEOUT,
 * detail[1] = the wait site of the first timeout (kernel variant and wait:
 * nonzero), detail[2] = its block index, detail[3] = that wait's progress
 * counter. */
MOE_API int moe_read_status_detail(const void* workspace, moe_stream_t stream, int* detail /* [4] */);

/* Test hook of the bounded waits (process-wide; not for production use).
 * MOE_INJECT_GEMM_NO_LOADS makes the expert GEMMs' producer issue no loads, so
 * their consumers' first waits run out after wait_limit_ns and the call latches
 * MOE_ERR_DEVICE_TIMEOUT with nothing in flight: every kernel still returns and
 * the device stays usable. wait_limit_ns bounds every wait of the expert GEMMs
 * (0 restores the default of 2 s). MOE_INJECT_NONE with 0 restores normal
 * operation. */
enum { MOE_INJECT_NONE = 0, MOE_INJECT_GEMM_NO_LOADS = 1 };
MOE_API int moe_debug_inject(int what, uint64_t wait_limit_ns);

/* Text for a status code (static storage). */
MOE_API const char* moe_status_string(int status);

/* Per-kernel timing of moe_forward: when enabled, moe_forward records a CUDA
 * event before and after each of its kernels on its stream. */
MOE_API int moe_profile_enable(int enable);

/* Synchronises on the last recorded event and writes the kernel times (ms) of
 * the most recent profiled moe_forward into ms[0..n); *n_out = number of
 * kernels. Names come from moe_profile_kernel_name. */
MOE_API int moe_profile_read(float* ms, int n, int* n_out);
MOE_API const char* moe_profile_kernel_name(int i);

/* Expert-GEMM variant (process-wide; default MOE_GEMM_AUTO). SINGLE runs one
 * CTA per 128-row tile; PAIR runs 2-SM CTA pairs on 256-row tiles (each weight
 * tile crosses L2 -> SM once per 256 rows; NVFP4 runs SINGLE); SWAP (FP8 and
 * NVFP4 storage; BF16 runs SINGLE) makes the weight rows the MMA's M side and
 * runs each group in chunks of 32 rows, for decode-sized groups (NVFP4: the
 * weights expanded into tensor memory). AUTO runs both FP8 GEMMs swapped when
 * n_experts <= top_k * T <= 16 * n_experts and both NVFP4 GEMMs swapped when
 * top_k * T <= 16 * n_experts, else the gate/up GEMM on pairs when
 * top_k * T >= 128 * n_experts (routed groups of 128+ rows on average) and
 * everything else on single CTAs. The stage entry point applies the same rules
 * with its R rows and n_experts + n_shared groups. All variants compute the
 * same layer and are held to the same tolerance by the tests. */
enum { MOE_GEMM_AUTO = 0, MOE_GEMM_SINGLE = 1, MOE_GEMM_PAIR = 2, MOE_GEMM_SWAP = 3 };
MOE_API int moe_set_gemm_variant(int variant);

/* Kernels this library has launched in this process so far (every entry
 * point, every device); the difference across a region counts its launches. */
MOE_API int moe_launch_count(uint64_t* n);

/* Number of streaming multiprocessors the kernels size their grids for
 * (current device). */
MOE_API int moe_device_sm_count(int* sms);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

// moe_permute_noalloc: the histogram/scan/permute of moe_permute for callers
// that cannot allocate device memory.
//
// Who needs it: code that runs where device allocation is off limits or too
// costly -- a plugin inside a host framework that owns all device memory and
// forbids cudaMalloc, a serving loop whose memory was reserved up front, or a
// latency-critical path where an allocation (and the device synchronisation
// cudaMalloc/cudaFree can imply) is not acceptable. moe_permute asks such a
// caller for a workspace; this entry point needs none. Its scratch is a
// file-scope device array of fixed size that every GPU loading the library
// holds until the process exits.
//
// The kernels are the ones moe_permute launches; only where their scratch lives
// differs.
#include <mutex>

#include "common.cuh"
#include "moe.h"

namespace moe {

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB per device
constexpr size_t kStatusOff = 0;                     // int status word (256 B reserved)
constexpr size_t kMtOff = 256;                       // int [G + 1], G <= 513
constexpr size_t kMpOff = kMtOff + 4096;             // int [G + 1]
constexpr size_t kChunkOff = kMpOff + 4096;          // int [E, ceil(T / 256)]
constexpr size_t kChunkInts = (kScratchBytes - kChunkOff) / 4;
constexpr int kMaxDevices = 64;

// Scratch of moe_permute_noalloc. In host code this name is only a stand-in for
// the symbol, never a device address: the address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).
int scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED_SHAPE;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_ptr[dev]);
  return MOE_OK;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_permute_noalloc(const moe_config* cfg, int64_t T, const int32_t* topk_idx, int32_t* counts,
                                   int32_t* offsets, int32_t* perm, int32_t* pos, int* device_status,
                                   moe_stream_t stream) {
  if (!cfg || T < 0) return MOE_ERR_INVALID_ARG;
  if (cfg->n_experts <= 0 || cfg->top_k <= 0 || cfg->n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared > 1 || cfg->n_experts > kMaxExperts || cfg->top_k > kMaxTopK || cfg->top_k > cfg->n_experts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)(cfg->top_k + cfg->n_shared) * T >= ((int64_t)1 << 31) - 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!topk_idx || !counts || !offsets || !perm || !pos) return MOE_ERR_INVALID_ARG;
  const int64_t chunks = ceil_div(T > 0 ? T : 1, kHistChunk);
  // The per-chunk expert counts must fit in the static scratch.
  if ((int64_t)cfg->n_experts * chunks > (int64_t)kChunkInts) return MOE_ERR_UNSUPPORTED_SHAPE;

  unsigned char* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = device_status ? device_status : reinterpret_cast<int*>(scratch + kStatusOff);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  const int G = cfg->n_experts + cfg->n_shared;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, (size_t)G * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(offsets, 0, (size_t)(G + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  PermuteParams pp{};
  pp.T = (int32_t)T;
  pp.E = cfg->n_experts;
  pp.k = cfg->top_k;
  pp.S = cfg->n_shared;
  pp.G = G;
  pp.e0 = 0;
  pp.E_all = cfg->n_experts;
  pp.sh_t0 = 0;
  pp.sh_t1 = (int32_t)T;
  pp.chunks = (int32_t)chunks;
  pp.idx = topk_idx;
  pp.gate = nullptr;
  pp.chunk_base = reinterpret_cast<int32_t*>(scratch + kChunkOff);
  pp.counts = counts;
  pp.offsets = offsets;
  pp.mt_prefix = reinterpret_cast<int32_t*>(scratch + kMtOff);
  pp.mp_prefix = reinterpret_cast<int32_t*>(scratch + kMpOff);
  pp.perm = perm;
  pp.pos = pos;
  pp.row_gate = nullptr;
  pp.status = status;
  if (launch_histogram(pp, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_scan(pp, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_scatter(pp, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

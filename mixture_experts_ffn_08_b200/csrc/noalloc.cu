// moe_permute_noalloc: the dispatch stage (pairs bucketed by expert, x rows gathered)
// for callers that cannot give the library any device memory of its own.
//
// Who needs it: code that runs inside a host framework which owns every byte of device
// memory and offers no scratch hook to plug-ins, and latency-critical serving loops
// where a cudaMalloc (which can synchronise the device) or a pooled-allocator round
// trip is not allowed between launches.  Such callers can pass their inputs and
// outputs, but not a workspace.
//
// The only scratch the permute kernels need is the per-chunk expert histogram (one
// int32 per 256-pair chunk and expert).  Here it lives in a fixed, file-scope device
// array instead of the caller's workspace:
//   * size: kNoAllocScratchInts int32 = 1 MiB, loaded with the library on every GPU
//     that uses it and held until the process exits;
//   * calls whose ceil(T*K/256) * E exceeds that are rejected (MOE_ERR_UNSUPPORTED);
//   * every call shares the one array, so two calls that overlap on the GPU (different
//     streams, or different host threads on one device) race and corrupt each other;
//     serialise them on one stream.  The histogram is fully rewritten by each call, so
//     nothing in it has to start at zero; the caller's status word is cleared by the
//     caller.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {
namespace {

constexpr long long kNoAllocScratchInts = 1LL << 18;  // 1 MiB of int32

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

// Device address of g_permute_scratch for each device.  In host code the array's name
// only stands in for the symbol; the address must come from cudaGetSymbolAddress with
// the device current.  Looked up on the first call made on each device.
std::mutex g_mu;
int32_t* g_addr[64] = {nullptr};

moe_status_t scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_permute_scratch) != cudaSuccess || ptr == nullptr)
      return MOE_ERR_CUDA;
    g_addr[dev] = static_cast<int32_t*>(ptr);
  }
  *out = g_addr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const moe_params_t* p, const int32_t* topk_ids,
                                            const void* x, const float* x_scale, int32_t* counts,
                                            int32_t* offsets_padded, int32_t* row_of_pair,
                                            int32_t* pair_of_row, void* x_perm,
                                            float* x_perm_scale, int32_t* device_status,
                                            void* stream) {
  using namespace moe;
  if (moe_max_padded_rows(p) < 0) return MOE_ERR_INVALID_ARG;  // same parameter checks as moe_permute
  const bool empty = p->T == 0;  // same empty-batch rule as moe_permute
  if ((!empty && (!topk_ids || !x || !row_of_pair)) || !counts || !offsets_padded || !pair_of_row || !x_perm)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  if (act_e4m3(*p) && ((!empty && !x_scale) || !x_perm_scale)) return MOE_ERR_INVALID_ARG;
  const long long pairs = static_cast<long long>(p->T) * p->K;
  const long long chunks = (pairs + kPermChunk - 1) / kPermChunk;
  if ((chunks > 0 ? chunks : 1) * p->E > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  const moe_status_t s = scratch_for_current_device(&scratch);
  if (s != MOE_OK) return s;
  const cudaError_t e = launch_permute(*p, moe_effective_block_m(p), topk_ids, x, x_scale, counts, offsets_padded, row_of_pair,
                                       pair_of_row, x_perm, x_perm_scale, scratch, device_status,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

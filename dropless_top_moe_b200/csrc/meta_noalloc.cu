// Dispatch metadata without a caller workspace (moe_dispatch_meta_noalloc).
//
// Some callers cannot call cudaMalloc: code embedded in another runtime that
// owns all device memory and gives its plugins no allocator, or a
// latency-critical path where an allocation (which may synchronise the
// device) is not allowed.  This entry point keeps the metadata kernels'
// scratch (per-chunk expert counts and the per-expert starts) in a fixed
// file-scope device array instead of a workspace.  The caller still passes
// every input and output.
//
// The array is sized for n_chunks * E <= kNoAllocChunkExperts, where
// n_chunks = ceil(N / 128) chunks of 128 tokens; with E = 256 that is
// N <= 131,072 tokens.  Every device that loads the library holds the array
// (about 1 MB) until exit.
#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr int kNoAllocChunkExperts = 262144;
constexpr int kNoAllocScratchInts = kNoAllocChunkExperts + 2 * 256;

// Shared by every call on a device; keeps the last call's contents.
__device__ __align__(256) int32_t g_meta_scratch[kNoAllocScratchInts];

}  // namespace

extern "C" moe_status moe_dispatch_meta_noalloc(const int32_t* top_experts, int32_t N, int32_t K,
                                                int32_t E, int32_t* indices, int32_t* bin_ids,
                                                int32_t* bins, int32_t* padded_bins, int32_t* pos,
                                                int32_t* status, moe_stream_t stream) {
  if (N < 0 || K <= 0 || E <= 0 || K > E) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  if (!padded_bins || (N > 0 && (!top_experts || !pos))) return MOE_ERR_INVALID_ARG;
  if (moe::meta_workspace_bytes(N, E) > sizeof(g_meta_scratch)) return MOE_ERR_WORKSPACE;
  // The array's name is a host-side stand-in, so the kernels get its device
  // address, looked up with the caller's device current.  The lookup runs on
  // every call (it allocates nothing and is cheap once the module is loaded):
  // an address kept from an earlier call could belong to a context that a
  // device reset has since destroyed.
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_meta_scratch) != cudaSuccess || scratch == nullptr) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  // The count kernel writes every chunk count (zeros included) and the scan
  // writes every start, so nothing in the array needs clearing first.
  return moe::dispatch_meta(top_experts, N, K, E, indices, bin_ids, bins, padded_bins, pos, scratch, status,
                            (cudaStream_t)stream, 0);
}

// Dispatch metadata: stable counting sort of the flat assignments by expert,
// histogram, inclusive cumsums, round-up of each group to 128 rows
// ("MegaBlocks - architecture", sec. 2.1/2.3 and sec. 4: the sort key is the
// expert id only, a few bits).
//
// A counting sort is the whole sort when keys are at most 8 bits wide:
//   1. count  - per chunk of 2048 assignments, a shared-memory histogram
//               (integer atomics: counts do not depend on their order);
//   2. scan   - one block turns the chunk counts into exclusive per-chunk
//               offsets per expert and forms bins / padded_bins;
//   3. place  - per chunk, assignments are visited in increasing flat id, in
//               rounds of 1024; within a warp the rank among equal experts
//               comes from __match_any_sync, across warps from a scan of the
//               per-warp counts.  Rank order = flat-id order: the sort is stable.
// Everything is integer work, so the outputs are exact and run-to-run equal.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kMetaChunk = 2048;
constexpr int kMetaPlaceThreads = 1024;

__global__ void __launch_bounds__(256)
meta_count_kernel(const int32_t* __restrict__ top, int64_t NK, int E, int32_t* __restrict__ chunk_counts,
                  int* status) {
  extern __shared__ int s_hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kMetaChunk;
  for (int j = threadIdx.x; j < kMetaChunk; j += blockDim.x) {
    const int64_t i = base + j;
    if (i >= NK) break;
    const int e = top[i];
    if (e < 0 || e >= E) { raise_status(status, MOE_DEVERR_EXPERT_ID); continue; }
    atomicAdd(&s_hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// One block of 256 threads (E <= 256).
__global__ void __launch_bounds__(256)
meta_scan_kernel(int32_t* __restrict__ chunk_counts, int n_chunks, int E, int capacity,
                 int32_t* __restrict__ bins, int32_t* __restrict__ padded_bins,
                 int32_t* __restrict__ sorted_start, int32_t* __restrict__ padded_start,
                 int32_t* __restrict__ routed_bins) {
  __shared__ int s_a[256], s_b[256], s_r[256];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int c = 0; c < n_chunks; ++c) {
      const int v = chunk_counts[(size_t)c * E + e];
      chunk_counts[(size_t)c * E + e] = total;   // exclusive offset of chunk c
      total += v;
    }
  }
  s_r[e] = (e < E) ? total : 0;   // routed, before any capacity drop
  // token-dropping variant: only the first `capacity` assignments are kept
  if (capacity > 0 && total > capacity) total = capacity;
  const int padded = (int)round_up(total, kTile);
  s_a[e] = (e < E) ? total : 0;
  s_b[e] = (e < E) ? padded : 0;
  __syncthreads();
  // inclusive Hillis-Steele scan over experts (integers: order is irrelevant)
  for (int off = 1; off < 256; off <<= 1) {
    const int a = (e >= off) ? s_a[e - off] : 0;
    const int b = (e >= off) ? s_b[e - off] : 0;
    const int r = (e >= off) ? s_r[e - off] : 0;
    __syncthreads();
    s_a[e] += a;
    s_b[e] += b;
    s_r[e] += r;
    __syncthreads();
  }
  if (e < E) {
    if (routed_bins) routed_bins[e] = s_r[e];
    if (bins) bins[e] = s_a[e];
    padded_bins[e] = s_b[e];
    sorted_start[e] = s_a[e] - total;
    padded_start[e] = s_b[e] - padded;
  }
}

__global__ void __launch_bounds__(kMetaPlaceThreads)
meta_place_kernel(const int32_t* __restrict__ top, int64_t NK, int E, int capacity,
                  const int32_t* __restrict__ chunk_offsets, const int32_t* __restrict__ sorted_start,
                  const int32_t* __restrict__ padded_start, int32_t* __restrict__ indices,
                  int32_t* __restrict__ bin_ids, int32_t* __restrict__ pos) {
  extern __shared__ int s_mem[];
  constexpr int W = kMetaPlaceThreads / 32;
  int* s_warp = s_mem;              // [W][E] per-warp counts, then exclusive offsets
  int* s_base = s_mem + W * E;      // [E] rank base of this round inside the expert
  int* s_tot = s_base + E;          // [E] this round's count per expert
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    s_base[e] = chunk_offsets[(size_t)blockIdx.x * E + e];
  const int64_t base = (int64_t)blockIdx.x * kMetaChunk;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < kMetaChunk / kMetaPlaceThreads; ++r) {
    for (int q = threadIdx.x; q < W * E; q += blockDim.x) s_warp[q] = 0;
    __syncthreads();
    const int64_t i = base + (int64_t)r * kMetaPlaceThreads + threadIdx.x;
    int e = (i < NK) ? top[i] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & lt_mask);     // earlier lanes with the same expert
    if (e >= 0 && rank_w == 0) s_warp[warp * E + e] = __popc(peers);
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += blockDim.x) {
      int run = 0;
      for (int w = 0; w < W; ++w) {                 // exclusive scan over warps
        const int v = s_warp[w * E + ee];
        s_warp[w * E + ee] = run;
        run += v;
      }
      s_tot[ee] = run;
    }
    __syncthreads();
    if (i < NK) {
      if (e >= 0) {
        // rank among all of expert e's assignments, in flat-id order
        const int rank = s_base[e] + s_warp[warp * E + e] + rank_w;
        if (capacity > 0 && rank >= capacity) {
          pos[i] = -1;                      // dropped: beyond the expert's capacity
        } else {
          if (indices) indices[sorted_start[e] + rank] = (int32_t)i;
          if (bin_ids) bin_ids[sorted_start[e] + rank] = e;
          pos[i] = padded_start[e] + rank;
        }
      } else {
        pos[i] = -1;
      }
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += blockDim.x) s_base[ee] += s_tot[ee];
    __syncthreads();
  }
}

size_t meta_workspace_bytes(int64_t NK, int E) {
  const int64_t chunks = cdiv(NK > 0 ? NK : 1, kMetaChunk);
  return (size_t)(chunks * E + 2 * E) * sizeof(int32_t);
}

moe_status dispatch_meta(const int32_t* top, int64_t NK, int E, int32_t* indices, int32_t* bin_ids,
                         int32_t* bins, int32_t* padded_bins, int32_t* pos, void* scratch,
                         int* status, cudaStream_t s, int capacity, int32_t* routed_bins) {
  const int n_chunks = (int)cdiv(NK > 0 ? NK : 1, kMetaChunk);
  int32_t* chunk_counts = (int32_t*)scratch;
  int32_t* sorted_start = chunk_counts + (size_t)n_chunks * E;
  int32_t* padded_start = sorted_start + E;
  MOE_TRACED("meta_count", s, (meta_count_kernel<<<n_chunks, 256, E * sizeof(int), s>>>(top, NK, E, chunk_counts, status)));
  MOE_LAUNCH_CHECK();
  MOE_TRACED("meta_scan", s, (meta_scan_kernel<<<1, 256, 0, s>>>(chunk_counts, n_chunks, E, capacity, bins, padded_bins, sorted_start,
                                     padded_start, routed_bins)));
  MOE_LAUNCH_CHECK();
  if (NK > 0) {
    // (32 + 2) * E counters: at most 34 KB for E <= 256, within the default
    // 48 KB of dynamic shared memory, so no attribute call is needed
    const size_t smem = (size_t)(kMetaPlaceThreads / 32 + 2) * E * sizeof(int);
    MOE_TRACED("meta_place", s, (meta_place_kernel<<<n_chunks, kMetaPlaceThreads, smem, s>>>(top, NK, E, capacity, chunk_counts,
                                                                sorted_start, padded_start, indices,
                                                                bin_ids, pos)));
    MOE_LAUNCH_CHECK();
  }
  return MOE_OK;
}

}  // namespace moe

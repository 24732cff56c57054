// Dispatch metadata: stable counting sort of the flat assignments by expert,
// histogram, inclusive cumsums, round-up of each group to 128 rows
// ("MegaBlocks - architecture", sec. 2.1/2.3 and sec. 4: the sort key is the
// expert id only, a few bits).
//
// A counting sort is the whole sort when keys are at most 8 bits wide.  The
// assignments are cut into chunks of T tokens (T*K flat ids; T = 128, or the
// router's chunk when it supplies the counts):
//   count  - per chunk, a shared-memory histogram of its expert ids (integer
//            atomics: a count does not depend on their order).  The bf16
//            layer skips this launch: its router epilogue writes the same
//            per-chunk counts.
//   place  - per chunk, one block: (a) every block sums the chunk counts of
//            all chunks and of the chunks before its own (integer sums, in
//            any order), so it knows each expert's total, its start in the
//            sorted order and in the padded rows, and the rank of its own
//            chunk's first assignment of each expert; block 0 writes bins,
//            padded_bins and the routed counts.  (b) The chunk's assignments
//            are visited in increasing flat id, in rounds of 1024; within a
//            warp the rank among equal experts comes from __match_any_sync,
//            across warps from a scan of the per-warp counts.  Rank order =
//            flat-id order: the sort is stable.
// Step (a) reads n_chunks^2 * E counts over the grid; past about 16 MB of
// such reads (more than 32768 tokens at E = 64) a separate one-block scan
// turns the counts into per-chunk offsets first and the place blocks read
// their own row of offsets only.
// Everything is integer work, so the outputs are exact and run-to-run equal.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kMetaThreads = 1024;       // place / scan blocks
constexpr int64_t kInlineScanReads = int64_t(1) << 22;   // counts read over the grid by step (a)

__host__ __device__ inline int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

int64_t meta_chunks(int64_t N, int T) { return cdiv(N > 0 ? N : 1, T); }

__global__ void __launch_bounds__(256)
meta_count_kernel(const int32_t* __restrict__ top, int64_t NK, int K, int E, int T,
                  int32_t* __restrict__ chunk_counts, int* status) {
  extern __shared__ int s_hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int64_t per = (int64_t)T * K;
  const int64_t base = (int64_t)blockIdx.x * per;
  const int64_t end = base + per < NK ? base + per : NK;
  for (int64_t i0 = base + threadIdx.x; i0 < end; i0 += 4 * (int64_t)blockDim.x) {
    int ev[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {   // loads first, then the histogram updates
      const int64_t i = i0 + (int64_t)u * blockDim.x;
      ev[u] = i < end ? top[i] : -2;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (ev[u] == -2) continue;
      if (ev[u] < 0 || ev[u] >= E) { raise_status(status, MOE_DEVERR_EXPERT_ID); continue; }
      atomicAdd(&s_hist[ev[u]], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// Per-expert starts from the per-expert totals (threads 0..255 of the block,
// E <= 256): routed = all assignments, kept = the first `capacity` of them in
// the token-dropping variant, padded = kept rounded up to 128.  Writes the
// layer-facing cumsums when `write` is set.
__device__ __forceinline__ void expert_starts(int total, int E, int capacity, int* s_a, int* s_b, int* s_r,
                                              int* s_sorted, int* s_padded, bool write, int32_t* bins,
                                              int32_t* padded_bins, int32_t* routed_bins) {
  const int e = threadIdx.x;
  int kept = total;
  if (capacity > 0 && kept > capacity) kept = capacity;   // token dropping
  const int padded = (int)round_up(kept, kTile);
  if (e < 256) {
    s_a[e] = e < E ? kept : 0;
    s_b[e] = e < E ? padded : 0;
    s_r[e] = e < E ? total : 0;
  }
  __syncthreads();
  // inclusive Hillis-Steele scans over the experts (integers: order is irrelevant)
  for (int off = 1; off < 256; off <<= 1) {
    int a = 0, b = 0, r = 0;
    if (e < 256 && e >= off) { a = s_a[e - off]; b = s_b[e - off]; r = s_r[e - off]; }
    __syncthreads();
    if (e < 256) { s_a[e] += a; s_b[e] += b; s_r[e] += r; }
    __syncthreads();
  }
  if (e < E) {
    s_sorted[e] = s_a[e] - kept;
    s_padded[e] = s_b[e] - padded;
    if (write) {
      if (bins) bins[e] = s_a[e];
      padded_bins[e] = s_b[e];
      if (routed_bins) routed_bins[e] = s_r[e];
    }
  }
}

// One block of kMetaThreads for a grid with too many chunks for the inline
// scan: chunk_counts becomes per-chunk exclusive offsets in place, starts =
// sorted_start[E] | padded_start[E], and the cumsums are written.
__global__ void __launch_bounds__(kMetaThreads)
meta_scan_kernel(int32_t* __restrict__ chunk_counts, int n_chunks, int E, int capacity, int32_t* __restrict__ bins,
                 int32_t* __restrict__ padded_bins, int32_t* __restrict__ routed_bins, int32_t* __restrict__ starts) {
  __shared__ int s_grp[kMetaThreads];
  __shared__ int s_a[256], s_b[256], s_r[256], s_tot[256];
  const int Ep = pow2_at_least(E);
  const int G = kMetaThreads / Ep;
  const int g = threadIdx.x / Ep, e = threadIdx.x % Ep;
  const int L = (n_chunks + G - 1) / G;        // contiguous chunks per group
  const int c0 = g * L, c1 = c0 + L < n_chunks ? c0 + L : n_chunks;
  int sum = 0;
  if (e < E) {
#pragma unroll 4
    for (int c = c0; c < c1; ++c) sum += chunk_counts[(size_t)c * E + e];
  }
  s_grp[threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.x < Ep) {        // exclusive offsets of the groups, in group order
    int run = 0;
    for (int gg = 0; gg < G; ++gg) {
      const int v = s_grp[gg * Ep + threadIdx.x];
      s_grp[gg * Ep + threadIdx.x] = run;
      run += v;
    }
    if (threadIdx.x < 256) s_tot[threadIdx.x] = run;
  }
  __syncthreads();
  if (e < E) {
    int run = s_grp[threadIdx.x];
    for (int c = c0; c < c1; ++c) {
      const int v = chunk_counts[(size_t)c * E + e];
      chunk_counts[(size_t)c * E + e] = run;
      run += v;
    }
  }
  const int total = threadIdx.x < 256 && threadIdx.x < E ? s_tot[threadIdx.x] : 0;
  expert_starts(total, E, capacity, s_a, s_b, s_r, starts, starts + E, true, bins, padded_bins, routed_bins);
}

// One block per chunk.  INLINE: chunk_counts holds counts and the block finds
// its offsets and the expert starts itself; otherwise chunk_counts holds the
// exclusive offsets and starts the expert starts (meta_scan_kernel).
template <bool INLINE>
__global__ void __launch_bounds__(kMetaThreads)
meta_place_kernel(const int32_t* __restrict__ top, int64_t NK, int K, int E, int T, int n_chunks, int capacity,
                  const int32_t* __restrict__ chunk_counts, const int32_t* __restrict__ starts,
                  int32_t* __restrict__ bins, int32_t* __restrict__ padded_bins, int32_t* __restrict__ routed_bins,
                  int32_t* __restrict__ indices, int32_t* __restrict__ bin_ids, int32_t* __restrict__ pos) {
  constexpr int W = kMetaThreads / 32;
  __shared__ int s_warp[W * 256];      // [W][E] per-warp counts, then exclusive offsets
  __shared__ int s_base[256];          // rank base of this round inside the expert
  __shared__ int s_tot[256];           // this round's count per expert
  __shared__ int s_sorted[256], s_padded[256];
  const int c = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if constexpr (INLINE) {
    // (a) totals and this chunk's offsets from every chunk's counts
    int* s_lt = s_warp;                      // [G][Ep] partial sums, reused below
    __shared__ int s_all[kMetaThreads];
    const int Ep = pow2_at_least(E);
    const int G = kMetaThreads / Ep;
    const int g = threadIdx.x / Ep, e = threadIdx.x % Ep;
    int lt = 0, all = 0;
    if (e < E) {
#pragma unroll 4
      for (int c2 = g; c2 < n_chunks; c2 += G) {
        const int v = chunk_counts[(size_t)c2 * E + e];
        all += v;
        lt += c2 < c ? v : 0;
      }
    }
    s_lt[threadIdx.x] = lt;
    s_all[threadIdx.x] = all;
    __syncthreads();
    int total = 0;
    if (threadIdx.x < E) {
      int a = 0, b = 0;
      for (int gg = 0; gg < G; ++gg) { a += s_lt[gg * Ep + threadIdx.x]; b += s_all[gg * Ep + threadIdx.x]; }
      s_base[threadIdx.x] = a;
      total = b;
    }
    __syncthreads();
    int* s_a = s_warp;            // scan scratch (s_lt is consumed)
    expert_starts(total, E, capacity, s_a, s_a + 256, s_a + 512, s_sorted, s_padded, c == 0, bins, padded_bins,
                  routed_bins);
  } else {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      s_base[e] = chunk_counts[(size_t)c * E + e];
      s_sorted[e] = starts[e];
      s_padded[e] = starts[E + e];
    }
  }
  __syncthreads();
  // (b) placement, in increasing flat id
  const int64_t base = (int64_t)c * T * K;
  int64_t end = base + (int64_t)T * K;
  if (end > NK) end = NK;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int64_t r0 = base; r0 < end; r0 += kMetaThreads) {
    for (int q = threadIdx.x; q < W * E; q += blockDim.x) s_warp[q] = 0;
    __syncthreads();
    const int64_t i = r0 + threadIdx.x;
    int e = (i < end) ? top[i] : -1;
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
    if (i < end) {
      if (e >= 0) {
        // rank among all of expert e's assignments, in flat-id order
        const int rank = s_base[e] + s_warp[warp * E + e] + rank_w;
        if (capacity > 0 && rank >= capacity) {
          pos[i] = -1;                      // dropped: beyond the expert's capacity
        } else {
          if (indices) indices[s_sorted[e] + rank] = (int32_t)i;
          if (bin_ids) bin_ids[s_sorted[e] + rank] = e;
          pos[i] = s_padded[e] + rank;
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

size_t meta_workspace_bytes(int64_t N, int E, int T) {
  return (size_t)(meta_chunks(N, T) * E + 2 * E) * sizeof(int32_t);
}

moe_status dispatch_meta(const int32_t* top, int64_t N, int K, int E, int32_t* indices, int32_t* bin_ids,
                         int32_t* bins, int32_t* padded_bins, int32_t* pos, void* scratch, int* status,
                         cudaStream_t s, int capacity, int32_t* routed_bins, bool counts_ready, int T) {
  const int64_t NK = N * K;
  const int n_chunks = (int)meta_chunks(N, T);
  int32_t* chunk_counts = (int32_t*)scratch;
  int32_t* starts = chunk_counts + (size_t)n_chunks * E;
  if (N == 0) {
    // no assignments: every count is zero (the place kernel would see no chunk)
    MOE_TRACED("meta_scan", s, (meta_scan_kernel<<<1, kMetaThreads, 0, s>>>(nullptr, 0, E, capacity, bins,
                                                                           padded_bins, routed_bins, starts)));
    MOE_LAUNCH_CHECK();
    return MOE_OK;
  }
  if (!counts_ready) {
    MOE_TRACED("meta_count", s, (meta_count_kernel<<<n_chunks, 256, E * sizeof(int), s>>>(top, NK, K, E, T,
                                                                                           chunk_counts, status)));
    MOE_LAUNCH_CHECK();
  }
  if ((int64_t)n_chunks * n_chunks * E <= kInlineScanReads) {
    MOE_TRACED("meta_place", s, (meta_place_kernel<true><<<n_chunks, kMetaThreads, 0, s>>>(
                                    top, NK, K, E, T, n_chunks, capacity, chunk_counts, nullptr, bins, padded_bins,
                                    routed_bins, indices, bin_ids, pos)));
  } else {
    MOE_TRACED("meta_scan", s, (meta_scan_kernel<<<1, kMetaThreads, 0, s>>>(chunk_counts, n_chunks, E, capacity,
                                                                           bins, padded_bins, routed_bins, starts)));
    MOE_LAUNCH_CHECK();
    MOE_TRACED("meta_place", s, (meta_place_kernel<false><<<n_chunks, kMetaThreads, 0, s>>>(
                                    top, NK, K, E, T, n_chunks, capacity, chunk_counts, starts, nullptr, nullptr,
                                    nullptr, indices, bin_ids, pos)));
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe

// Tensor-core router for bf16 layers: logits = x W_r, softmax, top-K (equal
// values to the lower expert id), renormalised weights ("MoE computation
// principle and execution", sec. 2.1-2.2), plus the per-chunk expert
// histogram the dispatch metadata starts from ("MegaBlocks - architecture",
// sec. 2.3: histogram of the sorted expert ids).
//
// The router reads x once and does little arithmetic per byte (E FLOP per
// byte of x), so it is bound by HBM as long as enough CTAs stream x.  A CTA
// multiplies one 128-token row tile (TMA -> shared memory -> tcgen05.mma,
// fp32 accumulators in TMEM), one CTA per SM.  When the row tiles are too
// few to fill the GPU (small N), a tile's H is split over a cluster of S CTAs
// (S = 2..8):
// each writes its 128 x E partial logits to a global scratch (it stays in
// L2), a cluster barrier publishes them, and CTA r then finishes rows
// [r*128/S, (r+1)*128/S) of the tile, summing the S partials in the fixed
// order s = 0..S-1.  S depends only on N, H, E and K, never on the device, so
// the logits are the same bits on every run.
//
// Warps: 0 TMA producer, 1 TMEM owner and MMA issuer, 2-5 TMEM -> shared
// memory (S = 1) or global scratch; then one thread per row finishes a row:
// the sum of the partials, the max, a sorted top-K list (ties to the lower
// id), the softmax when asked, the renormalisation, and its experts into this
// CTA's histogram (integer shared-memory atomics), which is written as the
// count row of the CTA's 128/S-token chunk.  Every mbarrier wait is bounded
// (MOE_DEVERR_TIMEOUT); no TMA load uses multicast.
//
// B operand: W_r [H, E] is read MN-major straight from the caller's matrix
// when E is a multiple of 8 (64-expert boxes, experts past E read as zeros);
// otherwise a K-major copy W_r^T [E rounded up to 16, H] is made first.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace moe {
namespace {

using namespace umma;

constexpr int kRows = 128;                 // tokens per row tile
constexpr int kRBK = 64;                   // k block (one 128-byte swizzle row of bf16)
constexpr int kRouteThreads = 192;       // router weight gradient
constexpr int kRouteRowThreads = 256;    // router: 2 (S = 1) to 16 (S = 8) threads per routed row
constexpr int kA = kRows * kRBK * 2;       // A bytes per stage
constexpr uint64_t kRouteTimeoutNs = 2000000000ull;
constexpr int kRouteSlots = 148;           // SMs the split aims to fill (fixed: results must not depend on the GPU)

struct RouteParams {
  CUtensorMap tx;          // x [N, H]: 64 x 128 boxes
  CUtensorMap tw;          // W_r [H, E] (64 x 64 boxes, MN-major) or W_r^T [n_mma, H] (64 x n_mma, K-major)
  int N, H, E, K;
  int n_mma;               // MMA N: E rounded up to 16
  int nkb;                 // k blocks over H
  float* part;             // S > 1: partial logits [S][N][n_mma]
  float* logits;
  float* probs;
  int32_t* top;
  float* weights;
  int32_t* chunk_counts;   // [tiles * S][E] or NULL
  int* status;
};

template <int EPT>
struct RouteShape {
  static constexpr int NB = EPT == 8 ? 4 : (EPT == 4 ? 2 : 1);    // 64-column B boxes per k block
  static constexpr int KB = 1;                                     // k blocks per stage
  static constexpr int B_BYTES = NB * 8192;                        // per k block
  static constexpr int STAGE = KB * (kA + B_BYTES);
  static constexpr int STAGES = (192 * 1024) / STAGE;              // one CTA per SM
  static constexpr int STRIDE = EPT * 32 + 1;   // partial-logit row stride (floats), odd: no bank conflicts
  static constexpr int PART_BYTES = kRows * STRIDE * 4;
  static_assert(PART_BYTES <= STAGES * STAGE, "partial logits reuse the pipeline buffers");
  static constexpr uint32_t TMEM_COLS = EPT * 32 < 32 ? 32 : EPT * 32;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + 1024 + 8 * (2 * STAGES + 1) + 16 + 256 * 4;
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Insert (v, id) into a descending list of the K largest; a strict '>' keeps
// an earlier, lower id above an equal value, so ties go to the lower id when
// ids arrive in increasing order.
template <int KMAX, bool EXACT = false>
__device__ __forceinline__ void topk_insert(float v, int id, int K, float (&vals)[KMAX], int (&ids)[KMAX]) {
#pragma unroll
  for (int j = KMAX - 1; j >= 0; --j) {
    if ((EXACT || j < K) && v > vals[j]) {
      if (j > 0 && v > vals[j - 1]) {
        vals[j] = vals[j - 1];
        ids[j] = ids[j - 1];
      } else {
        vals[j] = v;
        ids[j] = id;
      }
    }
  }
}

// Top-K of one routed row over experts [e0, e1) of its logits in shared
// memory (`mine`), merged across the TPR threads of the row (consecutive
// lanes): each thread keeps the sorted list of its own expert range, then
// the lists fold pairwise towards the row's first thread, the higher-id
// partner's list inserted into the lower one's in its sorted order.  With
// strict '>' insertion an equal value stays behind every element already in
// the list, and the lower thread holds the lower ids, so the result equals
// one pass over all experts in increasing id order (ties to the lower id).
template <int KMAX, bool EXACT>
__device__ __forceinline__ void row_topk(const float* mine, int e0, int e1, int K, int TPR, int lane,
                                         float (&vals)[KMAX], int (&ids)[KMAX]) {
#pragma unroll
  for (int j = 0; j < KMAX; ++j) { vals[j] = -INFINITY; ids[j] = 0; }
#pragma unroll 4
  for (int e = e0; e < e1; ++e) topk_insert<KMAX, EXACT>(mine[e], e, K, vals, ids);
  const int sub = lane % TPR;
  for (int d = 1; d < TPR; d <<= 1) {
    float ov[KMAX];
    int oi[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ov[j] = __shfl_down_sync(0xffffffffu, vals[j], d);
      oi[j] = __shfl_down_sync(0xffffffffu, ids[j], d);
    }
    if (sub % (2 * d) == 0) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (EXACT || j < K) topk_insert<KMAX, EXACT>(ov[j], oi[j], K, vals, ids);
    }
  }
}

template <int EPT, bool B_MN, int KMAX>
__global__ void __launch_bounds__(kRouteRowThreads, 1) route_kernel(const __grid_constant__ RouteParams p) {
  using S_ = RouteShape<EPT>;
  constexpr int STAGES = S_::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t bar_base = base + STAGES * S_::STAGE;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t tfull = bar_base + 8u * (2 * STAGES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + STAGES * S_::STAGE + 8 * (2 * STAGES + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* s_hist = reinterpret_cast<int*>(tmem_holder + 4);    // [256] expert counts of this CTA's rows
  const uint32_t part = base;                                 // the (partial) logits, after the main loop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t S = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int tile = (int)cluster_id_x();
  const int row0 = tile * kRows;
  // this CTA's contiguous share of the stages of KB k blocks
  const int q = (p.nkb / S_::KB) / (int)S, rem = (p.nkb / S_::KB) % (int)S;
  const int kb0 = (int)rank * q + ((int)rank < rem ? (int)rank : rem);
  const int nk = q + ((int)rank < rem ? 1 : 0);

  for (int e = threadIdx.x; e < 256; e += blockDim.x) s_hist[e] = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tx);
    tma_prefetch_desc(&p.tw);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), S_::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint32_t tx_bytes = S_::KB * (kA + (B_MN ? S_::B_BYTES : (uint32_t)p.n_mma * kRBK * 2));
      int stage = 0;
      uint32_t phase = 0;
      for (int i = 0; i < nk; ++i) {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status, kRouteTimeoutNs)) break;
        const uint32_t sa0 = base + stage * S_::STAGE;
        mbar_expect_tx(full_bar(stage), tx_bytes);
#pragma unroll
        for (int b = 0; b < S_::KB; ++b)     // x first: the row pieces of one stage back to back
          tma_load_2d(sa0 + b * kA, &p.tx, full_bar(stage), ((kb0 + i) * S_::KB + b) * kRBK, row0);
#pragma unroll
        for (int b = 0; b < S_::KB; ++b) {
          const uint32_t sb = sa0 + S_::KB * kA + b * S_::B_BYTES;
          const int k = ((kb0 + i) * S_::KB + b) * kRBK;
          if constexpr (B_MN) {
#pragma unroll
            for (int j = 0; j < S_::NB; ++j) tma_load_2d(sb + j * 8192, &p.tw, full_bar(stage), 64 * j, k);
          } else {
            tma_load_2d(sb, &p.tw, full_bar(stage), k, 0);
          }
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA
      const uint32_t idesc = idesc_bf16(kRows, p.n_mma, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status, kRouteTimeoutNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa0 = base + stage * S_::STAGE;
#pragma unroll
        for (int b = 0; b < S_::KB; ++b) {
          const uint32_t sa = sa0 + b * kA, sb = sa0 + S_::KB * kA + b * S_::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < kRBK / 16; ++kk) {
            const uint64_t ad = desc_k_sw128(sa + kk * 32);
            const uint64_t bd = B_MN ? desc_mn_sw128(sb + kk * 2048, 8192) : desc_k_sw128(sb + kk * 32);
            mma_bf16(tmem_base, ad, bd, idesc, (i | b | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) mma_commit(tfull);
      else *abort_flag = 1;
    }
  } else if (warp < 6) {
    // --------------------------------- TMEM -> (partial) logits in shared memory
    int ok = 0;
    if (lane == 0) ok = mbar_wait_bounded(tfull, 0, abort_flag, p.status, kRouteTimeoutNs) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    tc_fence_after();
    const int qd = warp & 3;                       // TMEM lane quarter of this warp
    const int row = qd * 32 + lane;
    const uint32_t dst = part + (uint32_t)(row * S_::STRIDE) * 4u;
#pragma unroll
    for (int c = 0; c < EPT; ++c) {
      if (c * 32 >= p.n_mma) break;
      uint32_t r[32];
      if (ok) {
        tmem_ld_32(tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(c * 32), r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) st_shared_f32(dst + (uint32_t)(c * 32 + j) * 4u, __uint_as_float(r[j]));
    }
  }
  tc_fence_before();
  __syncthreads();               // this CTA's (partial) logits of its 128 rows are in shared memory
  if (S > 1) {
    // publish the rows other CTAs of the cluster finish: this CTA's partial
    // [rank][N][n_mma] block, coalesced 16-byte stores; its own rows stay here
    const int vpr = p.n_mma / 4;
    const float* rb = reinterpret_cast<const float*>(gbase);
    for (int v = (int)threadIdx.x; v < kRows * vpr; v += (int)blockDim.x) {
      const int row = v / vpr, c = (v % vpr) * 4;
      const int64_t t = (int64_t)row0 + row;
      if (row / (kRows / (int)S) != (int)rank && t < p.N) {
        const float* src = rb + row * S_::STRIDE + c;
        *reinterpret_cast<float4*>(p.part + ((size_t)rank * p.N + t) * p.n_mma + c) =
            make_float4(src[0], src[1], src[2], src[3]);
      }
    }
    cluster_sync();              // every CTA's partials published (release / acquire, cluster scope)
  }
  tc_fence_after();

  // ------------------------------------------------ rows: partials -> routing
  // CTA r finishes rows [r*R, (r+1)*R), R = 128 / S.  With S > 1 all threads
  // first sum the rows' partial logits (over s = 0..S-1 in order, coalesced)
  // into this CTA's shared-memory rows (the pipeline buffers are free); with
  // S = 1 the logits are there already.  Then TPR = blockDim / R threads per
  // row select its top K (row_topk) and the row's first thread finishes it.
  const int rows_per = kRows / (int)S;
  float* const rowbuf = reinterpret_cast<float*>(gbase);
  if (S > 1) {
    // this CTA's rows of partial s are one contiguous [rows][n_mma] block;
    // 16-byte loads, four per thread in flight per partial; its own partial
    // (s = rank) is read from shared memory, the sum kept in the order s = 0..S-1
    const int cols = p.n_mma;                              // a multiple of 16
    const int64_t first = (int64_t)row0 + (int64_t)rank * rows_per;
    const int64_t left = p.N - first;
    const int nrows = left < rows_per ? (left > 0 ? (int)left : 0) : rows_per;
    const int vpr = cols / 4, nvec = nrows * vpr;
    for (int v0 = (int)threadIdx.x; v0 < nvec; v0 += 4 * (int)blockDim.x) {
      float4 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (uint32_t s = 0; s < S; ++s) {
        const float4* src = reinterpret_cast<const float4*>(p.part + ((size_t)s * p.N + first) * cols);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * (int)blockDim.x;
          if (v < nvec) {
            float4 x;
            if (s == rank) {
              const float* o = rowbuf + ((int)rank * rows_per + v / vpr) * S_::STRIDE + (v % vpr) * 4;
              x = make_float4(o[0], o[1], o[2], o[3]);
            } else {
              x = src[v];
            }
            acc[u].x += x.x; acc[u].y += x.y; acc[u].z += x.z; acc[u].w += x.w;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * (int)blockDim.x;
        if (v < nvec) {
          float* dst = rowbuf + ((int)rank * rows_per + v / vpr) * S_::STRIDE + (v % vpr) * 4;
          dst[0] = acc[u].x; dst[1] = acc[u].y; dst[2] = acc[u].z; dst[3] = acc[u].w;
        }
      }
    }
    __syncthreads();
  }
  {
    const int TPR = (int)blockDim.x / rows_per;            // 2, 4, 8 or 16: divides 32
    const int row = (int)rank * rows_per + (int)threadIdx.x / TPR;
    const int sub = (int)threadIdx.x % TPR;
    const int64_t t = (int64_t)row0 + row;
    const float* mine = rowbuf + row * S_::STRIDE;
    const int span = (p.E + TPR - 1) / TPR;
    const int e0 = t < p.N ? (sub * span < p.E ? sub * span : p.E) : 0;
    const int e1 = t < p.N ? ((sub + 1) * span < p.E ? (sub + 1) * span : p.E) : 0;
    float vals[KMAX];
    int ids[KMAX];
    if (p.K == KMAX) row_topk<KMAX, true>(mine, e0, e1, p.K, TPR, lane, vals, ids);
    else row_topk<KMAX, false>(mine, e0, e1, p.K, TPR, lane, vals, ids);
    if (p.logits)
      for (int e = e0; e < e1; ++e) p.logits[t * p.E + e] = mine[e];
    if (t < p.N && sub == 0) {
      const float m = vals[0];   // the row's largest logit
      if (p.probs) {
        float Z = 0.f;
        for (int e = 0; e < p.E; ++e) Z += expf(mine[e] - m);
        for (int e = 0; e < p.E; ++e) p.probs[t * p.E + e] = expf(mine[e] - m) / Z;
      }
      // kept probabilities renormalised: exp(l_k - l_max) / sum_j exp(l_j - l_max)
      float ev[KMAX], Ssum = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        ev[j] = j < p.K ? expf(vals[j] - vals[0]) : 0.f;
        Ssum += ev[j];
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < p.K) {
          p.top[t * p.K + j] = ids[j];
          p.weights[t * p.K + j] = ev[j] / Ssum;
          if (p.chunk_counts) atomicAdd(&s_hist[ids[j]], 1);
        }
      }
    }
  }
  __syncthreads();
  if (p.chunk_counts) {
    // this CTA's rows are chunk tile * S + rank of 128 / S tokens; a chunk
    // that starts at or past N does not exist (the last tile's trailing CTAs)
    const int64_t chunk = (int64_t)tile * S + rank;
    if (chunk * rows_per < p.N)
      for (int e = threadIdx.x; e < p.E; e += blockDim.x) p.chunk_counts[chunk * p.E + e] = s_hist[e];
  }
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, S_::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// 2-D bf16 map over a row-major [outer, inner] matrix, 128-byte swizzle;
// elements outside the matrix read as zero.
bool map2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
           uint32_t box_outer) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int route_ept(int E) {
  const int n_mma = (int)round_up(E, 16);
  return n_mma <= 32 ? 1 : n_mma <= 64 ? 2 : n_mma <= 128 ? 4 : 8;
}

template <int EPT, bool B_MN, int KMAX>
moe_status launch_route(const RouteParams& p, int S, int tiles, cudaStream_t s) {
  using S_ = RouteShape<EPT>;
  auto kern = route_kernel<EPT, B_MN, KMAX>;
  static bool smem_set[64] = {false};        // once per device: later calls (a graph capture among them) only launch
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!smem_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_::SMEM) != cudaSuccess) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    smem_set[dev] = true;
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(tiles * S), 1, 1);
  cfg.blockDim = dim3(kRouteRowThreads, 1, 1);
  cfg.dynamicSmemBytes = S_::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaSuccess;
  MOE_TRACED("route_umma", s, (err = cudaLaunchKernelEx(&cfg, kern, p)));
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace

bool route_umma_supported(int N, int H, int E, int K) {
  (void)N;
  return E >= 1 && E <= 256 && K >= 1 && K <= 32 && K <= E && H % kRBK == 0;
}

// H slices per row tile: the largest power of two (up to 8) that keeps
// tiles * S CTAs within one per SM, with at least four k blocks per slice.
// (More CTAs than SMs would not shorten the busiest SM's share of x.)
int route_split(int N, int H, int E, int K) {
  (void)E;
  (void)K;
  const int tiles = (int)cdiv(N > 0 ? N : 1, kRows);
  const int stages = H / kRBK;
  int S = 1;
  while (S < 8 && tiles * S * 2 <= kRouteSlots && stages / (S * 2) >= 4) S *= 2;
  return S;
}

int route_chunk_tokens(int N, int H, int E, int K) { return kRows / route_split(N, H, E, K); }

size_t route_umma_scratch(int N, int H, int E, int K) {
  const size_t n_mma = (size_t)round_up(E, 16);
  const size_t wt = E % 8 == 0 ? 0 : (size_t)round_up(n_mma * H * 2, 256);
  const int S = route_split(N, H, E, K);
  return wt + (S > 1 ? (size_t)S * N * n_mma * sizeof(float) : 0);
}

moe_status route_umma(const void* x, const void* W_r, int N, int H, int E, int K, float* logits, float* probs,
                      int32_t* top, float* w, void* scratch, int* status, cudaStream_t s, int32_t* chunk_counts) {
  if (N == 0) return MOE_OK;
  RouteParams p;
  memset(&p, 0, sizeof(p));
  const int n_mma = (int)round_up(E, 16);
  const int ept = route_ept(E);
  const bool mn = E % 8 == 0;
  const size_t wt_bytes = mn ? 0 : (size_t)round_up((int64_t)n_mma * H * 2, 256);
  if (!map2d(&p.tx, x, H, N, 64, kRows)) return MOE_ERR_CUDA;
  if (mn) {
    // MN-major B straight from W_r [H, E]: 64-expert boxes, experts past E read as zeros
    if (!map2d(&p.tw, W_r, E, H, 64, 64)) return MOE_ERR_CUDA;
  } else {
    // K-major B: W_r^T [n_mma, H] in the workspace, rows E.. zero
    moe_status st = transpose_matrix(W_r, H, E, MOE_BF16, scratch, s, n_mma);
    if (st != MOE_OK) return st;
    if (!map2d(&p.tw, scratch, H, n_mma, 64, (uint32_t)n_mma)) return MOE_ERR_CUDA;
  }
  p.N = N;
  p.H = H;
  p.E = E;
  p.K = K;
  p.n_mma = n_mma;
  p.nkb = H / kRBK;
  p.part = (float*)((char*)scratch + wt_bytes);
  p.logits = logits;
  p.probs = probs;
  p.top = top;
  p.weights = w;
  p.chunk_counts = chunk_counts;
  p.status = status;
  const int tiles = (int)cdiv(N, kRows);
  const int S = route_split(N, H, E, K);
#define MOE_ROUTE_K(EPT_, MN_)                                                               \
  return K <= 2 ? launch_route<EPT_, MN_, 2>(p, S, tiles, s)                                 \
                : K <= 4 ? launch_route<EPT_, MN_, 4>(p, S, tiles, s)                        \
                         : K <= 8 ? launch_route<EPT_, MN_, 8>(p, S, tiles, s)               \
                                  : (K <= 16 ? launch_route<EPT_, MN_, 16>(p, S, tiles, s)   \
                                             : launch_route<EPT_, MN_, 32>(p, S, tiles, s))
  switch (ept * 2 + (mn ? 1 : 0)) {
    case 3: MOE_ROUTE_K(1, true);
    case 2: MOE_ROUTE_K(1, false);
    case 5: MOE_ROUTE_K(2, true);
    case 4: MOE_ROUTE_K(2, false);
    case 9: MOE_ROUTE_K(4, true);
    case 8: MOE_ROUTE_K(4, false);
    case 17: MOE_ROUTE_K(8, true);
    default: MOE_ROUTE_K(8, false);
  }
#undef MOE_ROUTE_K
}

// ---------------------------------------------------------------------------
// Router weight gradient on tensor cores: dW_r = x^T D, D [N, E] bf16 holding
// each token's logit gradients (zero outside the experts that receive one).
// x is read once: the tokens are cut into chunks of whole 64-token k blocks,
// and CTA (chunk c, expert tile, 256-column slice of H) computes the fp32
// partial D[c]^T x[c] (M = experts, N = H columns, K = the chunk's tokens;
// both operands MN-major straight from the row-major D and x), stored as
// part[c][e][h].  A second kernel sums the chunks in increasing c and writes
// dW_r [H, E] transposed through shared memory.  The chunking depends only on
// N, H and E, so the result is the same bits on every run and every GPU.
namespace {

constexpr int kWgSlots = 148;   // CTAs the chunking aims at (one per SM)

struct RwParams {
  CUtensorMap td;          // D [N, E]: 64 x 64 boxes
  CUtensorMap tx;          // x [N, H]: 64 x 64 boxes
  int N, H, E;
  int chunk;               // tokens per chunk, a multiple of 64
  int n_tiles;             // H / BN
  int m_tiles;             // ceil(E / 128)
  float* part;             // [n_chunks][E][H]
  int* status;
};

template <int BN>
struct RwShape {
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = BN * 64 * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (192 * 1024) / STAGE;
  static constexpr uint32_t TMEM_COLS = BN;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + 1024 + 8 * (2 * STAGES + 1) + 16;
};

template <int BN>
__global__ void __launch_bounds__(kRouteThreads, 1) router_wgrad_kernel(const __grid_constant__ RwParams p) {
  using S_ = RwShape<BN>;
  constexpr int STAGES = S_::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t bar_base = base + STAGES * S_::STAGE;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t tfull = bar_base + 8u * (2 * STAGES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + STAGES * S_::STAGE + 8 * (2 * STAGES + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x % p.n_tiles;
  const int rest = blockIdx.x / p.n_tiles;
  const int mt = rest % p.m_tiles, c = rest / p.m_tiles;
  const int t0 = c * p.chunk;
  const int t1 = t0 + p.chunk < p.N ? t0 + p.chunk : p.N;
  const int nkb = t1 > t0 ? (t1 - t0 + 63) / 64 : 0;
  const int e0 = mt * 128;
  // 64-expert boxes of A this tile needs; rows of the 128-row MMA past them
  // hold stale shared memory and only reach accumulator rows that are not stored
  const int a_boxes = (p.E - e0) > 64 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.td);
    tma_prefetch_desc(&p.tx);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), S_::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t tx_bytes = (uint32_t)(a_boxes * 8192 + S_::B_BYTES);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status, kRouteTimeoutNs)) break;
        const uint32_t sa = base + stage * S_::STAGE, sb = sa + S_::A_BYTES;
        const int t = t0 + kb * 64;
        mbar_expect_tx(full_bar(stage), tx_bytes);
        for (int j = 0; j < a_boxes; ++j) tma_load_2d(sa + j * 8192, &p.td, full_bar(stage), e0 + 64 * j, t);
#pragma unroll
        for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, &p.tx, full_bar(stage), nt * BN + 64 * j, t);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, BN, true, true);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status, kRouteTimeoutNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = base + stage * S_::STAGE, sb = sa + S_::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem_base, desc_mn_sw128(sa + kk * 2048, 8192), desc_mn_sw128(sb + kk * 2048, 8192), idesc,
                   (kb | kk) != 0 ? 1u : 0u);
        mma_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok && nkb > 0) mma_commit(tfull);
      else *abort_flag = 1;
    }
  } else {
    int ok = 0;
    if (lane == 0) ok = (nkb > 0 && mbar_wait_bounded(tfull, 0, abort_flag, p.status, kRouteTimeoutNs)) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    tc_fence_after();
    const int qd = warp & 3;
    const int e = e0 + qd * 32 + lane;
#pragma unroll 1
    for (int cc = 0; cc < BN / 32; ++cc) {
      uint32_t r[32];
      if (ok) {
        tmem_ld_32(tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(cc * 32), r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      }
      if (e < p.E) {
        float4* d = reinterpret_cast<float4*>(p.part + ((size_t)c * p.E + e) * p.H + nt * BN + cc * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                             __uint_as_float(r[4 * j + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, S_::TMEM_COLS);
  }
}

// dW_r[h][e] = sum over chunks c, in increasing c, of part[c][e][h]; a 32 x 32
// (e, h) tile per block, transposed through shared memory so that both the
// reads (along h) and the writes (along e) are coalesced.
__global__ void __launch_bounds__(256)
router_wgrad_reduce_tc_kernel(const float* __restrict__ part, int n_chunks, int H, int E, __nv_bfloat16* __restrict__ dWr) {
  __shared__ float tile[32][33];
  const int h0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int el = ty + 8 * i, e = e0 + el, h = h0 + tx;
    float acc = 0.f;
    if (e < E && h < H)
      for (int c = 0; c < n_chunks; ++c) acc += part[((size_t)c * E + e) * H + h];
    tile[el][tx] = acc;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int hl = ty + 8 * i, h = h0 + hl, e = e0 + tx;
    if (e < E && h < H) dWr[(size_t)h * E + e] = __float2bfloat16_rn(tile[tx][hl]);
  }
}

struct RwPlan {
  int bn, n_tiles, m_tiles, chunk, n_chunks;
};

RwPlan rw_plan(int N, int H, int E) {
  RwPlan pl;
  pl.bn = H % 256 == 0 ? 256 : 128;
  pl.n_tiles = H / pl.bn > 0 ? H / pl.bn : 1;   // callers check router_wgrad_tc_supported first
  pl.m_tiles = E > 0 ? (E + 127) / 128 : 1;
  const int per_chunk = pl.n_tiles * pl.m_tiles;
  int n = kWgSlots / per_chunk;
  const int max_chunks = (int)cdiv(N > 0 ? N : 1, 64);
  if (n < 1) n = 1;
  if (n > max_chunks) n = max_chunks;
  pl.chunk = (int)round_up(cdiv(N > 0 ? N : 1, n), 64);
  pl.n_chunks = (int)cdiv(N > 0 ? N : 1, pl.chunk);
  return pl;
}

template <int BN>
moe_status launch_router_wgrad(const RwParams& p, int blocks, cudaStream_t s) {
  using S_ = RwShape<BN>;
  auto kern = router_wgrad_kernel<BN>;
  static bool smem_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!smem_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_::SMEM) != cudaSuccess) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    smem_set[dev] = true;
  }
  MOE_TRACED("router_wgrad", s, (kern<<<blocks, kRouteThreads, S_::SMEM, s>>>(p)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace

bool router_wgrad_tc_supported(int H, int E) { return E % 8 == 0 && E <= 256 && H % 128 == 0; }

size_t router_wgrad_tc_scratch(int N, int H, int E) {
  if (!router_wgrad_tc_supported(H, E)) return 0;
  const RwPlan pl = rw_plan(N, H, E);
  return (size_t)pl.n_chunks * E * H * sizeof(float);
}

moe_status router_wgrad_tc(const void* x, const void* Dh, int N, int H, int E, void* dWr, void* scratch, int* status,
                           cudaStream_t s) {
  if (!router_wgrad_tc_supported(H, E)) return MOE_ERR_UNSUPPORTED;
  if (N == 0) return MOE_OK;
  const RwPlan pl = rw_plan(N, H, E);
  RwParams p;
  memset(&p, 0, sizeof(p));
  if (!map2d(&p.td, Dh, E, N, 64, 64) || !map2d(&p.tx, x, H, N, 64, 64)) return MOE_ERR_CUDA;
  p.N = N;
  p.H = H;
  p.E = E;
  p.chunk = pl.chunk;
  p.n_tiles = pl.n_tiles;
  p.m_tiles = pl.m_tiles;
  p.part = (float*)scratch;
  p.status = status;
  const int blocks = pl.n_chunks * pl.m_tiles * pl.n_tiles;
  moe_status st = pl.bn == 256 ? launch_router_wgrad<256>(p, blocks, s) : launch_router_wgrad<128>(p, blocks, s);
  if (st != MOE_OK) return st;
  dim3 g((unsigned)cdiv(H, 32), (unsigned)cdiv(E, 32));
  MOE_TRACED("router_wgrad_reduce", s, (router_wgrad_reduce_tc_kernel<<<g, 256, 0, s>>>(
                                          (const float*)scratch, pl.n_chunks, H, E, (__nv_bfloat16*)dWr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe

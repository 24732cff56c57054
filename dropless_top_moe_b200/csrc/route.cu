// Router for small expert counts: logits = x W_r, softmax, top-K, renormalise
// ("MoE computation principle and execution", sec. 2.1-2.2), one warp per token.
//
// Each lane accumulates partial dot products of its 16-byte slices of the
// token row against every expert column, then an xor-butterfly of warp
// shuffles completes all E logits on every lane.  W_r is staged transposed
// ([E][H]) in shared memory so that the lane-strided 16-byte reads are free of
// bank conflicts.  HBM traffic is one read of x plus the outputs; this is the
// bandwidth-bound regime (E small).  Large E goes through the tensor-core
// router in route_umma.cu.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

template <typename T, int EMAX>
__global__ void __launch_bounds__(256)
route_simt_kernel(const T* __restrict__ x, const T* __restrict__ W_r, int N, int H, int E, int K,
                  float* __restrict__ logits, float* __restrict__ probs,
                  int32_t* __restrict__ top_experts, float* __restrict__ weights) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* wrT = reinterpret_cast<T*>(smem_raw);          // [E][H]
  // transposed staging with h fastest across threads: conflict-free smem writes
  for (int idx = threadIdx.x; idx < H * E; idx += blockDim.x) {
    const int e = idx / H, h = idx - e * H;
    wrT[idx] = W_r[(size_t)h * E + e];
  }
  __syncthreads();

  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int nwarps = gridDim.x * warps_per_block;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < N; t += nwarps) {
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    const T* xr = x + (size_t)t * H;
    for (int h0 = lane * V; h0 < H; h0 += 32 * V) {
      float xf[V];
      Vec<T>::to_float(ld_nc_v4(xr + h0), xf);
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          float wf[V];
          Vec<T>::to_float(*reinterpret_cast<const uint4*>(wrT + (size_t)e * H + h0), wf);
#pragma unroll
          for (int j = 0; j < V; ++j) acc[e] = fmaf(xf[j], wf[j], acc[e]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) acc[e] = warp_sum(acc[e]);

    // every lane now holds the same E logits
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) m = fmaxf(m, acc[e]);
    if (logits || probs) {
      float Z = 0.f;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E) Z += expf(acc[e] - m);
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E && (e & 31) == lane) {
          if (logits) logits[(size_t)t * E + e] = acc[e];
          if (probs) probs[(size_t)t * E + e] = expf(acc[e] - m) / Z;
        }
      }
    }
    // top-K by repeated arg-max over the logits; strict '>' while scanning
    // upward keeps the lowest id among equal values.  Lane k keeps choice k.
    uint64_t taken = 0;
    int my_id = 0;
    float my_l = 0.f;
    for (int k = 0; k < K; ++k) {
      int best = -1;
      float bv = 0.f;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E && !((taken >> e) & 1ull) && (best < 0 || acc[e] > bv)) {
          best = e;
          bv = acc[e];
        }
      }
      taken |= 1ull << best;
      if (lane == k) { my_id = best; my_l = bv; }
    }
    // kept probabilities renormalised: exp(l_k - m) / sum_j exp(l_j - m)
    const float ek = (lane < K) ? expf(my_l - m) : 0.f;
    const float S = warp_sum(ek);
    if (lane < K) {
      top_experts[(size_t)t * K + lane] = my_id;
      weights[(size_t)t * K + lane] = ek / S;
    }
  }
}

template <typename T>
static moe_status launch_route_simt(const T* x, const T* W_r, int N, int H, int E, int K,
                                    float* logits, float* probs, int32_t* top, float* w,
                                    cudaStream_t s) {
  const size_t smem = (size_t)H * E * sizeof(T);
  const int threads = 256;
  int blocks = (int)cdiv(N, threads / 32);
  const int per_sm = smem > 0 ? (int)(200 * 1024 / smem) : 8;
  blocks = blocks < 148 * (per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm))
               ? blocks : 148 * (per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm));
  if (blocks < 1) blocks = 1;
#define MOE_ROUTE_CASE(EM)                                                                     \
  if (E <= EM) {                                                                               \
    static bool smem_set[64] = {false};                  /* once per device: the 200 KB cap */ \
    int dev = 0;                                                                               \
    cudaGetDevice(&dev);                                                                       \
    if (dev < 0 || dev >= 64) dev = 0;                                                         \
    if (!smem_set[dev]) {                                                                      \
      cudaFuncSetAttribute(route_simt_kernel<T, EM>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           200 * 1024);                                                        \
      smem_set[dev] = true;                                                                    \
    }                                                                                          \
    MOE_TRACED("route_simt", s,                                                                 \
               (route_simt_kernel<T, EM><<<blocks, threads, smem, s>>>(x, W_r, N, H, E, K, logits,  \
                                                                       probs, top, w)));       \
    MOE_LAUNCH_CHECK();                                                                        \
    return MOE_OK;                                                                             \
  }
  MOE_ROUTE_CASE(8)
  MOE_ROUTE_CASE(16)
  MOE_ROUTE_CASE(32)
  MOE_ROUTE_CASE(64)
#undef MOE_ROUTE_CASE
  return MOE_ERR_UNSUPPORTED;
}

bool route_simt_supported(int H, int E, int K, int elem_bytes) {
  return E <= 64 && K <= 32 && (size_t)H * E * elem_bytes <= 200 * 1024;
}

moe_status route_simt(const void* x, const void* W_r, int N, int H, int E, int K, moe_dtype dt,
                      float* logits, float* probs, int32_t* top, float* w, cudaStream_t s) {
  if (dt == MOE_F32)
    return launch_route_simt<float>((const float*)x, (const float*)W_r, N, H, E, K, logits, probs,
                                    top, w, s);
  return launch_route_simt<__nv_bfloat16>((const __nv_bfloat16*)x, (const __nv_bfloat16*)W_r, N,
                                          H, E, K, logits, probs, top, w, s);
}

}  // namespace moe

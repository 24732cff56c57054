// Auxiliary load-balancing loss ("MoE computation principle and execution",
// sec. 4.2): L_aux = alpha * E * sum_i f_i * P_i, with f_i = (assignments
// routed to expert i) / (N*K) and P_i = mean over tokens of probs[:, i].
// f_i counts the router's assignments to expert i before any capacity drop
// (routed_bins: their inclusive cumsum), so the loss does not depend on the
// token-dropping variant's capacity.
//
// Forward: per-chunk column sums of probs (256 tokens per chunk, increasing
// token order), then one block sums the chunks in order and forms the loss
// with a fixed-order tree over experts.
//
// Backward (dense router gradient, used when the loss is on and by the
// token-dropping variant, whose dropped assignments still pass gradient to
// the router through the renormalised weights): the counts f_i are piecewise
// constant, so d L_aux / d p_t,i = alpha*E*f_i/N and, through
// the softmax, the logits of every expert receive
//   a_t,e = g * alpha*E/N * p_t,e * (f_e - sum_i f_i p_t,i)      (g = dL/dL_aux)
// D[t,e] = a_t,e + the renormalisation gradient of token t's kept experts.
// Then dx[t] = sum_k dX_perm[pos(t,k)] + sum_e D[t,e] W_r[:,e] and
// dW_r = x^T D.  bf16 layers with E % 64 == 0 and H % 256 == 0 run both as
// tcgen05 GEMMs on D rounded once to bf16 (gemm_umma.cu); otherwise tiled
// fp32 CUDA-core reductions here.  Every sum runs in a fixed order.
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kAuxChunk = 256;

__global__ void __launch_bounds__(256)
aux_colsum_kernel(const float* __restrict__ probs, int N, int E, float* __restrict__ part) {
  const int c = blockIdx.x;
  const int t0 = c * kAuxChunk;
  const int t1 = t0 + kAuxChunk < N ? t0 + kAuxChunk : N;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = 0.f;
    for (int t = t0; t < t1; ++t) acc += probs[(size_t)t * E + e];
    part[(size_t)c * E + e] = acc;
  }
}

// One block of 256 threads (E <= 256).
__global__ void __launch_bounds__(256)
aux_finalize_kernel(const float* __restrict__ part, int n_chunks, const int32_t* __restrict__ routed_bins,
                    int N, int K, int E, float alpha, float* __restrict__ loss, float* __restrict__ P_out) {
  __shared__ float s_v[256];
  const int e = threadIdx.x;
  float v = 0.f;
  if (e < E) {
    float Pe = 0.f;
    for (int c = 0; c < n_chunks; ++c) Pe += part[(size_t)c * E + e];
    Pe /= (float)N;
    const float cnt = (float)(routed_bins[e] - (e ? routed_bins[e - 1] : 0));
    const float fe = cnt / ((float)N * (float)K);
    v = fe * Pe;
    if (P_out) P_out[e] = Pe;
  }
  s_v[e] = v;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {     // fixed pairwise tree
    if (e < off) s_v[e] += s_v[e + off];
    __syncthreads();
  }
  if (e == 0) *loss = alpha * (float)E * s_v[0];
}

// D[t, e] for one token per warp, into D (fp32) or Dh (bf16, for the
// tensor-core kernels, which also get the token-chunk ends chunk_end[c] =
// min((c + 1) * chunk, N rounded up to 64)).  probs and routed_bins are read
// only with the load-balancing term on (probs != NULL and coef != 0); without
// it D holds the renormalisation gradient alone (token dropping) and the
// router probabilities, which the forward then does not write, are not read.
// f_e = routed_bins[e] - routed_bins[e-1] counts the assignments the router
// made to expert e, before any capacity drop.
__global__ void __launch_bounds__(256)
router_dense_dlogits_kernel(const float* __restrict__ probs, const float* __restrict__ dlogit,
                            const int32_t* __restrict__ top, const int32_t* __restrict__ routed_bins, int N,
                            int E, int K, float coef, float* __restrict__ D, __nv_bfloat16* __restrict__ Dh,
                            int32_t* __restrict__ chunk_end, int chunk) {
  if (chunk_end && blockIdx.x == 0) {
    const int n_chunks = (N + chunk - 1) / chunk;
    const int last = (int)round_up(N, 64);
    for (int c = threadIdx.x; c < n_chunks; c += blockDim.x)
      chunk_end[c] = (c + 1) * chunk < last ? (c + 1) * chunk : last;
  }
  const bool aux = probs != nullptr && coef != 0.f;
  __shared__ float s_f[256];
  if (aux) {
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      s_f[e] = (float)(routed_bins[e] - (e ? routed_bins[e - 1] : 0)) / ((float)N * (float)K);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < N; t += warps) {
    const float* p = aux ? probs + (size_t)t * E : nullptr;
    float s = 0.f;
    if (aux) {
      float part = 0.f;
      for (int e = lane; e < E; e += 32) part = fmaf(s_f[e], p[e], part);
      s = warp_sum(part);
    }
    for (int e = lane; e < E; e += 32) {
      float d = aux ? coef * p[e] * (s_f[e] - s) : 0.f;
      for (int k = 0; k < K; ++k)
        if (top[(size_t)t * K + k] == e) d += dlogit[(size_t)t * K + k];
      if (Dh) Dh[(size_t)t * E + e] = __float2bfloat16(d);
      else D[(size_t)t * E + e] = d;
    }
  }
}

constexpr int kDT = 64;   // tile edge of the dense router kernels
constexpr int kDK = 16;   // reduction slice

// dx[t, h] = sum_k dX_perm[pos(t,k), h] + sum_e D[t,e] * W_r[h,e]
template <typename T>
__global__ void __launch_bounds__(256)
dense_router_dx_kernel(const T* __restrict__ dx_perm, const int32_t* __restrict__ pos,
                       const float* __restrict__ D, const T* __restrict__ W_r, int N, int H, int E, int K,
                       T* __restrict__ dx) {
  __shared__ float Ds[kDK][kDT + 4];
  __shared__ float Ws[kDK][kDT + 4];
  const int t0 = blockIdx.y * kDT, h0 = blockIdx.x * kDT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int e0 = 0; e0 < E; e0 += kDK) {
    for (int q = threadIdx.x; q < kDT * kDK; q += 256) {
      const int kk = q % kDK, r = q / kDK;
      const int t = t0 + r, h = h0 + r, e = e0 + kk;
      Ds[kk][r] = (t < N && e < E) ? D[(size_t)t * E + e] : 0.f;
      Ws[kk][r] = (h < H && e < E) ? to_f<T>(W_r[(size_t)h * E + e]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kDK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Ds[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int h = h0 + tx * 4 + j;
      if (h >= H) continue;
      float s = 0.f;
      for (int k = 0; k < K; ++k) {
        const int p = pos[(size_t)t * K + k];
        if (p >= 0) s += to_f<T>(dx_perm[(size_t)p * H + h]);
      }
      dx[(size_t)t * H + h] = from_f<T>(s + acc[i][j]);
    }
  }
}

// part[c][h][e] = sum over tokens of chunk c (in order) of x[t,h] * D[t,e]
template <typename T>
__global__ void __launch_bounds__(256)
dense_router_wgrad_partial_kernel(const T* __restrict__ x, const float* __restrict__ D, int N, int H, int E,
                                  int chunk, float* __restrict__ part) {
  __shared__ float Xs[kDK][kDT + 4];
  __shared__ float Ds[kDK][kDT + 4];
  const int h0 = blockIdx.x * kDT, e0 = blockIdx.y * kDT, c = blockIdx.z;
  const int tb = c * chunk, te = tb + chunk < N ? tb + chunk : N;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int t0 = tb; t0 < te; t0 += kDK) {
    for (int q = threadIdx.x; q < kDT * kDK; q += 256) {
      const int j = q % kDT, kk = q / kDT;
      const int t = t0 + kk;
      Xs[kk][j] = (t < te && h0 + j < H) ? to_f<T>(x[(size_t)t * H + h0 + j]) : 0.f;
      Ds[kk][j] = (t < te && e0 + j < E) ? D[(size_t)t * E + e0 + j] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kDK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ds[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int h = h0 + ty * 4 + i;
    if (h >= H) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) part[((size_t)c * H + h) * E + e] = acc[i][j];
    }
  }
}

template <typename T>
__global__ void dense_router_wgrad_reduce_kernel(const float* __restrict__ part, int n_chunks, int H, int E,
                                                 T* __restrict__ dWr) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)H * E) return;
  float acc = 0.f;
  for (int c = 0; c < n_chunks; ++c) acc += part[(size_t)c * H * E + idx];
  dWr[idx] = from_f<T>(acc);
}

constexpr int kWgradChunk = 1024;

size_t aux_loss_scratch(int N, int E) { return (size_t)cdiv(N > 0 ? N : 1, kAuxChunk) * E * sizeof(float); }

size_t dense_router_bwd_scratch(int N, int H, int E) {
  // fp32 D (or bf16 D) | partials: [chunks, H, E] fp32 of the CUDA-core
  // weight gradient, or those of the tensor-core one
  const int64_t chunks = cdiv(N > 0 ? N : 1, kWgradChunk);
  const size_t simt = (size_t)chunks * H * E * sizeof(float);
  const size_t tc = router_wgrad_tc_supported(H, E) ? router_wgrad_tc_scratch(N, H, E) : 0;
  return (size_t)round_up((int64_t)N * E * sizeof(float), 256) + (simt > tc ? simt : tc);
}

moe_status scatter_dlogits(const float* dlogit, const int32_t* top, int N, int E, int K, void* Dh, cudaStream_t s) {
  if (N == 0) return MOE_OK;
  int blocks = (int)cdiv(N, 8);
  if (blocks > 148 * 8) blocks = 148 * 8;
  MOE_TRACED("router_dlogits", s, (router_dense_dlogits_kernel<<<blocks, 256, 0, s>>>(
                                      nullptr, dlogit, top, nullptr, N, E, K, 0.f, nullptr, (__nv_bfloat16*)Dh,
                                      nullptr, 1)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status aux_loss_fwd(const float* probs, const int32_t* routed_bins, int N, int K, int E, float alpha,
                        float* loss, float* P, void* scratch, cudaStream_t s) {
  const int n_chunks = (int)cdiv(N > 0 ? N : 1, kAuxChunk);
  float* part = (float*)scratch;
  MOE_TRACED("aux_colsum", s, (aux_colsum_kernel<<<n_chunks, 256, 0, s>>>(probs, N, E, part)));
  MOE_LAUNCH_CHECK();
  MOE_TRACED("aux_finalize", s, (aux_finalize_kernel<<<1, 256, 0, s>>>(part, N > 0 ? n_chunks : 0,
                                                                       routed_bins, N > 0 ? N : 1, K, E, alpha,
                                                                       loss, P)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

template <typename T>
static moe_status dense_router_bwd_t(const void* dx_perm, const float* dlogit, const void* x, const void* W_r,
                                     const int32_t* top, const int32_t* pos, const int32_t* routed_bins,
                                     const float* probs, int N, int H, int E, int K, float coef, void* dx,
                                     void* dWr, void* scratch, int* status, cudaStream_t s) {
  float* D = (float*)scratch;
  float* part = (float*)((char*)scratch + round_up((int64_t)N * E * sizeof(float), 256));
  const int warps = 8;
  int blocks = (int)cdiv(N, warps);
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  if (std::is_same<T, __nv_bfloat16>::value && router_bwd_umma_supported(H, E)) {
    // tensor cores: D in bf16 (rounded once from the fp32 value), then
    // dx = D * W_r^T + unpermute sum and dW_r = x^T * D as tcgen05 GEMMs
    // scratch: Dh [N, E] bf16 (in D's place) | partials of x^T * D
    __nv_bfloat16* Dh = (__nv_bfloat16*)scratch;
    MOE_TRACED("router_dense_dlogits", s, (router_dense_dlogits_kernel<<<blocks, 256, 0, s>>>(
                                              probs, dlogit, top, routed_bins, N, E, K, coef, nullptr, Dh, nullptr,
                                              1)));
    MOE_LAUNCH_CHECK();
    moe_status st = router_dx_umma(Dh, W_r, N, H, E, dx, status, s);
    if (st == MOE_OK) st = unpermute_add_rows(dx_perm, pos, N, H, K, MOE_BF16, dx, s);
    if (st == MOE_OK) st = router_wgrad_tc(x, Dh, N, H, E, dWr, part, status, s);
    return st;
  }
  MOE_TRACED("router_dense_dlogits", s, (router_dense_dlogits_kernel<<<blocks, 256, 0, s>>>(
                                            probs, dlogit, top, routed_bins, N, E, K, coef, D, nullptr, nullptr, 1)));
  MOE_LAUNCH_CHECK();
  dim3 g1((unsigned)cdiv(H, kDT), (unsigned)cdiv(N, kDT));
  MOE_TRACED("dense_router_dx", s, (dense_router_dx_kernel<T><<<g1, 256, 0, s>>>(
                                       (const T*)dx_perm, pos, D, (const T*)W_r, N, H, E, K, (T*)dx)));
  MOE_LAUNCH_CHECK();
  const int n_chunks = (int)cdiv(N, kWgradChunk);
  dim3 g2((unsigned)cdiv(H, kDT), (unsigned)cdiv(E, kDT), (unsigned)n_chunks);
  MOE_TRACED("dense_router_wgrad_partial", s, (dense_router_wgrad_partial_kernel<T><<<g2, 256, 0, s>>>(
                                                  (const T*)x, D, N, H, E, kWgradChunk, part)));
  MOE_LAUNCH_CHECK();
  MOE_TRACED("dense_router_wgrad_reduce", s, (dense_router_wgrad_reduce_kernel<T><<<(unsigned)cdiv((int64_t)H * E, 256),
                                                 256, 0, s>>>(part, n_chunks, H, E, (T*)dWr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status dense_router_bwd(const void* dx_perm, const float* dlogit, const void* x, const void* W_r,
                            const int32_t* top, const int32_t* pos, const int32_t* routed_bins,
                            const float* probs, int N, int H, int E, int K, moe_dtype dt, float aux_alpha,
                            float aux_grad, void* dx, void* dWr, void* scratch, int* status, cudaStream_t s) {
  if (N == 0) return MOE_OK;
  // without the load-balancing term neither probs nor the counts are read
  const bool aux = aux_alpha != 0.0f && probs != nullptr;
  const float coef = aux ? aux_grad * aux_alpha * (float)E / (float)N : 0.0f;
  if (!aux) probs = nullptr;
  return dt == MOE_F32
             ? dense_router_bwd_t<float>(dx_perm, dlogit, x, W_r, top, pos, routed_bins, probs, N, H, E, K, coef,
                                         dx, dWr, scratch, status, s)
             : dense_router_bwd_t<__nv_bfloat16>(dx_perm, dlogit, x, W_r, top, pos, routed_bins, probs, N, H, E,
                                                 K, coef, dx, dWr, scratch, status, s);
}

}  // namespace moe

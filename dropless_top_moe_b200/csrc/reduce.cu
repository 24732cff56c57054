// Rank-ordered sum of gradient shards, the local step of a deterministic
// data-parallel gradient all-reduce: out[j] = scale * sum_{r=0..n-1} in[r][j],
// summed in increasing r in fp32, rounded once.  Every rank therefore obtains
// the same bits whatever order the collective delivered the shards in.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

template <typename T>
__global__ void __launch_bounds__(256)
sum_ordered_kernel(const T* __restrict__ in, int n, int64_t numel, float scale, T* __restrict__ out) {
  constexpr int V = Vec<T>::N;
  const int64_t nvec = numel / V;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.f;
    for (int r = 0; r < n; ++r) {
      float f[V];
      Vec<T>::to_float(ld_nc_v4(in + (size_t)r * numel + (size_t)v * V), f);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += f[j];
    }
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] *= scale;
    st_v4(out + (size_t)v * V, Vec<T>::from_float(acc));
  }
}

}  // namespace moe

extern "C" moe_status moe_sum_rank_ordered(const void* shards, int32_t n_ranks, int64_t numel,
                                           moe_dtype dt, float scale, void* out, moe_stream_t stream) {
  using namespace moe;
  if (!shards || !out || n_ranks <= 0 || numel < 0) return MOE_ERR_INVALID_ARG;
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (((uintptr_t)shards & 15u) || ((uintptr_t)out & 15u)) return MOE_ERR_INVALID_ARG;
  const int V = dt == MOE_F32 ? 4 : 8;
  if (numel % V) return MOE_ERR_UNSUPPORTED;
  if (numel == 0) return MOE_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t nvec = numel / V;
  int64_t blocks = cdiv(nvec, 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (dt == MOE_F32)
    MOE_TRACED("sum_rank_ordered", s, (sum_ordered_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(
                                          (const float*)shards, n_ranks, numel, scale, (float*)out)));
  else
    MOE_TRACED("sum_rank_ordered", s, (sum_ordered_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
                                          (const __nv_bfloat16*)shards, n_ranks, numel, scale,
                                          (__nv_bfloat16*)out)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// Row movement kernels of the layer: padded gather (permute), weighted
// combine, and their backward counterparts ("MegaBlocks - architecture",
// sec. 2.1 padded_gather / padded_scatter; sec. 4: the backward of a gather is
// a scatter and the reverse).  All are HBM-bound copies with fp32 arithmetic
// in registers; rows move as 16-byte vectors, one warp per token, lanes over
// consecutive vectors so a warp touches 512 contiguous bytes per step.
//
// Reductions (the K-sum of combine, the dot products of its backward, the
// K-sum of the unpermute) run in a fixed order: increasing k, then a fixed
// xor-butterfly across lanes.  No floating-point atomics anywhere.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kRowThreads = 256;
constexpr int kSeg = 4;   // 16-byte vectors per lane held in registers at once
// combine_bwd streams two rows (dy and the expert output) per segment; 8 vectors
// per lane measured 15 % faster there, and slower in the one-row kernels.  A
// lane visits its vectors in increasing order either way, so the fp32 dot
// products are the same bits.
constexpr int kSegBwd = 8;
// combine: expert rows whose loads are issued before any is summed (15 %
// faster at K = 4 on B200; the unpermute, with more registers live, was 14 %
// slower this way and keeps one row at a time)
constexpr int kRowBatch = 4;

__device__ __forceinline__ int grid_warp() { return (blockIdx.x * blockDim.x + threadIdx.x) >> 5; }
__device__ __forceinline__ int grid_warps() { return (gridDim.x * blockDim.x) >> 5; }

// Zero the pad rows of every expert group: rows [start_e + count_e, end_e).
template <typename T>
__device__ __forceinline__ void zero_pad_rows(const int32_t* bins, const int32_t* padded_bins, int E,
                                              int H, T* buf) {
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int nvec = H / V;
  for (int q = grid_warp(); q < E * kTile; q += grid_warps()) {
    const int e = q / kTile, j = q - e * kTile;
    const int64_t lo = e ? padded_bins[e - 1] : 0;
    const int64_t cnt = bins[e] - (e ? bins[e - 1] : 0);
    const int64_t row = lo + cnt + j;
    if (row >= padded_bins[e]) continue;
    T* dst = buf + row * H;
    for (int v = lane; v < nvec; v += 32) st_v4(dst + (size_t)v * V, make_uint4(0, 0, 0, 0));
  }
}

template <typename T>
__global__ void __launch_bounds__(kRowThreads)
permute_kernel(const T* __restrict__ x, const int32_t* __restrict__ pos, const int32_t* __restrict__ bins,
               const int32_t* __restrict__ padded_bins, int N, int H, int E, int K, T* __restrict__ x_perm) {
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int nvec = H / V;
  for (int t = grid_warp(); t < N; t += grid_warps()) {
    const int my_pos = lane < K ? pos[(size_t)t * K + lane] : -1;
    const T* src = x + (size_t)t * H;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kSeg) {
      uint4 buf[kSeg];
#pragma unroll
      for (int s = 0; s < kSeg; ++s) {
        const int v = v0 + s * 32 + lane;
        if (v < nvec) buf[s] = ld_nc_v4(src + (size_t)v * V);
      }
      for (int k = 0; k < K; ++k) {
        const int p = __shfl_sync(0xffffffffu, my_pos, k);
        if (p < 0) continue;
        T* dst = x_perm + (size_t)p * H;
#pragma unroll
        for (int s = 0; s < kSeg; ++s) {
          const int v = v0 + s * 32 + lane;
          if (v < nvec) st_v4(dst + (size_t)v * V, buf[s]);
        }
      }
    }
  }
  zero_pad_rows<T>(bins, padded_bins, E, H, x_perm);
}

template <typename T>
__global__ void __launch_bounds__(kRowThreads)
combine_kernel(const T* __restrict__ out, const float* __restrict__ weights, const int32_t* __restrict__ pos,
               int N, int K, int H, T* __restrict__ y) {
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int nvec = H / V;
  for (int t = grid_warp(); t < N; t += grid_warps()) {
    const int my_pos = lane < K ? pos[(size_t)t * K + lane] : -1;
    const float my_w = lane < K ? weights[(size_t)t * K + lane] : 0.f;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kSeg) {
      float acc[kSeg][V];
#pragma unroll
      for (int s = 0; s < kSeg; ++s)
#pragma unroll
        for (int j = 0; j < V; ++j) acc[s][j] = 0.f;
      // kRowBatch expert rows in flight at a time, summed in the fixed order
      // k = 0, 1, ...
      for (int k0 = 0; k0 < K; k0 += kRowBatch) {
        int p[kRowBatch];
        float w[kRowBatch];
        uint4 buf[kRowBatch][kSeg];
#pragma unroll
        for (int u = 0; u < kRowBatch; ++u) {
          p[u] = k0 + u < K ? __shfl_sync(0xffffffffu, my_pos, k0 + u) : -1;
          w[u] = k0 + u < K ? __shfl_sync(0xffffffffu, my_w, k0 + u) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kRowBatch; ++u) {
          if (p[u] < 0) continue;
          const T* src = out + (size_t)p[u] * H;
#pragma unroll
          for (int s = 0; s < kSeg; ++s) {
            const int v = v0 + s * 32 + lane;
            if (v < nvec) buf[u][s] = ld_nc_v4(src + (size_t)v * V);
          }
        }
#pragma unroll
        for (int u = 0; u < kRowBatch; ++u) {
          if (p[u] < 0) continue;
#pragma unroll
          for (int s = 0; s < kSeg; ++s) {
            const int v = v0 + s * 32 + lane;
            if (v < nvec) {
              float f[V];
              Vec<T>::to_float(buf[u][s], f);
#pragma unroll
              for (int j = 0; j < V; ++j) acc[s][j] = fmaf(w[u], f[j], acc[s][j]);
            }
          }
        }
      }
#pragma unroll
      for (int s = 0; s < kSeg; ++s) {
        const int v = v0 + s * 32 + lane;
        if (v < nvec) st_v4(y + (size_t)t * H + (size_t)v * V, Vec<T>::from_float(acc[s]));
      }
    }
  }
}

// dw = <dy, out[pos]>, d_out[pos] = w * dy, dlogit = w * (dw - <w, dw>);
// with Dh, also the token's row of D: dlogit at its K experts, 0 elsewhere.
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
combine_bwd_kernel(const T* __restrict__ dy, const T* __restrict__ out, const float* __restrict__ weights,
                   const int32_t* __restrict__ pos, const int32_t* __restrict__ bins,
                   const int32_t* __restrict__ padded_bins, int N, int K, int H, int E,
                   float* __restrict__ dw, float* __restrict__ dlogit, T* __restrict__ d_out,
                   const int32_t* __restrict__ top, __nv_bfloat16* __restrict__ Dh) {
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int nvec = H / V;
  for (int t = grid_warp(); t < N; t += grid_warps()) {
    const int my_pos = lane < K ? pos[(size_t)t * K + lane] : -1;
    const float my_w = lane < K ? weights[(size_t)t * K + lane] : 0.f;
    const T* g = dy + (size_t)t * H;
    float my_dw = 0.f;
    for (int k = 0; k < K; ++k) {
      const int p = __shfl_sync(0xffffffffu, my_pos, k);
      const float w = __shfl_sync(0xffffffffu, my_w, k);
      float dot = 0.f;
      if (p >= 0) {
        const T* o = out + (size_t)p * H;
        T* d = d_out + (size_t)p * H;
        for (int v0 = lane; v0 < nvec; v0 += 32 * kSegBwd) {
          uint4 gv[kSegBwd], ov[kSegBwd];    // issue all loads of the segment first
#pragma unroll
          for (int u = 0; u < kSegBwd; ++u) {
            const int v = v0 + 32 * u;
            if (v < nvec) {
              gv[u] = ld_nc_v4(g + (size_t)v * V);
              ov[u] = ld_nc_v4(o + (size_t)v * V);
            }
          }
#pragma unroll
          for (int u = 0; u < kSegBwd; ++u) {
            const int v = v0 + 32 * u;
            if (v < nvec) {
              float gf[V], of[V], df[V];
              Vec<T>::to_float(gv[u], gf);
              Vec<T>::to_float(ov[u], of);
#pragma unroll
              for (int j = 0; j < V; ++j) {
                dot = fmaf(gf[j], of[j], dot);
                df[j] = w * gf[j];
              }
              st_v4(d + (size_t)v * V, Vec<T>::from_float(df));
            }
          }
        }
      }
      dot = warp_sum(dot);
      if (lane == k) my_dw = dot;
    }
    const float s = warp_sum(lane < K ? my_w * my_dw : 0.f);
    const float my_dl = my_w * (my_dw - s);
    if (lane < K) {
      if (dw) dw[(size_t)t * K + lane] = my_dw;
      dlogit[(size_t)t * K + lane] = my_dl;
    }
    if (Dh) {
      // lane writes experts 2*lane + 64*j and the next one (E <= 256, E even)
      const int my_e = lane < K ? top[(size_t)t * K + lane] : -1;
      float v[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      for (int k = 0; k < K; ++k) {
        const int ek = __shfl_sync(0xffffffffu, my_e, k);
        const float dk = __shfl_sync(0xffffffffu, my_dl, k);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 2 * lane + 64 * j;
          if (ek == e) v[j][0] = dk;
          if (ek == e + 1) v[j][1] = dk;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 2 * lane + 64 * j;
        if (e < E)
          *reinterpret_cast<uint32_t*>(Dh + (size_t)t * E + e) = pack_bf16x2(v[j][0], v[j][1]);
      }
    }
  }
  zero_pad_rows<T>(bins, padded_bins, E, H, d_out);
}

// outT[c][r] = in[r][c] for c < C, and 0 for C <= c < C_pad (zero rows that
// pad a transposed operand to an MMA width), through a shared-memory tile.
// status != NULL: the layer backward's first launch also checks the flags the
// forward recorded (status[1]) against `expect`, setting MOE_DEVERR_MODE.
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ in, int R, int C, int C_pad, T* __restrict__ outT,
                                 int* status, int expect) {
  if (status && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0 && status[1] != expect)
    atomicOr(status, MOE_DEVERR_MODE);
  __shared__ T tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C_pad) tile[i][threadIdx.x] = c < C ? in[(size_t)r * C + c] : from_f<T>(0.f);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C_pad) outT[(size_t)c * R + r] = tile[threadIdx.x][i];
  }
}

// dx[t] = sum_k dx_perm[pos[t,k]] + sum_k dlogit[t,k] * W_rT[top[t,k]];
// with ADD the second term is dx[t]'s own value instead (read, then
// overwritten by the same thread): the dense router backward stores its
// D * W_r^T there first.
template <typename T, bool ADD = false>
__global__ void __launch_bounds__(kRowThreads)
unpermute_dx_kernel(const T* __restrict__ dx_perm, const float* __restrict__ dlogit,
                    const T* __restrict__ WrT, const int32_t* __restrict__ top,
                    const int32_t* __restrict__ pos, int N, int H, int K, T* __restrict__ dx) {
  constexpr int V = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int nvec = H / V;
  for (int t = grid_warp(); t < N; t += grid_warps()) {
    const int my_pos = lane < K ? pos[(size_t)t * K + lane] : -1;
    const float my_dl = (!ADD && lane < K) ? dlogit[(size_t)t * K + lane] : 0.f;
    const int my_e = (!ADD && lane < K) ? top[(size_t)t * K + lane] : 0;
    for (int v0 = 0; v0 < nvec; v0 += 32 * kSeg) {
      float acc[kSeg][V];
#pragma unroll
      for (int s = 0; s < kSeg; ++s)
#pragma unroll
        for (int j = 0; j < V; ++j) acc[s][j] = 0.f;
      for (int k = 0; k < K; ++k) {
        const int p = __shfl_sync(0xffffffffu, my_pos, k);
        if (p < 0) continue;
        const T* src = dx_perm + (size_t)p * H;
#pragma unroll
        for (int s = 0; s < kSeg; ++s) {
          const int v = v0 + s * 32 + lane;
          if (v < nvec) {
            float f[V];
            Vec<T>::to_float(ld_nc_v4(src + (size_t)v * V), f);
#pragma unroll
            for (int j = 0; j < V; ++j) acc[s][j] += f[j];
          }
        }
      }
      if constexpr (ADD) {
        const T* add = dx + (size_t)t * H;
#pragma unroll
        for (int s = 0; s < kSeg; ++s) {
          const int v = v0 + s * 32 + lane;
          if (v < nvec) {
            float f[V];
            Vec<T>::to_float(*reinterpret_cast<const uint4*>(add + (size_t)v * V), f);
#pragma unroll
            for (int j = 0; j < V; ++j) acc[s][j] += f[j];
          }
        }
      }
      for (int k = 0; k < (ADD ? 0 : K); ++k) {
        const int p = __shfl_sync(0xffffffffu, my_pos, k);
        const float dl = __shfl_sync(0xffffffffu, my_dl, k);
        const int e = __shfl_sync(0xffffffffu, my_e, k);
        if (p < 0) continue;
        const T* wr = WrT + (size_t)e * H;
#pragma unroll
        for (int s = 0; s < kSeg; ++s) {
          const int v = v0 + s * 32 + lane;
          if (v < nvec) {
            float f[V];
            Vec<T>::to_float(ld_nc_v4(wr + (size_t)v * V), f);
#pragma unroll
            for (int j = 0; j < V; ++j) acc[s][j] = fmaf(dl, f[j], acc[s][j]);
          }
        }
      }
#pragma unroll
      for (int s = 0; s < kSeg; ++s) {
        const int v = v0 + s * 32 + lane;
        if (v < nvec) st_v4(dx + (size_t)t * H + (size_t)v * V, Vec<T>::from_float(acc[s]));
      }
    }
  }
}

// Partial dW_r columns: block (tile m of 128 sorted assignments of one expert,
// column slice).  part[m][h] = sum over the tile's assignments, in sorted order,
// of dlogit_i * x[token(i)][h].
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
router_wgrad_partial_kernel(const float* __restrict__ dlogit, const T* __restrict__ x,
                            const int32_t* __restrict__ indices, const int32_t* __restrict__ bins,
                            const int32_t* __restrict__ padded_bins, int E, int H, int K,
                            float* __restrict__ part) {
  constexpr int V = Vec<T>::N;
  const int64_t m = blockIdx.x;
  const int64_t row0 = m * kTile;
  if (row0 >= padded_bins[E - 1]) return;
  const int e = expert_of_row(padded_bins, E, row0);
  const int64_t pstart = e ? padded_bins[e - 1] : 0;
  const int64_t sstart = e ? bins[e - 1] : 0;
  const int64_t cnt = bins[e] - sstart;
  const int64_t r0 = row0 - pstart;                       // rank of the tile's first row
  const int64_t r1 = (r0 + kTile < cnt) ? r0 + kTile : cnt;
  const int h0 = (blockIdx.y * blockDim.x + threadIdx.x) * V;
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  // the tile's assignment ids and their dlogits, staged once per block
  __shared__ int s_row[kTile];
  __shared__ float s_dl[kTile];
  for (int q = threadIdx.x; q < kTile; q += blockDim.x) {
    const int64_t r = r0 + q;
    const int i = r < r1 ? indices[sstart + r] : -1;
    s_row[q] = i >= 0 ? i / K : -1;
    s_dl[q] = i >= 0 ? dlogit[i] : 0.f;
  }
  __syncthreads();
  if (h0 >= H) return;
  constexpr int U = 8;                      // rows in flight; summed in increasing r
  for (int q0 = 0; q0 < (int)(r1 - r0); q0 += U) {
    int idx[U];
    float dl[U];
    uint4 xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      idx[u] = (q0 + u < (int)(r1 - r0)) ? s_row[q0 + u] : -1;
      dl[u] = s_dl[q0 + u < kTile ? q0 + u : 0];
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (idx[u] >= 0) xv[u] = ld_nc_v4(x + (size_t)idx[u] * H + h0);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (idx[u] >= 0) {
        float f[V];
        Vec<T>::to_float(xv[u], f);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = fmaf(dl[u], f[j], acc[j]);
      }
    }
  }
  float* dst = part + m * H + h0;
#pragma unroll
  for (int j = 0; j < V; ++j) dst[j] = acc[j];
}

// dW_r[h][e] = sum over the expert's tiles m, in increasing m, of part[m][h].
template <typename T>
__global__ void router_wgrad_reduce_kernel(const float* __restrict__ part, const int32_t* __restrict__ padded_bins,
                                           int E, int H, T* __restrict__ dWr) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  const int e = blockIdx.y;
  if (h >= H) return;
  const int64_t m0 = (e ? padded_bins[e - 1] : 0) / kTile, m1 = padded_bins[e] / kTile;
  float acc = 0.f;
  for (int64_t m = m0; m < m1; ++m) acc += part[m * H + h];
  dWr[(size_t)h * E + e] = from_f<T>(acc);
}

static int row_grid(int64_t rows) {
  const int64_t warps = rows > 0 ? rows : 1;
  int64_t blocks = cdiv(warps, kRowThreads / 32);
  const int64_t cap = 148 * 16;
  return (int)(blocks < cap ? blocks : cap);
}

template <typename T>
static moe_status permute_t(const void* x, const int32_t* pos, const int32_t* bins, const int32_t* pb,
                            int N, int H, int E, int K, void* x_perm, cudaStream_t s) {
  const int64_t work = (int64_t)N > (int64_t)E * kTile ? N : (int64_t)E * kTile;
  MOE_TRACED("permute", s, (permute_kernel<T><<<row_grid(work), kRowThreads, 0, s>>>((const T*)x, pos, bins, pb, N, H, E, K,
                                                           (T*)x_perm)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status permute_rows(const void* x, const int32_t* pos, const int32_t* bins, const int32_t* pb,
                        int N, int H, int E, int K, moe_dtype dt, void* x_perm, cudaStream_t s) {
  return dt == MOE_F32 ? permute_t<float>(x, pos, bins, pb, N, H, E, K, x_perm, s)
                       : permute_t<__nv_bfloat16>(x, pos, bins, pb, N, H, E, K, x_perm, s);
}

template <typename T>
static moe_status combine_t(const void* out, const float* w, const int32_t* pos, int N, int K, int H,
                            void* y, cudaStream_t s) {
  MOE_TRACED("combine", s, (combine_kernel<T><<<row_grid(N), kRowThreads, 0, s>>>((const T*)out, w, pos, N, K, H, (T*)y)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status combine_rows(const void* out, const float* w, const int32_t* pos, int N, int K, int H,
                        moe_dtype dt, void* y, cudaStream_t s) {
  return dt == MOE_F32 ? combine_t<float>(out, w, pos, N, K, H, y, s)
                       : combine_t<__nv_bfloat16>(out, w, pos, N, K, H, y, s);
}

template <typename T>
static moe_status combine_bwd_t(const void* dy, const void* out, const float* w, const int32_t* pos,
                                const int32_t* bins, const int32_t* pb, int N, int K, int H, int E,
                                float* dw, float* dlogit, void* d_out, cudaStream_t s, const int32_t* top,
                                void* Dh) {
  const int64_t work = (int64_t)N > (int64_t)E * kTile ? N : (int64_t)E * kTile;
  MOE_TRACED("combine_bwd", s, (combine_bwd_kernel<T><<<row_grid(work), kRowThreads, 0, s>>>(
      (const T*)dy, (const T*)out, w, pos, bins, pb, N, K, H, E, dw, dlogit, (T*)d_out, top,
      (__nv_bfloat16*)Dh)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status combine_bwd_rows(const void* dy, const void* out, const float* w, const int32_t* pos,
                            const int32_t* bins, const int32_t* pb, int N, int K, int H, int E,
                            moe_dtype dt, float* dw, float* dlogit, void* d_out, cudaStream_t s,
                            const int32_t* top, void* Dh) {
  if (Dh && (E % 2 != 0 || E > 256 || !top)) return MOE_ERR_INVALID_ARG;
  return dt == MOE_F32
             ? combine_bwd_t<float>(dy, out, w, pos, bins, pb, N, K, H, E, dw, dlogit, d_out, s, top, Dh)
             : combine_bwd_t<__nv_bfloat16>(dy, out, w, pos, bins, pb, N, K, H, E, dw, dlogit, d_out, s, top,
                                            Dh);
}

moe_status transpose_matrix(const void* in, int R, int C, moe_dtype dt, void* outT, cudaStream_t s,
                            int C_pad, int* status, int expect) {
  if (C_pad < C) C_pad = C;
  dim3 grid((unsigned)cdiv(C_pad, 32), (unsigned)cdiv(R, 32)), block(32, 8);
  if (dt == MOE_F32)
    MOE_TRACED("transpose", s, (transpose_kernel<float><<<grid, block, 0, s>>>((const float*)in, R, C, C_pad,
                                                                                (float*)outT, status, expect)));
  else
    MOE_TRACED("transpose", s, (transpose_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
                                   (const __nv_bfloat16*)in, R, C, C_pad, (__nv_bfloat16*)outT, status, expect)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// Scratch of the sparse router backward, in order (256-byte aligned):
// W_r^T [E, H] (at most fp32) | per-tile partials of the CUDA-core weight
// gradient [P/128, H] fp32 | D [N, E] bf16 | partials of the tensor-core one.
namespace {
size_t al256b(size_t b) { return (b + 255) & ~(size_t)255; }
}  // namespace

size_t unpermute_router_bwd_scratch(int N, int H, int E, int64_t P) {
  return al256b((size_t)E * H * 4) + al256b((size_t)(P / kTile) * H * sizeof(float)) +
         al256b((size_t)N * E * 2) + al256b(router_wgrad_tc_scratch(N, H, E));
}

void* unpermute_router_bwd_dh(void* scratch, int N, int H, int E, int64_t P) {
  (void)N;
  return (char*)scratch + al256b((size_t)E * H * 4) + al256b((size_t)(P / kTile) * H * sizeof(float));
}

template <typename T>
static moe_status unpermute_router_bwd_t(const void* dx_perm, const float* dlogit, const void* x,
                                         const void* W_r, const int32_t* top, const int32_t* pos,
                                         const int32_t* indices, const int32_t* bins,
                                         const int32_t* padded_bins, int N, int H, int E, int K,
                                         int64_t P, void* dx, void* dWr, void* scratch, int* status,
                                         cudaStream_t s, bool dh_ready, bool wrt_ready) {
  T* WrT = (T*)scratch;
  float* part = (float*)((char*)scratch + al256b((size_t)E * H * 4));
  moe_status st = MOE_OK;
  if (!wrt_ready) {
    st = transpose_matrix(W_r, H, E, sizeof(T) == 4 ? MOE_F32 : MOE_BF16, WrT, s);
    if (st != MOE_OK) return st;
  }
  MOE_TRACED("unpermute_dx", s, (unpermute_dx_kernel<T><<<row_grid(N), kRowThreads, 0, s>>>((const T*)dx_perm, dlogit, WrT, top, pos,
                                                             N, H, K, (T*)dx)));
  MOE_LAUNCH_CHECK();
  if (sizeof(T) == 2 && router_wgrad_tc_supported(H, E)) {
    // dW_r = x^T D on the tensor cores, x read once (D: the dlogits at each
    // token's experts, rounded once to bf16)
    void* Dh = unpermute_router_bwd_dh(scratch, N, H, E, P);
    if (!dh_ready) {
      st = scatter_dlogits(dlogit, top, N, E, K, Dh, s);
      if (st != MOE_OK) return st;
    }
    void* tc_part = (char*)Dh + al256b((size_t)N * E * 2);
    return router_wgrad_tc(x, Dh, N, H, E, dWr, tc_part, status, s);
  }
  constexpr int V = Vec<T>::N;
  dim3 g1((unsigned)(P / kTile), (unsigned)cdiv(H, kRowThreads * V));
  MOE_TRACED("router_wgrad_partial", s, (router_wgrad_partial_kernel<T><<<g1, kRowThreads, 0, s>>>(dlogit, (const T*)x, indices, bins,
                                                            padded_bins, E, H, K, part)));
  MOE_LAUNCH_CHECK();
  dim3 g2((unsigned)cdiv(H, 256), (unsigned)E);
  MOE_TRACED("router_wgrad_reduce", s, (router_wgrad_reduce_kernel<T><<<g2, 256, 0, s>>>(part, padded_bins, E, H, (T*)dWr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status unpermute_add_rows(const void* dx_perm, const int32_t* pos, int N, int H, int K, moe_dtype dt,
                              void* dx, cudaStream_t s) {
  if (N == 0) return MOE_OK;
  if (dt == MOE_F32) {
    MOE_TRACED("unpermute_dx", s, (unpermute_dx_kernel<float, true><<<row_grid(N), kRowThreads, 0, s>>>(
                                      (const float*)dx_perm, nullptr, nullptr, nullptr, pos, N, H, K, (float*)dx)));
  } else {
    MOE_TRACED("unpermute_dx", s, (unpermute_dx_kernel<__nv_bfloat16, true><<<row_grid(N), kRowThreads, 0, s>>>(
                                      (const __nv_bfloat16*)dx_perm, nullptr, nullptr, nullptr, pos, N, H, K,
                                      (__nv_bfloat16*)dx)));
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status unpermute_router_bwd(const void* dx_perm, const float* dlogit, const void* x,
                                const void* W_r, const int32_t* top, const int32_t* pos,
                                const int32_t* indices, const int32_t* bins, const int32_t* padded_bins,
                                int N, int H, int E, int K, int64_t P, moe_dtype dt, void* dx, void* dWr,
                                void* scratch, int* status, cudaStream_t s, bool dh_ready, bool wrt_ready) {
  return dt == MOE_F32
             ? unpermute_router_bwd_t<float>(dx_perm, dlogit, x, W_r, top, pos, indices, bins, padded_bins, N, H,
                                             E, K, P, dx, dWr, scratch, status, s, dh_ready, wrt_ready)
             : unpermute_router_bwd_t<__nv_bfloat16>(dx_perm, dlogit, x, W_r, top, pos, indices, bins,
                                                     padded_bins, N, H, E, K, P, dx, dWr, scratch, status, s,
                                                     dh_ready, wrt_ready);
}

}  // namespace moe

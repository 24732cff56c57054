// Grouped expert GEMMs on CUDA cores, used for MOE_F32 layers so that
// single-precision results keep full fp32 accuracy (the tensor-core paths
// round operands to bf16 / tf32).  Same grouping as the tensor-core kernels:
// every 64-row block of the padded rows lies inside one expert's group, whose
// expert is found from the device-side padded_bins (no host sync).
//
// rows mode   C[r, n] = sum_k A[r, k] * B_e(k, n)   (+ a second A, B pair)
//             with B_e(k, n) = B[e*sBe + k*sBk + n*sBn], so W and W^T are both
//             reachable by strides; epilogues: plain store, SwiGLU forward,
//             SwiGLU backward.
// wgrad mode  C_e[m, n] = sum over the group's rows r of A[r, m] * B[r, n]
// Accumulation is fp32 in increasing k: deterministic.  The next k slice is
// loaded into registers while the current one is multiplied from shared
// memory (small layers are latency-bound: one global round trip per slice).
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kSB = 64;   // block tile (rows and columns)
constexpr int kSK = 32;   // k slice
constexpr int kSL = kSB * kSK / 256;   // elements of a slice each thread loads, per operand

enum SimtEpi { SIMT_STORE = 0, SIMT_SWIGLU = 1, SIMT_SWIGLU_BWD = 2, SIMT_DUAL = 3 };

template <typename T, int EPI>
__global__ void __launch_bounds__(256)
gemm_rows_simt_kernel(const T* __restrict__ A0, const T* __restrict__ A1, int64_t lda,
                      const T* __restrict__ B0, const T* __restrict__ B1, int64_t sBe, int64_t sBk,
                      int64_t sBn, const int32_t* __restrict__ padded_bins, int E, int Kd, int Nd,
                      T* __restrict__ C0, T* __restrict__ C1, T* __restrict__ C2, int64_t ldc,
                      const T* __restrict__ aux0, const T* __restrict__ aux1) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  __shared__ float Bs2[(EPI == SIMT_SWIGLU) ? kSK : 1][kSB + 4];
  const int64_t row0 = (int64_t)blockIdx.y * kSB;
  const int n0 = blockIdx.x * kSB;
  if (row0 >= padded_bins[E - 1]) return;
  const int e = expert_of_row(padded_bins, E, row0);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4], acc2[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) { acc[i][j] = 0.f; acc2[i][j] = 0.f; }

  const int passes = (EPI == SIMT_DUAL) ? 2 : 1;
  const int nsl = (Kd + kSK - 1) / kSK, total = passes * nsl;
  float ra[kSL], rb[kSL], rb2[(EPI == SIMT_SWIGLU) ? kSL : 1];
  // slice sl: pass sl / nsl (SIMT_DUAL's second A, B pair), k from (sl % nsl) * kSK
  auto fetch = [&](int sl) {
    const int pass = sl / nsl, k0 = (sl % nsl) * kSK;
    const T* A = pass ? A1 : A0;
    const T* B = pass ? B1 : B0;
#pragma unroll
    for (int l = 0; l < kSL; ++l) {
      const int q = (int)threadIdx.x + l * 256;
      const int r = q / kSK, k = k0 + q % kSK;
      ra[l] = (k < Kd) ? to_f<T>(A[(row0 + r) * lda + k]) : 0.f;
      const int c = q % kSB, kb_k = k0 + q / kSB;
      const int64_t boff = (int64_t)e * sBe + (int64_t)kb_k * sBk + (int64_t)(n0 + c) * sBn;
      const bool ok = kb_k < Kd && n0 + c < Nd;
      rb[l] = ok ? to_f<T>(B[boff]) : 0.f;
      if (EPI == SIMT_SWIGLU) rb2[l] = ok ? to_f<T>(B1[boff]) : 0.f;
    }
  };
  fetch(0);
  for (int sl = 0; sl < total; ++sl) {
#pragma unroll
    for (int l = 0; l < kSL; ++l) {
      const int q = (int)threadIdx.x + l * 256;
      As[q % kSK][q / kSK] = ra[l];
      Bs[q / kSB][q % kSB] = rb[l];
      if (EPI == SIMT_SWIGLU) Bs2[q / kSB][q % kSB] = rb2[l];
    }
    __syncthreads();
    if (sl + 1 < total) fetch(sl + 1);
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      float a[4], b[4], b2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[j] = Bs[kk][tx * 4 + j];
        if (EPI == SIMT_SWIGLU) b2[j] = Bs2[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (EPI == SIMT_SWIGLU) acc2[i][j] = fmaf(a[i], b2[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = row0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= Nd) continue;
      const int64_t o = r * ldc + n;
      if (EPI == SIMT_STORE || EPI == SIMT_DUAL) {
        C0[o] = from_f<T>(acc[i][j]);
      } else if (EPI == SIMT_SWIGLU) {
        const float g = acc[i][j], u = acc2[i][j];
        if (C0) C0[o] = from_f<T>(silu_f(g) * u);
        if (C1) C1[o] = from_f<T>(g);
        if (C2) C2[o] = from_f<T>(u);
      } else {  // SIMT_SWIGLU_BWD: acc = dA, aux0 = G, aux1 = U
        const float g = to_f<T>(aux0[o]), u = to_f<T>(aux1[o]), da = acc[i][j];
        const float sig = 1.f / (1.f + expf(-g));
        C0[o] = from_f<T>(da * u * sig * (1.f + g * (1.f - sig)));
        C1[o] = from_f<T>(da * g * sig);
      }
    }
  }
}

// C_e[m, n] = sum_{r in group e} A[r, m] * B[r, n]; C_e at C + e*sCe, row stride ldc.
template <typename T>
__global__ void __launch_bounds__(256)
gemm_wgrad_simt_kernel(const T* __restrict__ A, int64_t lda, const T* __restrict__ B, int64_t ldb,
                       const int32_t* __restrict__ padded_bins, int Md, int Nd, T* __restrict__ C,
                       int64_t sCe, int64_t ldc) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  const int e = blockIdx.z;
  const int m0 = blockIdx.y * kSB, n0 = blockIdx.x * kSB;
  const int64_t r_begin = e ? padded_bins[e - 1] : 0, r_end = padded_bins[e];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  float ra[kSL], rb[kSL];
  auto fetch = [&](int64_t r0) {
#pragma unroll
    for (int l = 0; l < kSL; ++l) {
      const int q = (int)threadIdx.x + l * 256;
      const int c = q % kSB;
      const int64_t r = r0 + q / kSB;
      ra[l] = (r < r_end && m0 + c < Md) ? to_f<T>(A[r * lda + m0 + c]) : 0.f;
      rb[l] = (r < r_end && n0 + c < Nd) ? to_f<T>(B[r * ldb + n0 + c]) : 0.f;
    }
  };
  if (r_begin < r_end) fetch(r_begin);
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kSK) {
#pragma unroll
    for (int l = 0; l < kSL; ++l) {
      const int q = (int)threadIdx.x + l * 256;
      As[q / kSB][q % kSB] = ra[l];
      Bs[q / kSB][q % kSB] = rb[l];
    }
    __syncthreads();
    if (r0 + kSK < r_end) fetch(r0 + kSK);
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= Md) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < Nd) C[(int64_t)e * sCe + (int64_t)m * ldc + n] = from_f<T>(acc[i][j]);
    }
  }
}

template <typename T>
static moe_status swiglu_fwd_simt_t(const void* x_perm, const void* W1, const void* W3, const void* W2,
                                    const int32_t* pb, int E, int H, int F, int64_t P, void* act,
                                    void* out, void* gate_up, cudaStream_t s) {
  T* G = gate_up ? (T*)gate_up : nullptr;
  T* U = gate_up ? (T*)gate_up + (size_t)P * F : nullptr;
  dim3 g1((unsigned)cdiv(F, kSB), (unsigned)(P / kSB));
  // G, U = X W1_e, X W3_e ; W1 [E,H,F]: B(e,k=h,n=f) = W1[e*H*F + h*F + f]
  MOE_TRACED("simt_gemm1_swiglu", s, (gemm_rows_simt_kernel<T, SIMT_SWIGLU><<<g1, 256, 0, s>>>(
      (const T*)x_perm, nullptr, H, (const T*)W1, (const T*)W3, (int64_t)H * F, F, 1, pb, E, H, F,
      (T*)act, G, U, F, nullptr, nullptr)));
  MOE_LAUNCH_CHECK();
  dim3 g2((unsigned)cdiv(H, kSB), (unsigned)(P / kSB));
  // O = A W2_e ; W2 [E,F,H]
  MOE_TRACED("simt_gemm2", s, (gemm_rows_simt_kernel<T, SIMT_STORE><<<g2, 256, 0, s>>>(
      (const T*)act, nullptr, F, (const T*)W2, nullptr, (int64_t)F * H, H, 1, pb, E, F, H, (T*)out,
      nullptr, nullptr, H, nullptr, nullptr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status grouped_swiglu_simt(const void* x_perm, const void* W1, const void* W3, const void* W2,
                               const int32_t* pb, int E, int H, int F, int64_t P, moe_dtype dt,
                               void* act, void* out, void* gate_up, cudaStream_t s) {
  if (dt != MOE_F32) return MOE_ERR_UNSUPPORTED;
  return swiglu_fwd_simt_t<float>(x_perm, W1, W3, W2, pb, E, H, F, P, act, out, gate_up, s);
}

template <typename T>
static moe_status swiglu_bwd_simt_t(const void* d_out, const void* x_perm, const void* act,
                                    const void* gate_up, const void* W1, const void* W3, const void* W2,
                                    const int32_t* pb, int E, int H, int F, int64_t P, void* d_gate_up,
                                    void* dW1, void* dW3, void* dW2, void* dx_perm, cudaStream_t s) {
  const T* G = (const T*)gate_up;
  const T* U = G + (size_t)P * F;
  T* dG = (T*)d_gate_up;
  T* dU = dG + (size_t)P * F;
  // dA = dO W2_e^T : B(e,k=h,n=f) = W2[e*F*H + f*H + h]  -> sBk = 1, sBn = H
  dim3 g1((unsigned)cdiv(F, kSB), (unsigned)(P / kSB));
  MOE_TRACED("simt_dgrad_w2_swiglu_bwd", s, (gemm_rows_simt_kernel<T, SIMT_SWIGLU_BWD><<<g1, 256, 0, s>>>(
      (const T*)d_out, nullptr, H, (const T*)W2, nullptr, (int64_t)F * H, 1, H, pb, E, H, F, dG, dU,
      nullptr, F, G, U)));
  MOE_LAUNCH_CHECK();
  // dW2_e = act^T dO  [F,H];  dW1_e = X^T dG, dW3_e = X^T dU  [H,F]
  dim3 gw2((unsigned)cdiv(H, kSB), (unsigned)cdiv(F, kSB), (unsigned)E);
  MOE_TRACED("simt_wgrad_w2", s, (gemm_wgrad_simt_kernel<T><<<gw2, 256, 0, s>>>((const T*)act, F, (const T*)d_out, H, pb, F, H,
                                                (T*)dW2, (int64_t)F * H, H)));
  MOE_LAUNCH_CHECK();
  dim3 gw1((unsigned)cdiv(F, kSB), (unsigned)cdiv(H, kSB), (unsigned)E);
  MOE_TRACED("simt_wgrad_w1", s, (gemm_wgrad_simt_kernel<T><<<gw1, 256, 0, s>>>((const T*)x_perm, H, dG, F, pb, H, F, (T*)dW1,
                                                (int64_t)H * F, F)));
  MOE_LAUNCH_CHECK();
  MOE_TRACED("simt_wgrad_w3", s, (gemm_wgrad_simt_kernel<T><<<gw1, 256, 0, s>>>((const T*)x_perm, H, dU, F, pb, H, F, (T*)dW3,
                                                (int64_t)H * F, F)));
  MOE_LAUNCH_CHECK();
  // dx_perm = dG W1_e^T + dU W3_e^T : B(e,k=f,n=h) = W1[e*H*F + h*F + f] -> sBk = 1, sBn = F
  dim3 g3((unsigned)cdiv(H, kSB), (unsigned)(P / kSB));
  MOE_TRACED("simt_dgrad_x", s, (gemm_rows_simt_kernel<T, SIMT_DUAL><<<g3, 256, 0, s>>>(
      dG, dU, F, (const T*)W1, (const T*)W3, (int64_t)H * F, 1, F, pb, E, F, H, (T*)dx_perm, nullptr,
      nullptr, H, nullptr, nullptr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status grouped_swiglu_bwd_simt(const void* d_out, const void* x_perm, const void* act,
                                   const void* gate_up, const void* W1, const void* W3, const void* W2,
                                   const int32_t* pb, int E, int H, int F, int64_t P, moe_dtype dt,
                                   void* d_gate_up, void* dW1, void* dW3, void* dW2, void* dx_perm,
                                   cudaStream_t s) {
  if (dt != MOE_F32) return MOE_ERR_UNSUPPORTED;
  return swiglu_bwd_simt_t<float>(d_out, x_perm, act, gate_up, W1, W3, W2, pb, E, H, F, P, d_gate_up,
                                  dW1, dW3, dW2, dx_perm, s);
}

}  // namespace moe

namespace moe {

// G, U = X W1_e, X W3_e only (the backward's recompute of the saved gates).
moe_status gate_up_simt(const void* x_perm, const void* W1, const void* W3, const int32_t* pb, int E, int H,
                        int F, int64_t P, void* G, void* U, cudaStream_t s) {
  typedef float T;
  dim3 g1((unsigned)cdiv(F, kSB), (unsigned)(P / kSB));
  MOE_TRACED("simt_gate_up_recompute", s, (gemm_rows_simt_kernel<T, SIMT_SWIGLU><<<g1, 256, 0, s>>>(
      (const T*)x_perm, nullptr, H, (const T*)W1, (const T*)W3, (int64_t)H * F, F, 1, pb, E, H, F,
      nullptr, (T*)G, (T*)U, F, nullptr, nullptr)));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe

// Internal launch functions behind the C ABI (all asynchronous on `s`).
#pragma once

#include "common.cuh"

namespace moe {

// route.cu - warp-per-token router (small E)
bool route_simt_supported(int H, int E, int K, int elem_bytes);
moe_status route_simt(const void* x, const void* W_r, int N, int H, int E, int K, moe_dtype dt,
                      float* logits, float* probs, int32_t* top, float* w, cudaStream_t s);

// route_umma.cu - tensor-core router (bf16, 16 <= E <= 256, E % 16 == 0)
bool route_umma_supported(int N, int H, int E, int K);
size_t route_umma_scratch(int H, int E);
moe_status route_umma(const void* x, const void* W_r, int N, int H, int E, int K, float* logits,
                      float* probs, int32_t* top, float* w, void* scratch, int* status,
                      cudaStream_t s);

// meta.cu
size_t meta_workspace_bytes(int64_t NK, int E);
moe_status dispatch_meta(const int32_t* top, int64_t NK, int E, int32_t* indices, int32_t* bin_ids,
                         int32_t* bins, int32_t* padded_bins, int32_t* pos, void* scratch,
                         int* status, cudaStream_t s, int capacity = 0, int32_t* routed_bins = nullptr);

// permute.cu
moe_status permute_rows(const void* x, const int32_t* pos, const int32_t* bins, const int32_t* pb,
                        int N, int H, int E, int K, moe_dtype dt, void* x_perm, cudaStream_t s);
// dx[t] = (sum_k dx_perm[pos[t, k]], in increasing k) + dx[t], in place
moe_status unpermute_add_rows(const void* dx_perm, const int32_t* pos, int N, int H, int K, moe_dtype dt,
                              void* dx, cudaStream_t s);
moe_status combine_rows(const void* out, const float* w, const int32_t* pos, int N, int K, int H,
                        moe_dtype dt, void* y, cudaStream_t s);
moe_status combine_bwd_rows(const void* dy, const void* out, const float* w, const int32_t* pos,
                            const int32_t* bins, const int32_t* pb, int N, int K, int H, int E,
                            moe_dtype dt, float* dw, float* dlogit, void* d_out, cudaStream_t s);
moe_status transpose_matrix(const void* in, int R, int C, moe_dtype dt, void* outT, cudaStream_t s,
                            int C_pad = 0);
size_t unpermute_router_bwd_scratch(int H, int E, int64_t P);
moe_status unpermute_router_bwd(const void* dx_perm, const float* dlogit, const void* x,
                                const void* W_r, const int32_t* top, const int32_t* pos,
                                const int32_t* indices, const int32_t* bins, const int32_t* padded_bins,
                                int N, int H, int E, int K, int64_t P, moe_dtype dt, void* dx,
                                void* dWr, void* scratch, cudaStream_t s);

// aux.cu - load-balancing loss and the dense router backward it needs
size_t aux_loss_scratch(int N, int E);
size_t dense_router_bwd_scratch(int N, int H, int E);
// routed_bins: inclusive cumsum of the assignments routed to each expert,
// before any capacity drop (equal to bins when dropless).
moe_status aux_loss_fwd(const float* probs, const int32_t* routed_bins, int N, int K, int E, float alpha,
                        float* loss, float* P, void* scratch, cudaStream_t s);
// probs and routed_bins are read only when aux_alpha != 0 and probs != NULL.
moe_status dense_router_bwd(const void* dx_perm, const float* dlogit, const void* x, const void* W_r,
                            const int32_t* top, const int32_t* pos, const int32_t* routed_bins,
                            const float* probs, int N, int H, int E, int K, moe_dtype dt, float aux_alpha,
                            float aux_grad, void* dx, void* dWr, void* scratch, int* status, cudaStream_t s);

// gemm_simt.cu - fp32 grouped GEMMs
moe_status grouped_swiglu_simt(const void* x_perm, const void* W1, const void* W3, const void* W2,
                               const int32_t* pb, int E, int H, int F, int64_t P, moe_dtype dt,
                               void* act, void* out, void* gate_up, cudaStream_t s);
moe_status grouped_swiglu_bwd_simt(const void* d_out, const void* x_perm, const void* act,
                                   const void* gate_up, const void* W1, const void* W3,
                                   const void* W2, const int32_t* pb, int E, int H, int F, int64_t P,
                                   moe_dtype dt, void* d_gate_up, void* dW1, void* dW3, void* dW2,
                                   void* dx_perm, cudaStream_t s);

moe_status gate_up_simt(const void* x_perm, const void* W1, const void* W3, const int32_t* pb, int E, int H,
                        int F, int64_t P, void* G, void* U, cudaStream_t s);

// gemm_umma.cu - bf16 tcgen05 grouped GEMMs
//
// Row gather in place of x_perm: the GEMMs that read the permuted tokens
// (GEMM1 and the dW1/dW3 weight gradient) can fetch padded row r of expert e
// straight from x as token indices[bins[e-1] + r - padded_bins[e-1]] / K
// (pad rows read zeros), so the permuted copy is never written.
struct RowGather {
  const void* x;            // [N, H] tokens
  const int32_t* indices;   // sorted flat assignment ids (dispatch metadata)
  const int32_t* bins;      // inclusive cumsum of per-expert (kept) counts
  int N;
  int K;
};
moe_status gemm1_umma(const void* x_perm, const void* W1, const void* W3, const int32_t* pb, int E, int H,
                      int F, int64_t P, void* act, void* G, void* U, int* status, cudaStream_t s,
                      const char* name, const RowGather* ga = nullptr);
bool umma_shape_supported(int H, int F);
moe_status grouped_swiglu_umma(const void* x_perm, const void* W1, const void* W3, const void* W2,
                               const int32_t* pb, int E, int H, int F, int64_t P, void* act,
                               void* out, void* gate_up, int* status, cudaStream_t s,
                               const RowGather* ga = nullptr);
// Dense router backward (bf16, E % 64 == 0, H % 256 == 0): dx = D * W_r^T
// (then unpermute_add_rows), and per-token-chunk fp32 partials of x^T * D
// (then an in-order reduction over the chunks); D [N, E] bf16.
bool router_bwd_umma_supported(int H, int E);
moe_status router_dx_umma(const void* D, const void* W_r, int N, int H, int E, void* dx, int* status,
                          cudaStream_t s);
moe_status router_wgrad_umma(const void* x, const void* D, const int32_t* chunk_end, int n_chunks, int N,
                             int H, int E, float* part, int* status, cudaStream_t s);
moe_status grouped_swiglu_bwd_umma(const void* d_out, const void* x_perm, const void* act,
                                   const void* gate_up, const void* W1, const void* W3,
                                   const void* W2, const int32_t* pb, int E, int H, int F, int64_t P,
                                   void* d_gate_up, void* dW1, void* dW3, void* dW2, void* dx_perm,
                                   int* status, cudaStream_t s, const RowGather* ga = nullptr);

}  // namespace moe

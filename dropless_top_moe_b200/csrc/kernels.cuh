// Internal launch functions behind the C ABI (all asynchronous on `s`).
#pragma once

#include "common.cuh"

namespace moe {

// route.cu - warp-per-token router (small E)
bool route_simt_supported(int H, int E, int K, int elem_bytes);
moe_status route_simt(const void* x, const void* W_r, int N, int H, int E, int K, moe_dtype dt,
                      float* logits, float* probs, int32_t* top, float* w, cudaStream_t s);

// router.cu - router weight gradient on tensor cores: dW_r [H, E] = x^T D
// for bf16 with E % 8 == 0, E <= 256 and H % 128 == 0; D [N, E] bf16.
bool router_wgrad_tc_supported(int H, int E);
size_t router_wgrad_tc_scratch(int N, int H, int E);
moe_status router_wgrad_tc(const void* x, const void* Dh, int N, int H, int E, void* dWr, void* scratch,
                           int* status, cudaStream_t s);

// router.cu - tensor-core router (bf16, E <= 256, H % 64 == 0).  With
// chunk_counts it also writes the per-chunk expert counts of the dispatch
// metadata ([ceil(N / T)][E], T = route_chunk_tokens tokens per chunk, see
// dispatch_meta).
bool route_umma_supported(int N, int H, int E, int K);
int route_chunk_tokens(int N, int H, int E, int K);
size_t route_umma_scratch(int N, int H, int E, int K);
moe_status route_umma(const void* x, const void* W_r, int N, int H, int E, int K, float* logits,
                      float* probs, int32_t* top, float* w, void* scratch, int* status,
                      cudaStream_t s, int32_t* chunk_counts = nullptr);

// meta.cu - metadata over chunks of T tokens (T a power of two <= 128).
// Scratch: per-chunk expert counts [meta_chunks(N, T)][E] (which the bf16
// router can fill with its own chunking: counts_ready), then 2*E ints.
int64_t meta_chunks(int64_t N, int T = 128);
size_t meta_workspace_bytes(int64_t N, int E, int T = 128);
moe_status dispatch_meta(const int32_t* top, int64_t N, int K, int E, int32_t* indices, int32_t* bin_ids,
                         int32_t* bins, int32_t* padded_bins, int32_t* pos, void* scratch, int* status,
                         cudaStream_t s, int capacity = 0, int32_t* routed_bins = nullptr,
                         bool counts_ready = false, int T = 128);

// permute.cu
moe_status permute_rows(const void* x, const int32_t* pos, const int32_t* bins, const int32_t* pb,
                        int N, int H, int E, int K, moe_dtype dt, void* x_perm, cudaStream_t s);
// dx[t] = (sum_k dx_perm[pos[t, k]], in increasing k) + dx[t], in place
moe_status unpermute_add_rows(const void* dx_perm, const int32_t* pos, int N, int H, int K, moe_dtype dt,
                              void* dx, cudaStream_t s);
moe_status combine_rows(const void* out, const float* w, const int32_t* pos, int N, int K, int H,
                        moe_dtype dt, void* y, cudaStream_t s);
// With top and Dh (bf16 only), also D[t, e] = dlogit[t, k] at e = top[t, k]
// and 0 at the other experts, as bf16 [N, E] (the router weight gradient's
// operand).
moe_status combine_bwd_rows(const void* dy, const void* out, const float* w, const int32_t* pos,
                            const int32_t* bins, const int32_t* pb, int N, int K, int H, int E,
                            moe_dtype dt, float* dw, float* dlogit, void* d_out, cudaStream_t s,
                            const int32_t* top = nullptr, void* Dh = nullptr);
// status != NULL: the same launch checks the layer forward's recorded flags
// (status[1]) against `expect` and sets MOE_DEVERR_MODE on a mismatch.
moe_status transpose_matrix(const void* in, int R, int C, moe_dtype dt, void* outT, cudaStream_t s,
                            int C_pad = 0, int* status = nullptr, int expect = 0);
size_t unpermute_router_bwd_scratch(int N, int H, int E, int64_t P);
// W_r^T sits at its start (the layer backward makes it in its first launch:
// wrt_ready); where, inside that scratch, the bf16 D [N, E] of the
// tensor-core router weight gradient lives (combine_bwd_rows can write it
// there: dh_ready).
void* unpermute_router_bwd_dh(void* scratch, int N, int H, int E, int64_t P);
moe_status unpermute_router_bwd(const void* dx_perm, const float* dlogit, const void* x,
                                const void* W_r, const int32_t* top, const int32_t* pos,
                                const int32_t* indices, const int32_t* bins, const int32_t* padded_bins,
                                int N, int H, int E, int K, int64_t P, moe_dtype dt, void* dx,
                                void* dWr, void* scratch, int* status, cudaStream_t s, bool dh_ready = false,
                                bool wrt_ready = false);

// aux.cu - load-balancing loss and the dense router backward it needs
size_t aux_loss_scratch(int N, int E);
size_t dense_router_bwd_scratch(int N, int H, int E);
// routed_bins: inclusive cumsum of the assignments routed to each expert,
// before any capacity drop (equal to bins when dropless).
// D[t, e] = dlogit[t, k] at e = top[t, k], 0 elsewhere, as bf16 [N, E].
moe_status scatter_dlogits(const float* dlogit, const int32_t* top, int N, int E, int K, void* Dh, cudaStream_t s);
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
// (then unpermute_add_rows); D [N, E] bf16.
bool router_bwd_umma_supported(int H, int E);
moe_status router_dx_umma(const void* D, const void* W_r, int N, int H, int E, void* dx, int* status,
                          cudaStream_t s);

moe_status grouped_swiglu_bwd_umma(const void* d_out, const void* x_perm, const void* act,
                                   const void* gate_up, const void* W1, const void* W3,
                                   const void* W2, const int32_t* pb, int E, int H, int F, int64_t P,
                                   void* d_gate_up, void* dW1, void* dW3, void* dW2, void* dx_perm,
                                   int* status, cudaStream_t s, const RowGather* ga = nullptr);

}  // namespace moe

/*
 * moe.h - C ABI of the B200 dropless top-k Mixture-of-Experts layer library
 * (libmoe_b200.so, sm_100a).
 *
 * The layer (one device, forward and backward), after the pages describing it:
 *   router      logits = x W_r, probs = softmax(logits), keep the K largest,
 *               renormalise the kept values to sum to one
 *               ("MoE computation principle and execution", sec. 2.1-2.2)
 *   metadata    sort assignments by expert, histogram, cumsum, round each
 *               expert's count up to 128 rows, cumsum
 *               ("MegaBlocks - architecture", sec. 2.1 and 2.3)
 *   permute     gather token rows into expert order, zero-padded groups
 *               (MegaBlocks sec. 2.1, padded_gather)
 *   experts     SwiGLU per expert: A = silu(X W1_e) * (X W3_e), O = A W2_e
 *               ("LLaMA MoE tutorial", sec. 2.1; icman sec. 2.3), as grouped
 *               GEMMs over the padded groups (MegaBlocks sec. 2.1, grouped path)
 *   combine     y_t = sum_k w_{t,k} O[pos(t,k)]  (icman sec. 2.3; MegaBlocks
 *               sec. 2.1, padded_scatter)
 *   backward    the chain rule of the above; the gather/scatter pair swap
 *               roles (MegaBlocks sec. 4) and the router receives gradient
 *               through the kept softmax weights only (icman sec. 2.2).
 *
 * Conventions for every entry point
 *   - Every pointer argument is a DEVICE pointer allocated by the caller,
 *     unless stated otherwise; the library never allocates, frees or
 *     synchronises (except moe_get_device_status, which must return a value).
 *   - Matrices are dense row-major.  x[N,H]; W_r[H,E]; W1, W3 [E,H,F];
 *     W2 [E,F,H]; y, dy, dx [N,H]; top_experts, weights [N,K]; flat assignment
 *     id i = t*K + k.  Element type: MOE_F32 -> float, MOE_BF16 -> bfloat16
 *     for x, W_r, W1, W3, W2, y and the activations; routing weights,
 *     logits and probabilities are always float32, ids and offsets int32.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *   - The return value reports host-detectable errors only (shapes, dtype,
 *     alignment, workspace size).  Errors found on the device (an expert id
 *     outside [0,E), a padded-row count above the buffer, a bounded wait that
 *     gave up, a layer backward whose flags differ from the forward's) are
 *     OR-ed into the 32-bit status word at the start of the workspace; read
 *     it with moe_get_device_status.  Kernels never trap.
 *   - Outputs are overwritten, never accumulated into.
 *   - Results are bitwise identical from run to run for identical inputs:
 *     no floating-point atomics, every reduction has a fixed order.
 *   - Pointers must be 16-byte aligned.  BF16 layers need H and F multiples
 *     of 128 and E <= 256; F32 layers need H multiple of 4 (tensor cores are
 *     not used for F32, so F32 results keep full single precision).
 *   - Rows of padded buffers at or beyond padded_bins[E-1] are never read
 *     and are left unwritten.
 */
#ifndef DROPLESS_TOP_MOE_B200_MOE_H
#define DROPLESS_TOP_MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, K > E, misalignment */
  MOE_ERR_UNSUPPORTED = 2,   /* valid shape outside what the kernels implement */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  MOE_ERR_CUDA = 4           /* a CUDA runtime call failed (launch error etc.) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Bits of the device status word (first 4 bytes of every workspace; the
 * layer calls keep a record of the forward's flags in the next 4). */
#define MOE_DEVERR_EXPERT_ID 0x1   /* a top_experts entry was outside [0,E) */
#define MOE_DEVERR_TIMEOUT 0x2     /* a bounded pipeline wait gave up */
#define MOE_DEVERR_ROWS 0x4        /* padded rows exceeded the buffer's rows */
#define MOE_DEVERR_MODE 0x8        /* moe_layer_bwd's training flags, aux loss (on/off) or token
                                      dropping (on/off) differ from those of the last
                                      moe_layer_fwd on this workspace: its outputs are
                                      meaningless */

/* The caller's cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

/* Rows per expert group tile: each expert's rows are padded to a multiple of
 * this (MegaBlocks sec. 2.1 rounds up to 128).  Returns 128. */
int32_t moe_tile_rows(void);

/* Static upper bound on padded rows for N tokens, E experts, top-K:
 * round_up(N*K + E*127, 128).  Buffers of this many rows never overflow,
 * whatever the routing; no host synchronisation is needed to size them. */
int64_t moe_padded_rows_max(int32_t N, int32_t E, int32_t K);

/* Workspace bytes for each entry point.  A workspace is caller-owned device
 * memory; its first 256 bytes hold the device status word and must be
 * zeroed once (moe_workspace_init) before first use.  The router's and the
 * layer's sizes depend on the whole shape and are 0 for a shape the call
 * would reject. */
size_t moe_route_workspace_size(int32_t N, int32_t H, int32_t E, int32_t K, moe_dtype dt);
size_t moe_dispatch_meta_workspace_size(int32_t N, int32_t K, int32_t E);
size_t moe_grouped_workspace_size(void);
/* Whole layer.  training: 0 = forward only; 1 = keep what the backward pass
 * reads, including the SwiGLU gate and up projections G, U; 2 = memory-
 * optimised training: G and U are not kept (2*P*F elements less) and the
 * backward recomputes them (+4*N*K*H*F FLOPs).  The same workspace must then
 * be passed to moe_layer_bwd unchanged.  Returns 0 for a shape or flag the
 * layer calls would reject. */
size_t moe_workspace_size(int32_t N, int32_t H, int32_t E, int32_t K, int32_t F,
                          moe_dtype dt, int32_t training);

/* Flag OR-ed into `training` (the same value for moe_workspace_size,
 * moe_layer_fwd and moe_layer_bwd), bf16 only: GEMM1 and the dW1/dW3
 * contraction fetch their rows straight from x with TMA row gathers
 * (padded row r of expert e = token indices[bins[e-1] + r - padded_bins[e-1]]
 * / K, pad rows zero) instead of a permuted copy, so the permute step and its
 * P*H-element buffer disappear ("MegaBlocks - architecture", sec. 2.1: the
 * permute only feeds the grouped GEMM).  Results are bit-identical to the
 * default path.  The gathers move four 128-byte rows per TMA instruction, and
 * on B200 their issue rate holds GEMM1 to roughly a third of its default
 * speed, so this is a memory option, off by default.  With fp32 the
 * workspace size is 0 and the layer calls return MOE_ERR_INVALID_ARG. */
#define MOE_LAYER_GATHER_ROWS 4

/* Zero the device status word of `ws` (async on `stream`). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Copy the device status word to *status_out (host pointer).  Synchronises
 * `stream`.  0 means no device-side error since the last moe_workspace_init. */
moe_status moe_get_device_status(const void* ws, int32_t* status_out, moe_stream_t stream);

/* Router: logits = x W_r (fp32 accumulation), probs = softmax(logits),
 * top_experts[t, 0..K-1] = the K largest, in descending order, equal values
 * resolved to the lower expert id; weights = kept probs / their sum.
 * (icman sec. 2.1-2.2.)  Selection is made on the fp32 logits, which orders
 * experts exactly as the probabilities do (softmax is monotone).
 *   x [N,H], W_r [H,E] (dt); logits, probs [N,E] float32 (each may be NULL);
 *   top_experts [N,K] int32; weights [N,K] float32.
 *   Needs 1 <= K <= E <= 256. */
moe_status moe_route(const void* x, const void* W_r, int32_t N, int32_t H, int32_t E, int32_t K,
                     moe_dtype dt, float* logits, float* probs, int32_t* top_experts,
                     float* weights, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Dispatch metadata (MegaBlocks sec. 2.1/2.3): stable sort of the N*K flat
 * assignment ids by expert, histogram, inclusive cumsums.
 *   capacity: 0 = dropless.  > 0 gives the token-dropping variant (icman
 *   sec. 3.4): each expert keeps its first `capacity` assignments in flat-id
 *   order and drops the rest; counts, bins, padded_bins and indices then
 *   cover kept assignments only (indices holds bins[E-1] entries) and dropped
 *   assignments get pos -1.
 *   top_experts [N*K] int32 in [0,E).
 *   indices [N*K]  flat ids in expert order (stable: increasing id within an expert)
 *   bin_ids [N*K]  expert of indices[j]
 *   bins [E]       inclusive cumsum of the per-expert counts
 *   padded_bins [E] inclusive cumsum of counts rounded up to 128
 *   pos [N*K]      padded row of assignment i: start of its expert's padded
 *                  group + its rank among that expert's assignments
 * Any output pointer except padded_bins and pos may be NULL.  Ids outside
 * [0,E) set MOE_DEVERR_EXPERT_ID; their pos is -1 and they are skipped. */
moe_status moe_dispatch_meta(const int32_t* top_experts, int32_t N, int32_t K, int32_t E,
                             int32_t capacity, int32_t* indices, int32_t* bin_ids, int32_t* bins,
                             int32_t* padded_bins, int32_t* pos, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/* Dispatch metadata for callers that cannot allocate device memory (dropless,
 * capacity 0).  The
 * pages have no counterpart to this entry point.  Some callers cannot call
 * cudaMalloc: code embedded in another runtime that owns all device memory
 * and gives its plugins no allocator, or a latency-critical path where an
 * allocation (which may synchronise the device) is not allowed.  Same
 * outputs as moe_dispatch_meta, but the scratch lives in a fixed device
 * array inside the library (about 1 MB per device that loads it, held until
 * exit) instead of a workspace; the caller still passes every input and
 * output.
 *   Limit: ceil(N / 128) * E <= 262144 (with E = 256: N <= 131072 tokens);
 *   larger sizes return MOE_ERR_WORKSPACE before any device work.
 *   status: NULL, or a device int32 the caller zeroed; MOE_DEVERR_* bits are
 *   OR-ed into it.
 *   Every call looks up the array's device address (cudaGetSymbolAddress)
 *   on the current device, so a device reset or a new context needs no
 *   re-initialisation.  The first call on a device may load the library's
 *   device code there: make that first call before any stream capture.  All
 *   calls on a device share the one array,
 *   which keeps the last call's contents: calls that overlap on the GPU (on
 *   different streams without ordering) race and give wrong results.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
moe_status moe_dispatch_meta_noalloc(const int32_t* top_experts, int32_t N, int32_t K, int32_t E,
                                     int32_t* indices, int32_t* bin_ids, int32_t* bins,
                                     int32_t* padded_bins, int32_t* pos, int32_t* status,
                                     moe_stream_t stream);

/* Padded gather (MegaBlocks sec. 2.1): x_perm[pos[t*K+k], :] = x[t, :]; the
 * pad rows of every expert group (count..round_up(count,128)) are zeroed.
 *   x [N,H]; x_perm [P,H] with P >= padded_bins[E-1] (dt); bins, padded_bins [E]. */
moe_status moe_permute(const void* x, const int32_t* pos, const int32_t* bins,
                       const int32_t* padded_bins, int32_t N, int32_t H, int32_t E, int32_t K,
                       moe_dtype dt, void* x_perm, moe_stream_t stream);

/* Grouped SwiGLU experts over padded groups: rows [padded_bins[e-1],
 * padded_bins[e]) use expert e:
 *   G = X W1_e, U = X W3_e, act = silu(G) * U, out = act W2_e
 * (LLaMA MoE tutorial sec. 2.1; icman sec. 2.3).  fp32 accumulation; act and
 * out are rounded once to dt.  P = rows of x_perm/act/out (multiple of 128);
 * groups reaching past row P are computed only up to P, and the tensor-core
 * (bf16) path then sets MOE_DEVERR_ROWS in the workspace's status word. 
 *   x_perm [P,H]; W1, W3 [E,H,F]; W2 [E,F,H]; act [P,F]; out [P,H];
 *   gate_up: NULL, or [2,P,F] receiving G then U (dt) for the backward pass. */
moe_status moe_grouped_swiglu(const void* x_perm, const void* W1, const void* W3, const void* W2,
                              const int32_t* padded_bins, int32_t E, int32_t H, int32_t F, int64_t P,
                              moe_dtype dt, void* act, void* out, void* gate_up,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/* Weighted combine (icman sec. 2.3): y[t] = sum_{k=0..K-1} weights[t,k] *
 * out[pos[t*K+k]], summed in increasing k in fp32, rounded once.
 *   out [P,H]; weights [N,K]; y [N,H]. */
moe_status moe_combine(const void* out, const float* weights, const int32_t* pos,
                       int32_t N, int32_t K, int32_t H, moe_dtype dt, void* y,
                       moe_stream_t stream);

/* Backward of combine and of the router's renormalised weights
 * (MegaBlocks sec. 4 duality; icman sec. 2.2):
 *   dw[t,k]  = <dy_t, out[pos[t*K+k]]>           (fixed-order fp32 dot)
 *   d_out[pos[t*K+k]] = weights[t,k] * dy_t      (pad rows zeroed)
 *   dlogit[t,k] = weights[t,k] * (dw[t,k] - sum_j weights[t,j] dw[t,j])
 * dlogit is the gradient of the router logit of expert top_experts[t,k]
 * (all other logits get zero).  dw, dlogit [N,K] float32 (dw may be NULL);
 * d_out [P,H] (dt). */
moe_status moe_combine_bwd(const void* dy, const void* out, const float* weights,
                           const int32_t* pos, const int32_t* bins, const int32_t* padded_bins,
                           int32_t N, int32_t K, int32_t H, int32_t E, moe_dtype dt,
                           float* dw, float* dlogit, void* d_out, moe_stream_t stream);

/* Backward of the grouped SwiGLU experts, per padded group e:
 *   dA = d_out W2_e^T;  dG = dA * U * silu'(G);  dU = dA * silu(G)
 *   dW2_e = act^T d_out;  dW1_e = X^T dG;  dW3_e = X^T dU
 *   dx_perm = dG W1_e^T + dU W3_e^T
 * gate_up is the [2,P,F] saved by moe_grouped_swiglu.  Experts with no rows
 * get zero weight gradients.  d_gate_up [2,P,F] is caller scratch.
 *   dW1, dW3 [E,H,F]; dW2 [E,F,H]; dx_perm [P,H] (dt). */
moe_status moe_grouped_swiglu_bwd(const void* d_out, const void* x_perm, const void* act,
                                  const void* gate_up, const void* W1, const void* W3,
                                  const void* W2, const int32_t* padded_bins, int32_t E,
                                  int32_t H, int32_t F, int64_t P, moe_dtype dt,
                                  void* d_gate_up, void* dW1, void* dW3, void* dW2,
                                  void* dx_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Backward of the permute and of the router GEMM:
 *   dx[t] = sum_k dx_perm[pos[t*K+k]] + sum_k dlogit[t,k] * W_r[:, top_experts[t,k]]
 *   dW_r[:, e] = sum over assignments i of expert e, in sorted order, of
 *                dlogit_i * x[token(i)]
 * (sums in fixed order, fp32).  indices/bins/padded_bins from
 * moe_dispatch_meta; P = rows of dx_perm.
 * With aux_alpha == 0 the router terms walk the assignments listed in
 * indices, so every assignment must have been kept (dropless metadata); the
 * token-dropping variant's router gradient comes from moe_layer_bwd.
 * With aux_alpha != 0 the router also receives the gradient of
 * aux_grad * L_aux (see moe_aux_loss): every logit gets
 *   a[t,e] = aux_grad*aux_alpha*E/N * probs[t,e] * (f_e - sum_i f_i probs[t,i]),
 * f_e = count_e / (N*K) with count_e = bins[e] - bins[e-1] taken as the
 * assignments routed to e (see moe_aux_loss), and the router terms use the
 * dense D = a + (dlogit scattered to the experts of every slot):
 *   dx[t] = sum_k dx_perm[pos[t*K+k]] + sum_e D[t,e] W_r[:,e],  dW_r = x^T D
 * (fixed-order fp32 reductions); probs [N,E] float32 is then required.
 * ws: moe_unpermute_router_bwd_workspace_size bytes.
 *   dx [N,H]; dW_r [H,E] (dt). */
size_t moe_unpermute_router_bwd_workspace_size(int32_t N, int32_t H, int32_t E, int64_t P);
moe_status moe_unpermute_router_bwd(const void* dx_perm, const float* dlogit, const void* x,
                                    const void* W_r, const int32_t* top_experts,
                                    const int32_t* pos, const int32_t* indices,
                                    const int32_t* bins, const int32_t* padded_bins,
                                    const float* probs, float aux_alpha, float aux_grad, int32_t N,
                                    int32_t H, int32_t E, int32_t K, int64_t P, moe_dtype dt,
                                    void* dx, void* dW_r, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* Auxiliary load-balancing loss ("MoE computation principle and execution",
 * sec. 4.2): *loss = alpha * E * sum_i f_i * P_i with f_i = count_i / (N*K)
 * and P_i = mean over tokens of probs[:, i].  count_i = bins[i] - bins[i-1]
 * is the number of assignments the router made to expert i: with token
 * dropping, pass the bins of a dropless (capacity 0) dispatch, since the loss
 * counts dropped assignments too (the layer calls do this).  Column sums
 * run over 256-token chunks in increasing order, then over the chunks in
 * order, then a fixed pairwise tree over experts: deterministic.
 *   probs [N,E] float32 (moe_route's probs); bins [E]; loss: device float;
 *   P: NULL or device float [E] receiving P_i.  ws: moe_aux_loss_workspace_size. */
size_t moe_aux_loss_workspace_size(int32_t N, int32_t E);
moe_status moe_aux_loss(const float* probs, const int32_t* bins, int32_t N, int32_t K, int32_t E,
                        float alpha, float* loss, float* P, void* ws, size_t ws_bytes,
                        moe_stream_t stream);

/* Whole layer forward: route -> dispatch_meta -> permute -> grouped SwiGLU
 * -> combine, all on `stream`, no host synchronisation.
 *   y [N,H] (dt); top_experts [N,K]; weights [N,K]; indices [N*K];
 *   bins, padded_bins [E] (all required; with N = 0 the token-sized ones
 *   may be NULL).
 *   capacity: 0 = dropless; > 0 = token-dropping variant (see
 *   moe_dispatch_meta): dropped (token, expert) pairs add nothing to y.
 *   aux_alpha != 0 also computes the load-balancing loss into *aux_loss (a
 *   device float, see moe_aux_loss; with token dropping its f_i still count
 *   every routed assignment) and keeps the router probabilities in the
 *   workspace for the backward pass; aux_alpha = 0 skips both.
 * ws: moe_workspace_size(..., training) bytes; with training != 0 it keeps
 * what moe_layer_bwd reads. */
moe_status moe_layer_fwd(const void* x, const void* W_r, const void* W1, const void* W3,
                         const void* W2, int32_t N, int32_t H, int32_t E, int32_t K, int32_t F,
                         moe_dtype dt, int32_t training, int32_t capacity, float aux_alpha,
                         float* aux_loss, void* y,
                         int32_t* top_experts, float* weights, int32_t* indices, int32_t* bins,
                         int32_t* padded_bins, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Whole layer backward of the forward run last on this workspace (the
 * forward must have run: the backward reads the token positions, the expert
 * outputs and the activations it left there).
 *   training: 1 or 2, the forward's value (with 2, G and U are recomputed
 *   here by the forward's own GEMM kernel, bit-identical).
 *   dy [N,H]; outputs dx [N,H], dW_r [H,E], dW1, dW3 [E,H,F], dW2 [E,F,H],
 *   all dt, overwritten.  top_experts, weights, indices, bins, padded_bins:
 *   the forward's outputs, unchanged.
 *   capacity and aux_alpha must equal the forward's (dropped pairs still pass
 *   gradient to the router through the renormalised weights).  A backward
 *   whose training flags, aux loss on/off or token dropping on/off differ
 *   from the forward's sets MOE_DEVERR_MODE (one 32-thread check kernel,
 *   first on the stream).
 *   aux_grad (used when aux_alpha != 0) = dObjective/dL_aux scales the
 *   load-balancing loss's gradient, which is added to the router's (dense
 *   router backward).
 *   N = 0: the token arrays may be NULL and the weight gradients are zeroed. */
moe_status moe_layer_bwd(const void* dy, const void* x, const void* W_r, const void* W1,
                         const void* W3, const void* W2, const int32_t* top_experts,
                         const float* weights, const int32_t* indices, const int32_t* bins,
                         const int32_t* padded_bins, int32_t N, int32_t H, int32_t E, int32_t K,
                         int32_t F, moe_dtype dt, int32_t training, int32_t capacity, float aux_alpha,
                         float aux_grad, void* dx,
                         void* dW_r, void* dW1, void* dW3, void* dW2, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Local step of a deterministic data-parallel gradient all-reduce (replicas of
 * the layer on several GPUs each hold gradients of their own tokens; a
 * trainer sums them).  shards: [n_ranks, numel] contiguous (dt), one row per
 * rank in rank order, as an all-to-all of equal shards delivers them;
 * out[j] = scale * sum_{r = 0..n_ranks-1} shards[r][j], summed in increasing r
 * in fp32 and rounded once, so every rank gets identical bits.  numel must be
 * a multiple of 8 (bf16) or 4 (fp32). */
moe_status moe_sum_rank_ordered(const void* shards, int32_t n_ranks, int64_t numel, moe_dtype dt,
                                float scale, void* out, moe_stream_t stream);

/* Diagnostics (no counterpart on the pages): one block waits, with the same
 * bounded mbarrier wait every tcgen05 GEMM pipeline stage uses, on a barrier
 * that nothing arrives at; after timeout_ns (1 us .. 1 s) it gives up and
 * sets MOE_DEVERR_TIMEOUT in *status (a device int32, OR-ed in; zero it
 * first).  The kernel then returns normally and the CUDA context stays
 * usable: this is how a stalled pipeline surfaces, as a status bit rather
 * than a hung GPU.  Asynchronous on `stream`; MOE_ERR_INVALID_ARG for a NULL
 * status or a limit out of range. */
moe_status moe_selftest_wait_timeout(int32_t* status, int64_t timeout_ns, moe_stream_t stream);

/* Per-launch timing.  While attached, every kernel launch made by any entry
 * point records events[2*i] on its stream just before launch i and
 * events[2*i+1] just after it, stores a static kernel name in labels[i]
 * (labels may be NULL) and increments *count (host memory), for up to
 * `capacity` launches.  The caller creates the events (cudaEvent_t, timing
 * enabled) and owns every buffer.  Process-wide, not thread-safe. */
moe_status moe_trace_attach(void* const* events, int32_t capacity, const char** labels, int32_t* count);
moe_status moe_trace_detach(void);

#ifdef __cplusplus
}
#endif

#endif /* DROPLESS_TOP_MOE_B200_MOE_H */

// C ABI of the dropless top-k MoE layer: argument validation, workspace
// carving and the fixed launch sequence of the forward and backward passes.
// No entry point allocates, frees or synchronises (moe_get_device_status
// excepted, since it must return a host value).
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"

using namespace moe;

namespace {

inline bool aligned16(const void* p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }
inline size_t elem_bytes(moe_dtype dt) { return dt == MOE_F32 ? 4 : 2; }
inline size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

// Sizes shared by every entry point.
moe_status check_shape(int N, int H, int E, int K, moe_dtype dt) {
  if (dt != MOE_F32 && dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (N < 0 || H <= 0 || E <= 0 || K <= 0 || K > E) return MOE_ERR_INVALID_ARG;
  if ((int64_t)N * K > (int64_t)0x7fffffff - (int64_t)E * kTile) return MOE_ERR_UNSUPPORTED;
  if (E > 256 || K > 32) return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_F32 && H % 4 != 0) return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_BF16 && H % 128 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ffn(int H, int F, moe_dtype dt) {
  if (F <= 0) return MOE_ERR_INVALID_ARG;
  if (dt == MOE_BF16 && !umma_shape_supported(H, F)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int64_t p_max(int N, int E, int K) { return round_up((int64_t)N * K + (int64_t)E * (kTile - 1), kTile); }

// Layer workspace, in order; every region 256-byte aligned.
struct LayerWs {
  int* status;
  void* route_scratch;
  void* meta_scratch;
  int32_t* routed_bins;   // inclusive cumsum of routed counts (before any capacity drop)
  int32_t* pos;
  void* x_perm;
  void* act;
  void* out;
  void* gate_up;     // training only
  void* d_out;       // training only (backward scratch from here on)
  void* d_gate_up;
  void* dx_perm;
  float* dlogit;
  void* ur_scratch;
  float* probs;      // router probabilities (written when the aux loss is on)
  void* aux_scratch;
  void* dense_scratch;   // training only: dense router backward
  size_t total;
};

bool routes_on_tensor_cores(int N, int H, int E, int K, moe_dtype dt) {
  return dt == MOE_BF16 && route_umma_supported(N, H, E, K);
}

size_t route_scratch_bytes(int N, int H, int E, int K, moe_dtype dt) {
  return routes_on_tensor_cores(N, H, E, K, dt) ? route_umma_scratch(N, H, E, K) : 0;
}

// Tokens per dispatch-metadata chunk in the layer: the tensor-core router
// counts each of its chunks' expert ids; otherwise the metadata counts 128.
int layer_meta_chunk(int N, int H, int E, int K, moe_dtype dt) {
  return routes_on_tensor_cores(N, H, E, K, dt) ? route_chunk_tokens(N, H, E, K) : 128;
}

// training: mode 0 / 1 / 2 in the low bits, MOE_LAYER_GATHER_ROWS (bf16 only) on top
bool layer_flags_ok(int32_t training, moe_dtype dt) {
  if ((training & ~(3 | MOE_LAYER_GATHER_ROWS)) != 0 || (training & 3) == 3) return false;
  return !(training & MOE_LAYER_GATHER_ROWS) || dt == MOE_BF16;
}

// Word 1 of the status region records the layout-deciding flags of the last
// layer forward on the workspace (mode, row gather, aux loss on, token
// dropping on) as one non-zero byte repeated four times.  The backward reads
// buffers the forward wrote at offsets these flags decide, so it compares the
// record with its own flags first; moe_workspace_init clears the record.
int layer_stamp_byte(int32_t flags, float aux_alpha, int32_t capacity) {
  return 1 + (flags & 7) + (aux_alpha != 0.0f ? 8 : 0) + (capacity > 0 ? 16 : 0);
}

__global__ void layer_stamp_check_kernel(int* status, int expect) {
  if (threadIdx.x == 0 && status[1] != expect) atomicOr(status, MOE_DEVERR_MODE);
}

LayerWs carve(void* base, int N, int H, int E, int K, int F, moe_dtype dt, int flags) {
  const int training = flags & 3;
  const bool gather = (flags & MOE_LAYER_GATHER_ROWS) != 0;
  LayerWs w;
  memset(&w, 0, sizeof(w));
  char* p = (char*)base;
  size_t off = 0;
  const int64_t P = p_max(N, E, K), NK = (int64_t)N * K;
  const size_t eb = elem_bytes(dt);
  auto take = [&](size_t bytes) -> void* {
    void* r = p ? (void*)(p + off) : nullptr;
    off += al256(bytes);
    return r;
  };
  w.status = (int*)take(kStatusBytes);
  w.route_scratch = take(route_scratch_bytes(N, H, E, K, dt));
  w.meta_scratch = take(meta_workspace_bytes(N, E, layer_meta_chunk(N, H, E, K, dt)));
  w.routed_bins = (int32_t*)take((size_t)E * 4);
  w.pos = (int32_t*)take(NK * 4);
  w.probs = (float*)take((size_t)N * E * 4);
  w.aux_scratch = take(aux_loss_scratch(N, E));
  w.x_perm = gather ? nullptr : take(P * H * eb);   // gathered rows need no permuted copy
  w.act = take(P * F * eb);
  w.out = take(P * H * eb);
  if (training) {
    // training == 2 (memory-optimised) keeps no G, U between the passes
    w.gate_up = training == 1 ? take(2 * P * F * eb) : nullptr;
    w.d_out = take(P * H * eb);
    w.d_gate_up = take(2 * P * F * eb);
    w.dx_perm = take(P * H * eb);
    w.dlogit = (float*)take(NK * 4);
    w.ur_scratch = take(unpermute_router_bwd_scratch(N, H, E, P));
    w.dense_scratch = take(dense_router_bwd_scratch(N, H, E));
  }
  w.total = off;
  return w;
}

// chunk_counts: with the tensor-core router, also the per-128-token expert
// counts the dispatch metadata starts from (NULL: not wanted).
moe_status route_any(const void* x, const void* W_r, int N, int H, int E, int K, moe_dtype dt,
                     float* logits, float* probs, int32_t* top, float* w, void* scratch, int* status,
                     cudaStream_t s, int32_t* chunk_counts = nullptr) {
  if (N == 0) return MOE_OK;
  if (routes_on_tensor_cores(N, H, E, K, dt))
    return route_umma(x, W_r, N, H, E, K, logits, probs, top, w, scratch, status, s, chunk_counts);
  if (route_simt_supported(H, E, K, (int)elem_bytes(dt)))
    return route_simt(x, W_r, N, H, E, K, dt, logits, probs, top, w, s);
  return MOE_ERR_UNSUPPORTED;
}

moe_status swiglu_any(const void* x_perm, const void* W1, const void* W3, const void* W2,
                      const int32_t* pb, int E, int H, int F, int64_t P, moe_dtype dt, void* act,
                      void* out, void* gate_up, int* status, cudaStream_t s, const RowGather* ga = nullptr) {
  if (dt == MOE_F32)
    return grouped_swiglu_simt(x_perm, W1, W3, W2, pb, E, H, F, P, dt, act, out, gate_up, s);
  return grouped_swiglu_umma(x_perm, W1, W3, W2, pb, E, H, F, P, act, out, gate_up, status, s, ga);
}

moe_status swiglu_bwd_any(const void* d_out, const void* x_perm, const void* act, const void* gate_up,
                          const void* W1, const void* W3, const void* W2, const int32_t* pb, int E,
                          int H, int F, int64_t P, moe_dtype dt, void* d_gate_up, void* dW1,
                          void* dW3, void* dW2, void* dx_perm, int* status, cudaStream_t s,
                          const RowGather* ga = nullptr) {
  if (dt == MOE_F32)
    return grouped_swiglu_bwd_simt(d_out, x_perm, act, gate_up, W1, W3, W2, pb, E, H, F, P, dt,
                                   d_gate_up, dW1, dW3, dW2, dx_perm, s);
  return grouped_swiglu_bwd_umma(d_out, x_perm, act, gate_up, W1, W3, W2, pb, E, H, F, P, d_gate_up,
                                 dW1, dW3, dW2, dx_perm, status, s, ga);
}

}  // namespace

#define MOE_TRY(expr)                      \
  do {                                     \
    moe_status _st = (expr);               \
    if (_st != MOE_OK) return _st;         \
  } while (0)

extern "C" {

int32_t moe_tile_rows(void) { return kTile; }

int64_t moe_padded_rows_max(int32_t N, int32_t E, int32_t K) {
  if (N < 0 || E <= 0 || K <= 0) return 0;
  return p_max(N, E, K);
}

size_t moe_route_workspace_size(int32_t N, int32_t H, int32_t E, int32_t K, moe_dtype dt) {
  if (check_shape(N, H, E, K, dt) != MOE_OK) return 0;
  return al256(kStatusBytes) + al256(route_scratch_bytes(N, H, E, K, dt));
}

size_t moe_dispatch_meta_workspace_size(int32_t N, int32_t K, int32_t E) {
  (void)K;
  return al256(kStatusBytes) + al256(meta_workspace_bytes(N, E));
}

size_t moe_grouped_workspace_size(void) { return al256(kStatusBytes); }

size_t moe_unpermute_router_bwd_workspace_size(int32_t N, int32_t H, int32_t E, int64_t P) {
  return al256(kStatusBytes) + al256(unpermute_router_bwd_scratch(N, H, E, P)) +
         al256(dense_router_bwd_scratch(N, H, E));
}

size_t moe_aux_loss_workspace_size(int32_t N, int32_t E) {
  return al256(kStatusBytes) + al256(aux_loss_scratch(N, E));
}

size_t moe_workspace_size(int32_t N, int32_t H, int32_t E, int32_t K, int32_t F, moe_dtype dt,
                          int32_t training) {
  if (check_shape(N, H, E, K, dt) != MOE_OK || check_ffn(H, F, dt) != MOE_OK || !layer_flags_ok(training, dt))
    return 0;
  return carve(nullptr, N, H, E, K, F, dt, training).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || ws_bytes < (size_t)kStatusBytes) return MOE_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_get_device_status(const void* ws, int32_t* status_out, moe_stream_t stream) {
  if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = v;
  return MOE_OK;
}

moe_status moe_route(const void* x, const void* W_r, int32_t N, int32_t H, int32_t E, int32_t K,
                     moe_dtype dt, float* logits, float* probs, int32_t* top_experts, float* weights,
                     void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  if (N > 0 && (!x || !W_r || !top_experts || !weights)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_route_workspace_size(N, H, E, K, dt)) return MOE_ERR_WORKSPACE;
  char* base = (char*)ws;
  return route_any(x, W_r, N, H, E, K, dt, logits, probs, top_experts, weights,
                   base + al256(kStatusBytes), (int*)ws, (cudaStream_t)stream);
}

moe_status moe_dispatch_meta(const int32_t* top_experts, int32_t N, int32_t K, int32_t E,
                             int32_t capacity, int32_t* indices, int32_t* bin_ids, int32_t* bins,
                             int32_t* padded_bins, int32_t* pos, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  if (N < 0 || K <= 0 || E <= 0 || K > E || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  if (!padded_bins || (N > 0 && (!top_experts || !pos))) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_dispatch_meta_workspace_size(N, K, E)) return MOE_ERR_WORKSPACE;
  char* base = (char*)ws;
  return dispatch_meta(top_experts, N, K, E, indices, bin_ids, bins, padded_bins, pos, base + al256(kStatusBytes),
                       (int*)ws, (cudaStream_t)stream, capacity);
}

moe_status moe_permute(const void* x, const int32_t* pos, const int32_t* bins, const int32_t* padded_bins,
                       int32_t N, int32_t H, int32_t E, int32_t K, moe_dtype dt, void* x_perm,
                       moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  if (!bins || !padded_bins || !x_perm || (N > 0 && (!x || !pos))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  return permute_rows(x, pos, bins, padded_bins, N, H, E, K, dt, x_perm, (cudaStream_t)stream);
}

moe_status moe_grouped_swiglu(const void* x_perm, const void* W1, const void* W3, const void* W2,
                              const int32_t* padded_bins, int32_t E, int32_t H, int32_t F, int64_t P,
                              moe_dtype dt, void* act, void* out, void* gate_up, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(0, H, E, 1, dt));
  MOE_TRY(check_ffn(H, F, dt));
  if (P < 0 || P % kTile != 0) return MOE_ERR_INVALID_ARG;
  if (!x_perm || !W1 || !W3 || !W2 || !padded_bins || !act || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(act) ||
      !aligned16(out) || !aligned16(gate_up))
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_grouped_workspace_size()) return MOE_ERR_WORKSPACE;
  if (P == 0) return MOE_OK;
  return swiglu_any(x_perm, W1, W3, W2, padded_bins, E, H, F, P, dt, act, out, gate_up, (int*)ws,
                    (cudaStream_t)stream);
}

moe_status moe_combine(const void* out, const float* weights, const int32_t* pos, int32_t N, int32_t K,
                       int32_t H, moe_dtype dt, void* y, moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, K, K, dt));
  if (N == 0) return MOE_OK;
  if (!out || !weights || !pos || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return combine_rows(out, weights, pos, N, K, H, dt, y, (cudaStream_t)stream);
}

moe_status moe_combine_bwd(const void* dy, const void* out, const float* weights, const int32_t* pos,
                           const int32_t* bins, const int32_t* padded_bins, int32_t N, int32_t K,
                           int32_t H, int32_t E, moe_dtype dt, float* dw, float* dlogit, void* d_out,
                           moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  if (!bins || !padded_bins || !d_out || (N > 0 && (!dy || !out || !weights || !pos || !dlogit)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(out) || !aligned16(d_out)) return MOE_ERR_INVALID_ARG;
  return combine_bwd_rows(dy, out, weights, pos, bins, padded_bins, N, K, H, E, dt, dw, dlogit, d_out,
                          (cudaStream_t)stream);
}

moe_status moe_grouped_swiglu_bwd(const void* d_out, const void* x_perm, const void* act,
                                  const void* gate_up, const void* W1, const void* W3, const void* W2,
                                  const int32_t* padded_bins, int32_t E, int32_t H, int32_t F, int64_t P,
                                  moe_dtype dt, void* d_gate_up, void* dW1, void* dW3, void* dW2,
                                  void* dx_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(0, H, E, 1, dt));
  MOE_TRY(check_ffn(H, F, dt));
  if (P < 0 || P % kTile != 0) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {d_out, x_perm, act, gate_up, W1, W3, W2, d_gate_up, dW1, dW3, dW2, dx_perm};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (!padded_bins) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_grouped_workspace_size()) return MOE_ERR_WORKSPACE;
  return swiglu_bwd_any(d_out, x_perm, act, gate_up, W1, W3, W2, padded_bins, E, H, F, P, dt,
                        d_gate_up, dW1, dW3, dW2, dx_perm, (int*)ws, (cudaStream_t)stream);
}

moe_status moe_unpermute_router_bwd(const void* dx_perm, const float* dlogit, const void* x,
                                    const void* W_r, const int32_t* top_experts, const int32_t* pos,
                                    const int32_t* indices, const int32_t* bins,
                                    const int32_t* padded_bins, const float* probs, float aux_alpha,
                                    float aux_grad, int32_t N, int32_t H, int32_t E, int32_t K, int64_t P,
                                    moe_dtype dt, void* dx, void* dW_r, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  if (P < 0 || P % kTile != 0) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {dx_perm, dlogit, x, W_r, top_experts, pos, indices, bins, padded_bins, dx, dW_r};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  const bool aux = aux_alpha != 0.0f && N > 0;
  if (aux && !probs) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_unpermute_router_bwd_workspace_size(N, H, E, P)) return MOE_ERR_WORKSPACE;
  char* scratch = (char*)ws + al256(kStatusBytes);
  if (aux)
    return dense_router_bwd(dx_perm, dlogit, x, W_r, top_experts, pos, bins, probs, N, H, E, K, dt, aux_alpha,
                            aux_grad, dx, dW_r, scratch + al256(unpermute_router_bwd_scratch(N, H, E, P)),
                            (int*)ws, (cudaStream_t)stream);
  return unpermute_router_bwd(dx_perm, dlogit, x, W_r, top_experts, pos, indices, bins, padded_bins, N,
                              H, E, K, P, dt, dx, dW_r, scratch, (int*)ws, (cudaStream_t)stream);
}

moe_status moe_aux_loss(const float* probs, const int32_t* bins, int32_t N, int32_t K, int32_t E,
                        float alpha, float* loss, float* P, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (N < 0 || K <= 0 || E <= 0 || K > E) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  if (!bins || !loss || (N > 0 && !probs)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_aux_loss_workspace_size(N, E)) return MOE_ERR_WORKSPACE;
  return aux_loss_fwd(probs, bins, N, K, E, alpha, loss, P, (char*)ws + al256(kStatusBytes),
                      (cudaStream_t)stream);
}

moe_status moe_layer_fwd(const void* x, const void* W_r, const void* W1, const void* W3, const void* W2,
                         int32_t N, int32_t H, int32_t E, int32_t K, int32_t F, moe_dtype dt,
                         int32_t training, int32_t capacity, float aux_alpha, float* aux_loss, void* y,
                         int32_t* top_experts, float* weights, int32_t* indices, int32_t* bins,
                         int32_t* padded_bins, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  MOE_TRY(check_ffn(H, F, dt));
  // token-sized arrays may be NULL for an empty batch (N = 0)
  const void* ptrs[] = {W_r, W1, W3, W2, bins, padded_bins, x, y, top_experts, weights, indices};
  for (int i = 0; i < 11; ++i)
    if ((!ptrs[i] && (i < 6 || N > 0)) || !aligned16(ptrs[i])) return MOE_ERR_INVALID_ARG;
  if (!layer_flags_ok(training, dt)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_workspace_size(N, H, E, K, F, dt, training);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  LayerWs w = carve(ws, N, H, E, K, F, dt, training);
  const int64_t P = p_max(N, E, K);
  const int32_t flags = training;
  const bool gather = (training & MOE_LAYER_GATHER_ROWS) != 0;
  training &= 3;
  const bool aux = aux_alpha != 0.0f;
  if ((aux && !aux_loss) || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (cudaMemsetAsync(w.status + 1, layer_stamp_byte(flags, aux_alpha, capacity), 4, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  // the tensor-core router also counts each 128-token chunk's expert ids
  // into the metadata scratch, which saves the metadata its counting pass
  const bool counted = N > 0 && routes_on_tensor_cores(N, H, E, K, dt);
  MOE_TRY(route_any(x, W_r, N, H, E, K, dt, nullptr, aux ? w.probs : nullptr, top_experts, weights,
                    w.route_scratch, w.status, s, counted ? (int32_t*)w.meta_scratch : nullptr));
  MOE_TRY(dispatch_meta(top_experts, N, K, E, indices, nullptr, bins, padded_bins, w.pos, w.meta_scratch,
                        w.status, s, capacity, w.routed_bins, counted, layer_meta_chunk(N, H, E, K, dt)));
  // f_i of the loss counts routed assignments, dropped ones included
  if (aux) MOE_TRY(aux_loss_fwd(w.probs, w.routed_bins, N, K, E, aux_alpha, aux_loss, nullptr, w.aux_scratch, s));
  if (N == 0) return MOE_OK;
  const RowGather ga = {x, indices, bins, N, K};
  if (!gather) MOE_TRY(permute_rows(x, w.pos, bins, padded_bins, N, H, E, K, dt, w.x_perm, s));
  MOE_TRY(swiglu_any(w.x_perm, W1, W3, W2, padded_bins, E, H, F, P, dt, w.act, w.out,
                     training == 1 ? w.gate_up : nullptr, w.status, s, gather ? &ga : nullptr));
  MOE_TRY(combine_rows(w.out, weights, w.pos, N, K, H, dt, y, s));
  return MOE_OK;
}

moe_status moe_layer_bwd(const void* dy, const void* x, const void* W_r, const void* W1, const void* W3,
                         const void* W2, const int32_t* top_experts, const float* weights,
                         const int32_t* indices, const int32_t* bins, const int32_t* padded_bins,
                         int32_t N, int32_t H, int32_t E, int32_t K, int32_t F, moe_dtype dt,
                         int32_t training, int32_t capacity, float aux_alpha, float aux_grad, void* dx,
                         void* dW_r, void* dW1, void* dW3, void* dW2, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  MOE_TRY(check_shape(N, H, E, K, dt));
  MOE_TRY(check_ffn(H, F, dt));
  // token-sized arrays may be NULL for an empty batch (N = 0)
  const void* ptrs[] = {W_r, W1, W3, W2, bins, padded_bins, dW_r, dW1, dW3, dW2,
                        dy, x, top_experts, weights, indices, dx};
  for (int i = 0; i < 16; ++i)
    if ((!ptrs[i] && (i < 10 || N > 0)) || !aligned16(ptrs[i])) return MOE_ERR_INVALID_ARG;
  if (!layer_flags_ok(training, dt) || ((training & 3) != 1 && (training & 3) != 2)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_workspace_size(N, H, E, K, F, dt, training);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    // no tokens: every weight gradient is an empty sum
    const size_t eb = elem_bytes(dt);
    if (cudaMemsetAsync(dW_r, 0, (size_t)H * E * eb, s) != cudaSuccess ||
        cudaMemsetAsync(dW1, 0, (size_t)E * H * F * eb, s) != cudaSuccess ||
        cudaMemsetAsync(dW3, 0, (size_t)E * H * F * eb, s) != cudaSuccess ||
        cudaMemsetAsync(dW2, 0, (size_t)E * F * H * eb, s) != cudaSuccess) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    return MOE_OK;
  }
  LayerWs w = carve(ws, N, H, E, K, F, dt, training);
  const int64_t P = p_max(N, E, K);
  const RowGather ga = {x, indices, bins, N, K};
  const uint32_t stamp = (uint32_t)layer_stamp_byte(training, aux_alpha, capacity) * 0x01010101u;
  // the sparse router backward walks the kept assignments only; the aux loss
  // and dropped assignments need every (token, expert) logit: dense path
  const bool dense_router = (aux_alpha != 0.0f || capacity > 0) && N > 0;
  // First launch: the check of the forward's recorded flags; on the sparse
  // router path it is fused into the W_r^T transpose that path needs.
  const bool wrt_first = !dense_router && N > 0;
  if (wrt_first) {
    MOE_TRY(transpose_matrix(W_r, H, E, dt, w.ur_scratch, s, 0, w.status, (int)stamp));
  } else {
    MOE_TRACED("layer_flags_check", s, (layer_stamp_check_kernel<<<1, 32, 0, s>>>(w.status, (int)stamp)));
    MOE_LAUNCH_CHECK();
  }
  const bool gather = (training & MOE_LAYER_GATHER_ROWS) != 0;
  training &= 3;
  void* gate_up = w.gate_up;
  if (training == 2) {
    // recompute G, U (same kernel and inputs as the forward: identical bits)
    // into the dG, dU scratch; the SwiGLU backward then runs in place there
    gate_up = w.d_gate_up;
    const size_t eb = elem_bytes(dt);
    void* G = w.d_gate_up;
    void* U = (char*)w.d_gate_up + (size_t)P * F * eb;
    if (dt == MOE_F32)
      MOE_TRY(gate_up_simt(w.x_perm, W1, W3, padded_bins, E, H, F, P, G, U, s));
    else
      MOE_TRY(gemm1_umma(w.x_perm, W1, W3, padded_bins, E, H, F, P, nullptr, G, U, w.status, s,
                         "gate_up_recompute", gather ? &ga : nullptr));
  }
  // the sparse router backward of a bf16 layer takes x^T D on the tensor
  // cores; the combine backward writes D (bf16) beside the dlogits
  void* Dh = (!dense_router && dt == MOE_BF16 && router_wgrad_tc_supported(H, E))
                 ? unpermute_router_bwd_dh(w.ur_scratch, N, H, E, P)
                 : nullptr;
  MOE_TRY(combine_bwd_rows(dy, w.out, weights, w.pos, bins, padded_bins, N, K, H, E, dt, nullptr,
                           w.dlogit, w.d_out, s, top_experts, Dh));
  MOE_TRY(swiglu_bwd_any(w.d_out, w.x_perm, w.act, gate_up, W1, W3, W2, padded_bins, E, H, F, P, dt,
                         w.d_gate_up, dW1, dW3, dW2, w.dx_perm, w.status, s, gather ? &ga : nullptr));
  // dense path: the router probabilities exist only when the forward
  // computed the loss
  if (dense_router)
    MOE_TRY(dense_router_bwd(w.dx_perm, w.dlogit, x, W_r, top_experts, w.pos, w.routed_bins,
                             aux_alpha != 0.0f ? w.probs : nullptr, N, H, E, K, dt, aux_alpha, aux_grad, dx,
                             dW_r, w.dense_scratch, w.status, s));
  else
    MOE_TRY(unpermute_router_bwd(w.dx_perm, w.dlogit, x, W_r, top_experts, w.pos, indices, bins,
                                 padded_bins, N, H, E, K, P, dt, dx, dW_r, w.ur_scratch, w.status, s,
                                 Dh != nullptr, wrt_first));
  return MOE_OK;
}

}  // extern "C"

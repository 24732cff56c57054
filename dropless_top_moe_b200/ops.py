"""Torch-facing wrappers over the C ABI, one per entry point, same names.

Each wrapper checks devices and dtypes, allocates the output tensors with
torch (device memory is torch's job here) and passes raw pointers plus the
current CUDA stream to libmoe_b200.so.  No arithmetic of the layer happens
in Python.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import MOE_BF16, MOE_F32, call, load

_DT = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")
    return _DT[t.dtype]


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _check(name: str, t: Optional[torch.Tensor], shape=None, dtype=None, numel=None):
    """Shape and dtype of an argument against the sizes the call derives from
    the others.  The library reads and writes through raw pointers with those
    sizes, so a mismatched tensor would be read or written out of bounds;
    it is refused here instead."""
    if t is None:
        return
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")


def _experts(W1, W3, W2, H: int, dtype):
    """E, F of the stacked expert weights W1, W3 [E,H,F] and W2 [E,F,H]."""
    if W1.dim() != 3:
        raise ValueError(f"W1: expected [E, H, F], got {tuple(W1.shape)}")
    E, _, F = W1.shape
    _check("W1", W1, (E, H, F), dtype)
    _check("W3", W3, (E, H, F), dtype)
    _check("W2", W2, (E, F, H), dtype)
    return E, F


def _stream():
    return torch.cuda.current_stream().cuda_stream


def tile_rows() -> int:
    return load().moe_tile_rows()


def padded_rows_max(N: int, E: int, K: int) -> int:
    return load().moe_padded_rows_max(N, E, K)


def workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned device workspace with its status word zeroed."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    call("moe_workspace_init", ws.data_ptr(), ws.numel(), _stream())
    return ws


def device_status(ws: torch.Tensor) -> int:
    import ctypes
    v = ctypes.c_int32(0)
    call("moe_get_device_status", ws.data_ptr(), ctypes.addressof(v), _stream())
    return v.value


def moe_route(x, W_r, K: int, want_logits: bool = False, want_probs: bool = False, ws=None) -> dict:
    N, H = x.shape
    E = W_r.shape[1]
    _check("W_r", W_r, (H, E), x.dtype)
    dev = x.device
    dt = _dt(x)
    if ws is None:
        ws = workspace(load().moe_route_workspace_size(N, H, E, K, dt), dev)
    out = {
        "top_experts": torch.empty(N, K, dtype=torch.int32, device=dev),
        "weights": torch.empty(N, K, dtype=torch.float32, device=dev),
        "logits": torch.empty(N, E, dtype=torch.float32, device=dev) if want_logits else None,
        "probs": torch.empty(N, E, dtype=torch.float32, device=dev) if want_probs else None,
        "ws": ws,
    }
    call("moe_route", _p(x), _p(W_r), N, H, E, K, dt, _p(out["logits"]), _p(out["probs"]),
         _p(out["top_experts"]), _p(out["weights"]), ws.data_ptr(), ws.numel(), _stream())
    return out


def moe_dispatch_meta(top_experts, E: int, ws=None, capacity: int = 0) -> dict:
    N, K = top_experts.shape
    _check("top_experts", top_experts, dtype=torch.int32)
    dev = top_experts.device
    if ws is None:
        ws = workspace(load().moe_dispatch_meta_workspace_size(N, K, E), dev)
    NK = N * K
    out = {k: torch.empty(NK, dtype=torch.int32, device=dev) for k in ("indices", "bin_ids", "pos")}
    out["bins"] = torch.empty(E, dtype=torch.int32, device=dev)
    out["padded_bins"] = torch.empty(E, dtype=torch.int32, device=dev)
    out["ws"] = ws
    call("moe_dispatch_meta", _p(top_experts), N, K, E, int(capacity), _p(out["indices"]), _p(out["bin_ids"]),
         _p(out["bins"]), _p(out["padded_bins"]), _p(out["pos"]), ws.data_ptr(), ws.numel(),
         _stream())
    return out


def moe_permute(x, pos, bins, padded_bins, K: int, P: Optional[int] = None, out=None):
    N, H = x.shape
    E = bins.shape[0]
    _check("pos", pos, dtype=torch.int32, numel=N * K)
    _check("bins", bins, (E,), torch.int32)
    _check("padded_bins", padded_bins, (E,), torch.int32)
    if P is None:
        P = padded_rows_max(N, E, K) if out is None else out.shape[0]
    _check("out", out, (P, H), x.dtype)
    if out is None:
        out = torch.empty(P, H, dtype=x.dtype, device=x.device)
    call("moe_permute", _p(x), _p(pos), _p(bins), _p(padded_bins), N, H, E, K, _dt(x), _p(out),
         _stream())
    return out


def moe_grouped_swiglu(x_perm, W1, W3, W2, padded_bins, save_gate_up: bool = False, ws=None):
    P, H = x_perm.shape
    E, F = _experts(W1, W3, W2, H, x_perm.dtype)
    _check("padded_bins", padded_bins, (E,), torch.int32)
    dev = x_perm.device
    if ws is None:
        ws = workspace(load().moe_grouped_workspace_size(), dev)
    act = torch.empty(P, F, dtype=x_perm.dtype, device=dev)
    out = torch.empty(P, H, dtype=x_perm.dtype, device=dev)
    gate_up = torch.empty(2, P, F, dtype=x_perm.dtype, device=dev) if save_gate_up else None
    call("moe_grouped_swiglu", _p(x_perm), _p(W1), _p(W3), _p(W2), _p(padded_bins), E, H, F, P,
         _dt(x_perm), _p(act), _p(out), _p(gate_up), ws.data_ptr(), ws.numel(), _stream())
    return act, out, gate_up


def moe_combine(out, weights, pos, N: int, y=None):
    _, H = out.shape
    K = weights.shape[1]
    _check("weights", weights, (N, K), torch.float32)
    _check("pos", pos, dtype=torch.int32, numel=N * K)
    _check("y", y, (N, H), out.dtype)
    if y is None:
        y = torch.empty(N, H, dtype=out.dtype, device=out.device)
    call("moe_combine", _p(out), _p(weights), _p(pos), N, K, H, _dt(out), _p(y), _stream())
    return y


def moe_combine_bwd(dy, out, weights, pos, bins, padded_bins):
    N, H = dy.shape
    K = weights.shape[1]
    E = bins.shape[0]
    P = out.shape[0]
    _check("out", out, (P, H), dy.dtype)
    _check("weights", weights, (N, K), torch.float32)
    _check("pos", pos, dtype=torch.int32, numel=N * K)
    _check("bins", bins, (E,), torch.int32)
    _check("padded_bins", padded_bins, (E,), torch.int32)
    dev = dy.device
    dw = torch.empty(N, K, dtype=torch.float32, device=dev)
    dlogit = torch.empty(N, K, dtype=torch.float32, device=dev)
    d_out = torch.empty(P, H, dtype=dy.dtype, device=dev)
    call("moe_combine_bwd", _p(dy), _p(out), _p(weights), _p(pos), _p(bins), _p(padded_bins), N, K, H,
         E, _dt(dy), _p(dw), _p(dlogit), _p(d_out), _stream())
    return dw, dlogit, d_out


def moe_grouped_swiglu_bwd(d_out, x_perm, act, gate_up, W1, W3, W2, padded_bins, ws=None):
    P, H = x_perm.shape
    E, F = _experts(W1, W3, W2, H, x_perm.dtype)
    _check("d_out", d_out, (P, H), x_perm.dtype)
    _check("act", act, (P, F), x_perm.dtype)
    _check("gate_up", gate_up, (2, P, F), x_perm.dtype)
    _check("padded_bins", padded_bins, (E,), torch.int32)
    dev = x_perm.device
    if ws is None:
        ws = workspace(load().moe_grouped_workspace_size(), dev)
    dt = x_perm.dtype
    d_gate_up = torch.empty(2, P, F, dtype=dt, device=dev)
    dW1 = torch.empty(E, H, F, dtype=dt, device=dev)
    dW3 = torch.empty(E, H, F, dtype=dt, device=dev)
    dW2 = torch.empty(E, F, H, dtype=dt, device=dev)
    dx_perm = torch.empty(P, H, dtype=dt, device=dev)
    call("moe_grouped_swiglu_bwd", _p(d_out), _p(x_perm), _p(act), _p(gate_up), _p(W1), _p(W3), _p(W2),
         _p(padded_bins), E, H, F, P, _dt(x_perm), _p(d_gate_up), _p(dW1), _p(dW3), _p(dW2),
         _p(dx_perm), ws.data_ptr(), ws.numel(), _stream())
    return {"d_gate_up": d_gate_up, "dW1": dW1, "dW3": dW3, "dW2": dW2, "dx_perm": dx_perm}


def moe_unpermute_router_bwd(dx_perm, dlogit, x, W_r, top_experts, pos, indices, bins, padded_bins,
                             probs=None, aux_alpha: float = 0.0, aux_grad: float = 1.0, ws=None):
    N, H = x.shape
    E = W_r.shape[1]
    K = top_experts.shape[1]
    P = dx_perm.shape[0]
    _check("dx_perm", dx_perm, (P, H), x.dtype)
    _check("dlogit", dlogit, (N, K), torch.float32)
    _check("W_r", W_r, (H, E), x.dtype)
    _check("top_experts", top_experts, (N, K), torch.int32)
    for name, t in (("pos", pos), ("indices", indices)):
        _check(name, t, dtype=torch.int32, numel=N * K)
    _check("bins", bins, (E,), torch.int32)
    _check("padded_bins", padded_bins, (E,), torch.int32)
    _check("probs", probs, (N, E), torch.float32)
    dev = x.device
    if ws is None:
        ws = workspace(load().moe_unpermute_router_bwd_workspace_size(N, H, E, P), dev)
    dx = torch.empty(N, H, dtype=x.dtype, device=dev)
    dW_r = torch.empty(H, E, dtype=x.dtype, device=dev)
    call("moe_unpermute_router_bwd", _p(dx_perm), _p(dlogit), _p(x), _p(W_r), _p(top_experts), _p(pos),
         _p(indices), _p(bins), _p(padded_bins), _p(probs), float(aux_alpha), float(aux_grad), N, H, E, K, P,
         _dt(x), _p(dx), _p(dW_r), ws.data_ptr(), ws.numel(), _stream())
    return dx, dW_r


def moe_aux_loss(probs, bins, K: int, alpha: float, ws=None):
    """Load-balancing loss alpha * E * sum_i f_i * P_i; returns (loss [1], P [E])."""
    N, E = probs.shape
    _check("probs", probs, dtype=torch.float32)
    _check("bins", bins, (E,), torch.int32)
    dev = probs.device
    if ws is None:
        ws = workspace(load().moe_aux_loss_workspace_size(N, E), dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    P = torch.empty(E, dtype=torch.float32, device=dev)
    call("moe_aux_loss", _p(probs), _p(bins), N, K, E, float(alpha), _p(loss), _p(P), ws.data_ptr(),
         ws.numel(), _stream())
    return loss, P


def selftest_wait_timeout(status, timeout_ns: int):
    """Run the bounded pipeline wait on a barrier nothing arrives at; after
    timeout_ns it sets MOE_DEVERR_TIMEOUT in status (a device int32 tensor)."""
    call("moe_selftest_wait_timeout", _p(status), int(timeout_ns), _stream())
    return status


class MoELayer:
    """Whole-layer forward / backward through moe_layer_fwd / moe_layer_bwd.

    Holds the workspace between the forward and the backward pass.  Weights
    are passed per call so the caller owns them (and their gradients).
    """

    def __init__(self, N: int, H: int, E: int, K: int, F: int, dtype=torch.bfloat16,
                 training: bool = False, device="cuda", aux_alpha: float = 0.0, capacity: int = 0,
                 gather_rows: bool = False):
        self.N, self.H, self.E, self.K, self.F = N, H, E, K, F
        self.dtype, self.training = dtype, bool(training)
        # training: False/0 forward only; True/1 keep G, U; 2 recompute them in backward.
        # gather_rows (bf16): GEMM1 and dW1/dW3 read rows of x directly, no permuted copy
        self.mode = (0 if not training else (2 if training == 2 else 1)) | \
            (_lib.MOE_LAYER_GATHER_ROWS if gather_rows else 0)
        self.aux_alpha = float(aux_alpha)
        self.capacity = int(capacity)   # 0 = dropless
        self.device = torch.device(device)
        self.dt = _DT[dtype]
        nbytes = load().moe_workspace_size(N, H, E, K, F, self.dt, self.mode)
        if nbytes == 0:
            raise _lib.MoEError("moe_workspace_size", _lib.MOE_ERR_UNSUPPORTED)
        self.ws = workspace(nbytes, self.device)
        dev = self.device
        self.y = torch.empty(N, H, dtype=dtype, device=dev)
        self.top_experts = torch.empty(N, K, dtype=torch.int32, device=dev)
        self.weights = torch.empty(N, K, dtype=torch.float32, device=dev)
        self.indices = torch.empty(N * K, dtype=torch.int32, device=dev)
        self.bins = torch.empty(E, dtype=torch.int32, device=dev)
        self.padded_bins = torch.empty(E, dtype=torch.int32, device=dev)
        self.aux_loss = torch.zeros(1, dtype=torch.float32, device=dev)
        self._grads = None

    def _check_params(self, x, W_r, W1, W3, W2):
        N, H, E, F, dt = self.N, self.H, self.E, self.F, self.dtype
        _check("x", x, (N, H), dt)
        _check("W_r", W_r, (H, E), dt)
        _check("W1", W1, (E, H, F), dt)
        _check("W3", W3, (E, H, F), dt)
        _check("W2", W2, (E, F, H), dt)

    def forward(self, x, W_r, W1, W3, W2, y=None):
        self._check_params(x, W_r, W1, W3, W2)
        _check("y", y, (self.N, self.H), self.dtype)
        y = self.y if y is None else y
        call("moe_layer_fwd", _p(x), _p(W_r), _p(W1), _p(W3), _p(W2), self.N, self.H, self.E, self.K,
             self.F, self.dt, self.mode, self.capacity, self.aux_alpha, _p(self.aux_loss), _p(y),
             _p(self.top_experts), _p(self.weights),
             _p(self.indices), _p(self.bins), _p(self.padded_bins), self.ws.data_ptr(),
             self.ws.numel(), _stream())
        return y

    def grad_buffers(self):
        if self._grads is None:
            dev, dt = self.device, self.dtype
            N, H, E, F = self.N, self.H, self.E, self.F
            self._grads = {"dx": torch.empty(N, H, dtype=dt, device=dev),
                           "dW_r": torch.empty(H, E, dtype=dt, device=dev),
                           "dW1": torch.empty(E, H, F, dtype=dt, device=dev),
                           "dW3": torch.empty(E, H, F, dtype=dt, device=dev),
                           "dW2": torch.empty(E, F, H, dtype=dt, device=dev)}
        return self._grads

    def backward(self, dy, x, W_r, W1, W3, W2, grads=None, aux_grad: float = 1.0):
        """Gradients of sum(y * dy) (+ aux_grad * aux_loss when aux_alpha != 0)."""
        if not self.training:
            raise RuntimeError("layer was built with training=False")
        self._check_params(x, W_r, W1, W3, W2)
        _check("dy", dy, (self.N, self.H), self.dtype)
        g = self.grad_buffers() if grads is None else grads
        shapes = {"dx": (self.N, self.H), "dW_r": (self.H, self.E), "dW1": (self.E, self.H, self.F),
                  "dW3": (self.E, self.H, self.F), "dW2": (self.E, self.F, self.H)}
        for k, shp in shapes.items():
            _check(k, g[k], shp, self.dtype)
        call("moe_layer_bwd", _p(dy), _p(x), _p(W_r), _p(W1), _p(W3), _p(W2), _p(self.top_experts),
             _p(self.weights), _p(self.indices), _p(self.bins), _p(self.padded_bins), self.N, self.H,
             self.E, self.K, self.F, self.dt, self.mode, self.capacity, self.aux_alpha, float(aux_grad),
             _p(g["dx"]),
             _p(g["dW_r"]),
             _p(g["dW1"]), _p(g["dW3"]),
             _p(g["dW2"]), self.ws.data_ptr(), self.ws.numel(), _stream())
        return g

    def status(self) -> int:
        return device_status(self.ws)

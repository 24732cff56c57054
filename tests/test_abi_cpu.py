"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/moe.h declares, and rejects bad arguments before any
device work.  Pointers passed here are never dereferenced (validation
returns first)."""
import os
import re

import pytest

from dropless_top_moe_b200 import _lib
from dropless_top_moe_b200._lib import (MOE_BF16, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED,
                                        MOE_ERR_WORKSPACE, MOE_F32, load)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:moe_status|size_t|int32_t|int64_t)\s+(moe_\w+)\s*\(",
                                 text, flags=re.M)))


def test_binding_constants_match_the_header():
    text = open(HEADER).read()
    defines = {m.group(1): int(m.group(2), 0)
               for m in re.finditer(r"^#define\s+(MOE_\w+)\s+(0x[0-9a-fA-F]+|\d+)", text, flags=re.M)}
    for name in ("MOE_DEVERR_EXPERT_ID", "MOE_DEVERR_TIMEOUT", "MOE_DEVERR_ROWS", "MOE_DEVERR_MODE",
                 "MOE_LAYER_GATHER_ROWS"):
        assert getattr(_lib, name) == defines[name], name
    bits = [defines[n] for n in defines if n.startswith("MOE_DEVERR_")]
    assert len(bits) == len(set(bits)) == 4 and all(b & (b - 1) == 0 for b in bits)


@pytest.fixture(scope="module")
def lib():
    from dropless_top_moe_b200.build import build
    build()
    return load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"{n} missing from the binding"
    assert set(_lib.SIGNATURES) == set(names)


def test_static_sizes(lib):
    assert lib.moe_tile_rows() == 128
    assert lib.moe_padded_rows_max(4096, 8, 2) == 9216
    assert lib.moe_padded_rows_max(8192, 256, 8) == 98048
    assert lib.moe_padded_rows_max(16384, 64, 6) == 106496
    assert lib.moe_padded_rows_max(16384, 64, 4) == 73728
    assert lib.moe_padded_rows_max(0, 4, 2) == 512


def test_workspace_sizes(lib):
    inf = lib.moe_workspace_size(4096, 4096, 8, 2, 14336, MOE_BF16, 0)
    trn = lib.moe_workspace_size(4096, 4096, 8, 2, 14336, MOE_BF16, 1)
    P = 9216
    assert inf >= P * (4096 * 2 + 14336) * 2
    assert trn > inf + 2 * P * 14336 * 2
    assert lib.moe_workspace_size(4096, 4000, 8, 2, 14336, MOE_BF16, 0) == 0   # H % 128
    assert lib.moe_workspace_size(16, 8, 4, 5, 8, MOE_F32, 0) == 0             # K > E
    assert lib.moe_dispatch_meta_workspace_size(100, 2, 4) >= 256


def test_gather_rows_flag_drops_the_permuted_copy(lib):
    N, H, E, K, F = 4096, 4096, 8, 2, 14336
    P = lib.moe_padded_rows_max(N, E, K)
    G = _lib.MOE_LAYER_GATHER_ROWS
    for mode in (0, 1, 2):
        plain = lib.moe_workspace_size(N, H, E, K, F, MOE_BF16, mode)
        gathered = lib.moe_workspace_size(N, H, E, K, F, MOE_BF16, mode | G)
        assert plain - gathered == P * H * 2, mode
    assert lib.moe_workspace_size(N, H, E, K, F, MOE_BF16, 3) == 0            # no mode 3
    assert lib.moe_workspace_size(N, H, E, K, F, MOE_BF16, 8) == 0            # unknown flag
    assert lib.moe_workspace_size(256, 128, 4, 2, 256, MOE_F32, 1 | G) == 0   # bf16 only


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_route_rejects_bad_shapes(lib):
    ws_size = 1 << 20
    assert lib.moe_route(FAKE, FAKE, 16, 128, 4, 5, MOE_F32, None, None, FAKE, FAKE, FAKE, ws_size,
                         None) == MOE_ERR_INVALID_ARG
    assert lib.moe_route(FAKE, FAKE, 16, 100, 4, 2, MOE_BF16, None, None, FAKE, FAKE, FAKE, ws_size,
                         None) == MOE_ERR_UNSUPPORTED
    assert lib.moe_route(FAKE, FAKE, 16, 128, 300, 2, MOE_BF16, None, None, FAKE, FAKE, FAKE, ws_size,
                         None) == MOE_ERR_UNSUPPORTED
    assert lib.moe_route(FAKE + 4, FAKE, 16, 128, 4, 2, MOE_F32, None, None, FAKE, FAKE, FAKE, ws_size,
                         None) == MOE_ERR_INVALID_ARG
    assert lib.moe_route(FAKE, FAKE, 16, 128, 4, 2, MOE_F32, None, None, FAKE, FAKE, FAKE, 8,
                         None) == MOE_ERR_WORKSPACE


def test_layer_rejects_bad_arguments(lib):
    # x W_r W1 W3 W2 | N H E K F dt training capacity aux_alpha aux_loss | y top w idx bins pbins
    args = [FAKE] * 5 + [64, 128, 4, 2, 256, MOE_BF16, 0, 0, 0.0, None] + [FAKE] * 6
    assert lib.moe_layer_fwd(*args, FAKE, 1024, None) == MOE_ERR_WORKSPACE
    bad = list(args)
    bad[0] = None
    assert lib.moe_layer_fwd(*bad, FAKE, 1 << 40, None) == MOE_ERR_INVALID_ARG
    bad = list(args)
    bad[9] = 100   # F not a multiple of 128 on the tensor-core path
    assert lib.moe_layer_fwd(*bad, FAKE, 1 << 40, None) == MOE_ERR_UNSUPPORTED
    bad = list(args)
    bad[8] = 5     # K > E
    assert lib.moe_layer_fwd(*bad, FAKE, 1 << 40, None) == MOE_ERR_INVALID_ARG
    bad = list(args)
    bad[13] = 0.01  # aux loss requested without an output pointer
    assert lib.moe_layer_fwd(*bad, FAKE, 1 << 40, None) == MOE_ERR_INVALID_ARG


def test_meta_and_grouped_reject_bad_arguments(lib):
    assert lib.moe_dispatch_meta(FAKE, 10, 3, 2, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
                                 None) == MOE_ERR_INVALID_ARG
    assert lib.moe_dispatch_meta(FAKE, 10, 2, 4, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16,
                                 None) == MOE_ERR_WORKSPACE
    assert lib.moe_dispatch_meta(FAKE, 10, 2, 4, -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
                                 None) == MOE_ERR_INVALID_ARG
    # P must be a multiple of 128
    assert lib.moe_grouped_swiglu(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 256, 100, MOE_BF16, FAKE, FAKE,
                                  None, FAKE, 4096, None) == MOE_ERR_INVALID_ARG


def test_stage_entry_points_reject_bad_arguments(lib):
    INV, UNS, WS = MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE
    big = 1 << 40
    # permute: x pos bins padded_bins N H E K dt x_perm
    assert lib.moe_permute(FAKE, FAKE, FAKE, FAKE, 16, 128, 4, 5, MOE_BF16, FAKE, None) == INV      # K > E
    assert lib.moe_permute(FAKE, FAKE, FAKE, FAKE, 16, 128, 4, 2, MOE_BF16, None, None) == INV
    assert lib.moe_permute(FAKE + 4, FAKE, FAKE, FAKE, 16, 128, 4, 2, MOE_BF16, FAKE, None) == INV
    assert lib.moe_permute(FAKE, FAKE, FAKE, FAKE, 16, 96, 4, 2, MOE_BF16, FAKE, None) == UNS        # H % 128
    # combine: out weights pos N K H dt y (an empty batch returns before any device work)
    assert lib.moe_combine(None, FAKE, FAKE, 16, 2, 128, MOE_BF16, FAKE, None) == INV
    assert lib.moe_combine(FAKE, FAKE, FAKE, 16, 2, 128, MOE_BF16, FAKE + 8, None) == INV
    assert lib.moe_combine(None, None, None, 0, 2, 128, MOE_BF16, None, None) == 0
    # combine_bwd: dy out weights pos bins padded_bins N K H E dt dw dlogit d_out
    assert lib.moe_combine_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 2, 128, 4, MOE_BF16, None, None,
                               FAKE, None) == INV                                               # no dlogit
    assert lib.moe_combine_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 2, 128, 4, MOE_BF16, None, FAKE,
                               None, None) == INV                                               # no d_out
    # grouped SwiGLU backward: 7 inputs, padded_bins, E H F P dt, 5 outputs, ws
    g = [FAKE] * 7 + [FAKE, 4, 128, 256]
    out = [FAKE] * 5
    assert lib.moe_grouped_swiglu_bwd(*g, 100, MOE_BF16, *out, FAKE, big, None) == INV          # P % 128
    assert lib.moe_grouped_swiglu_bwd(*g, 128, MOE_BF16, *out[:4], None, FAKE, big, None) == INV
    assert lib.moe_grouped_swiglu_bwd(*g, 128, MOE_BF16, *out, FAKE, 16, None) == WS
    assert lib.moe_grouped_swiglu_bwd(*g[:9], 200, 256, 128, MOE_BF16, *out, FAKE, big, None) == UNS
    # unpermute + router backward: 9 pointers, probs, aux_alpha aux_grad, N H E K P dt, dx dW_r, ws
    u = [FAKE] * 9
    assert lib.moe_unpermute_router_bwd(*u, None, 0.5, 1.0, 16, 128, 4, 2, 256, MOE_BF16, FAKE, FAKE,
                                        FAKE, big, None) == INV                                 # aux without probs
    assert lib.moe_unpermute_router_bwd(*u, None, 0.0, 1.0, 16, 128, 4, 2, 256, MOE_BF16, FAKE, FAKE,
                                        FAKE, 64, None) == WS
    assert lib.moe_unpermute_router_bwd(*u, None, 0.0, 1.0, 16, 128, 4, 2, 200, MOE_BF16, FAKE, FAKE,
                                        FAKE, big, None) == INV                                 # P % 128
    # aux loss: probs bins N K E alpha loss P ws
    assert lib.moe_aux_loss(FAKE, FAKE, 16, 5, 4, 0.01, FAKE, None, FAKE, big, None) == INV      # K > E
    assert lib.moe_aux_loss(FAKE, FAKE, 16, 2, 300, 0.01, FAKE, None, FAKE, big, None) == UNS
    assert lib.moe_aux_loss(FAKE, FAKE, 16, 2, 4, 0.01, None, None, FAKE, big, None) == INV     # no loss
    assert lib.moe_aux_loss(FAKE, FAKE, 16, 2, 4, 0.01, FAKE, None, FAKE, 8, None) == WS
    # rank-ordered sum: shards n_ranks numel dt scale out
    assert lib.moe_sum_rank_ordered(FAKE, 0, 64, MOE_BF16, 1.0, FAKE, None) == INV
    assert lib.moe_sum_rank_ordered(FAKE, 2, 64, 7, 1.0, FAKE, None) == INV                     # unknown dtype
    assert lib.moe_sum_rank_ordered(FAKE + 4, 2, 64, MOE_BF16, 1.0, FAKE, None) == INV
    assert lib.moe_sum_rank_ordered(FAKE, 2, 12, MOE_BF16, 1.0, FAKE, None) == UNS              # 12 % 8
    assert lib.moe_sum_rank_ordered(FAKE, 2, 0, MOE_BF16, 1.0, FAKE, None) == 0
    # dispatch metadata without allocation: the fixed scratch bounds N*K
    assert lib.moe_dispatch_meta_noalloc(FAKE, 16, 5, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == INV
    assert lib.moe_dispatch_meta_noalloc(FAKE, 16, 2, 300, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == UNS
    assert lib.moe_dispatch_meta_noalloc(FAKE, 16, 2, 4, FAKE, FAKE, FAKE, None, FAKE, None, None) == INV
    assert lib.moe_dispatch_meta_noalloc(FAKE, 1000000, 2, 256, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                         None) == WS
    # tracing
    assert lib.moe_trace_attach(None, 4, None, FAKE) == INV
    assert lib.moe_trace_attach(FAKE, 0, None, FAKE) == INV


def test_layer_backward_rejects_bad_flags(lib):
    G = _lib.MOE_LAYER_GATHER_ROWS
    # 11 pointers | N H E K F dt training capacity aux_alpha aux_grad | dx dW_r dW1 dW3 dW2
    def bwd(training, dt=MOE_BF16, ws_bytes=1 << 40):
        return lib.moe_layer_bwd(*([FAKE] * 11), 64, 128, 4, 2, 256, dt, training, 0, 0.0, 1.0,
                                 *([FAKE] * 5), FAKE, ws_bytes, None)
    assert bwd(0) == MOE_ERR_INVALID_ARG                 # a forward-only layer has no backward
    assert bwd(3) == MOE_ERR_INVALID_ARG
    assert bwd(1 | 8) == MOE_ERR_INVALID_ARG             # unknown flag bit
    assert bwd(1 | G, dt=MOE_F32) == MOE_ERR_INVALID_ARG  # row gathers are bf16 only
    assert bwd(1, ws_bytes=1024) == MOE_ERR_WORKSPACE
    for bad in (3, 8, 1 | 8):
        assert lib.moe_workspace_size(64, 128, 4, 2, 256, MOE_BF16, bad) == 0
    assert lib.moe_workspace_size(64, 128, 4, 2, 256, MOE_F32, 1 | G) == 0


def test_selftest_rejects_bad_arguments(lib):
    assert lib.moe_selftest_wait_timeout(None, 1000000, None) == MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(FAKE, 10, None) == MOE_ERR_INVALID_ARG            # < 1 us
    assert lib.moe_selftest_wait_timeout(FAKE, 5 * 10 ** 9, None) == MOE_ERR_INVALID_ARG   # > 1 s


def test_header_and_c_example_compile_as_c99():
    """include/moe.h is plain C: the C caller in tests/c_api compiles as C99
    (syntax and types only; running it needs a GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if not os.path.exists(os.path.join(cuda, "include", "cuda_runtime.h")):
        pytest.skip("no CUDA headers")
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                          "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                          os.path.join(ROOT, "tests", "c_api", "layer_fwd.c")], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_workspace_sizes_over_many_shapes_do_not_crash():
    """Every workspace-size query is host arithmetic on the shape alone: it
    must return for every valid shape (fp32 and bf16, tiny H, odd E, N = 0),
    and the layer's size must grow with the training mode."""
    import itertools
    lib = load()
    for N, H, E, K, F, dt in itertools.product([0, 1, 3, 700, 16384], [32, 64, 128, 384, 4096, 7168],
                                               [1, 3, 8, 16, 100, 256], [1, 2, 8], [48, 256], [0, 1]):
        if K > E:
            continue
        sizes = [lib.moe_workspace_size(N, H, E, K, F, dt, tr) for tr in (0, 1, 2)]
        P = lib.moe_padded_rows_max(N, E, K)
        assert lib.moe_unpermute_router_bwd_workspace_size(N, H, E, P) > 0
        assert lib.moe_dispatch_meta_workspace_size(N, K, E) > 0
        route = lib.moe_route_workspace_size(N, H, E, K, dt)
        assert route == 0 if (dt == 1 and H % 128) else route > 0
        if dt == 1 and (H % 128 or F % 128):
            assert sizes == [0, 0, 0]          # bf16 needs H, F multiples of 128
        else:
            assert 0 < sizes[0] < sizes[2] < sizes[1], (N, H, E, K, F, dt, sizes)

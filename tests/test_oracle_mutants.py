"""The oracle's pins must catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of the oracle's source (a
dropped term, a wrong sign, index or axis, a swapped operand, an off-by-one),
loads the copy as a separate module and runs every pin of
test_oracle_pins.py against it.  At least one pin must fail for each planted
mistake; the unmodified copy must pass them all.  Nothing here touches the
GPU or the library: the mistakes live only in the in-memory copy.
"""
import inspect
import itertools
import types

import pytest

from oracle import moe_oracle
from tests import test_oracle_pins as pins

SOURCE = inspect.getsource(moe_oracle)

# (name, text in the oracle, planted replacement)
MUTANTS = [
    # routing
    ("softmax_over_tokens", "z / z.sum(axis=-1, keepdims=True)", "z / z.sum(axis=0, keepdims=True)"),
    ("ties_to_highest_id", "best = np.argmax(p, axis=1)",
     "best = p.shape[1] - 1 - np.argmax(p[:, ::-1], axis=1)"),
    ("no_renormalisation", "return v / v.sum(axis=-1, keepdims=True)", "return v"),
    ("logits_transposed_weights", "return f64(x) @ f64(W_r)", "return f64(x) @ f64(W_r)[::-1]"),
    ("gaps_among_k_only", "m = min(K + 1, l.shape[1])", "m = min(K, l.shape[1])"),
    # dispatch metadata
    ("unstable_sort", "    for i, e in enumerate(te):\n        if not keep[i]:",
     "    for i, e in reversed(list(enumerate(te))):\n        if not keep[i]:"),
    ("exclusive_bins", "bins = np.cumsum(hist)\n", "bins = np.cumsum(hist) - hist\n"),
    ("pad_to_64", "padded_bins = np.cumsum(round_up(hist))", "padded_bins = np.cumsum(round_up(hist, 64))"),
    ("padded_bound_without_tail", "round_up(N * K + E * (TILE - 1))", "round_up(N * K + E)"),
    ("maxvio_mean_over_tokens", "np.max(hist) / (N * K / E) - 1.0", "np.max(hist) / (N / E) - 1.0"),
    ("capacity_off_by_one", "if seen[e] >= capacity:", "if seen[e] > capacity:"),
    ("capacity_mask_inverted", "w = np.where(kept_mask(te, W1.shape[0], capacity), w, 0.0)",
     "w = np.where(kept_mask(te, W1.shape[0], capacity), 0.0, w)"),
    # permute / expert math / combine
    ("permute_token_major_index", "out[p] = xv[i // K]", "out[p] = xv[i % xv.shape[0]]"),
    ("sigmoid_for_silu", "return g / (1.0 + np.exp(-g))", "return 1.0 / (1.0 + np.exp(-g))"),
    ("gate_and_up_swapped", "return (silu(G) * U) @ W2e", "return (G * silu(U)) @ W2e"),
    ("grouped_uses_w3_for_gate", "G = Xp[start:end] @ W1[e]", "G = Xp[start:end] @ W3[e]"),
    ("combine_slot_reversed", "y[t] += w[t, k] * Ov[p[t, k]]", "y[t] += w[t, K - 1 - k] * Ov[p[t, k]]"),
    # load-balancing loss
    ("aux_without_E", "return float(alpha * E * np.sum(f * P))", "return float(alpha * np.sum(f * P))"),
    ("aux_share_over_tokens", "f = np.bincount(te.reshape(-1), minlength=E) / (N * K)",
     "f = np.bincount(te.reshape(-1), minlength=E) / N"),
    # backward
    ("silu_derivative_sign", "sig * (1.0 + G * (1.0 - sig))", "sig * (1.0 - G * (1.0 - sig))"),
    ("du_without_gate", "dU = dA * G * sig", "dU = dA * sig"),
    ("do_without_weight", "dO = w[rows, slots][:, None] * dys[rows]", "dO = dys[rows]"),
    ("dx_w1_w3_swapped", "dG @ W1e.T + dU @ W3e.T", "dG @ W3e.T + dU @ W1e.T"),
    ("renorm_gradient_dropped",
     "dp_kept = dw / S - np.sum(dw * p_kept, axis=1, keepdims=True) / S ** 2", "dp_kept = dw / S"),
    ("softmax_gradient_sign", "probs * (dp - np.sum(dp * probs, axis=1, keepdims=True))",
     "probs * (dp + np.sum(dp * probs, axis=1, keepdims=True))"),
    ("router_dx_dropped", "dx += dlogits @ W_rv.T", "dx += 0.0 * (dlogits @ W_rv.T)"),
    ("aux_gradient_not_averaged", "aux_grad * aux_alpha * E * f_all[None, :] / N",
     "aux_grad * aux_alpha * E * f_all[None, :]"),
]


def load_copy(source: str, name: str) -> types.ModuleType:
    mod = types.ModuleType(name)
    mod.__file__ = moe_oracle.__file__
    exec(compile(source, f"<{name}>", "exec"), mod.__dict__)
    return mod


def pin_cases():
    """Every pin of test_oracle_pins.py with each of its parameter sets."""
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            yield name, fn, {}
            continue
        argsets = []
        for m in marks:
            names = [a.strip() for a in m.args[0].split(",")]
            argsets.append([dict(zip(names, v if isinstance(v, tuple) else (v,))) for v in m.args[1]])
        for combo in itertools.product(*argsets):
            kw = {}
            for d in combo:
                kw.update(d)
            yield name, fn, kw


def failing_pins(module, monkeypatch, stop_at_first: bool):
    monkeypatch.setattr(pins, "om", module)
    failed = []
    for name, fn, kw in pin_cases():
        try:
            fn(**kw)
        except Exception as exc:       # an assertion, or the mistake breaking a shape
            failed.append((name, kw, type(exc).__name__))
            if stop_at_first:
                break
    return failed


def test_unmodified_copy_passes_every_pin(monkeypatch):
    assert len(list(pin_cases())) >= 30
    assert failing_pins(load_copy(SOURCE, "oracle_copy"), monkeypatch, False) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, old, new, monkeypatch):
    assert SOURCE.count(old) == 1, f"{name}: the text to replace must occur once"
    mutant = load_copy(SOURCE.replace(old, new), f"oracle_{name}")
    assert failing_pins(mutant, monkeypatch, True), f"no pin caught {name}"

"""The oracle's pins have teeth: each plausible mistake, planted in a copy of the oracle,
fails at least one pin of ``tests/test_oracle.py`` (CPU only).

Every mutant is a one-place edit of the oracle's source text, compiled into a fresh
module in memory (the file on disk is never touched); the pins then run against that
module in place of the real one, and the first failing pin ends the mutant's run.
"""

import inspect
import types
from pathlib import Path

import pytest

from tests import test_oracle as P

SRC = (Path(__file__).resolve().parents[1] / "oracle" / "nmoe_oracle.py").read_text()

# name -> (text in the oracle, planted replacement)
MUTANTS = {
    # section 6: packed SwiGLU experts, first half gate (SiLU), second half up
    "gate and up swapped": ("h = silu(rows @ _f64(W1e)) * (rows @ _f64(W3e))",
                            "h = silu(rows @ _f64(W3e)) * (rows @ _f64(W1e))"),
    "SiLU sign": ("return g / (1.0 + np.exp(-g))", "return g / (1.0 + np.exp(g))"),
    # section 6.2: scores, then each expert's top-C by (score, -token)
    "softmax over tokens": (
        "m = l.max(axis=1, keepdims=True)\n        e = np.exp(l - m)\n"
        "        return e / e.sum(axis=1, keepdims=True)",
        "m = l.max(axis=0, keepdims=True)\n        e = np.exp(l - m)\n"
        "        return e / e.sum(axis=0, keepdims=True)"),
    "sigmoid sign": ("return 1.0 / (1.0 + np.exp(-l))", "return 1.0 / (1.0 + np.exp(l))"),
    "ties to the higher token": ("order = np.lexsort((tok, -col))",
                                 "order = np.lexsort((-tok, -col))"),
    "lowest scores chosen": ("order = np.lexsort((tok, -col))",
                             "order = np.lexsort((tok, col))"),
    "chosen tokens unsorted": ("chosen.append(np.sort(tok[order[:C]]))",
                               "chosen.append(tok[order[:C]])"),
    "selection over all tokens, not per segment": (
        "col = s[g * S:(g + 1) * S, e].astype(F64)\n            tok = np.arange(g * S, (g + 1) * S)",
        "col = s[:, e].astype(F64)\n            tok = np.arange(T)"),
    "scores not rounded to fp32": ("return _f64(p).astype(np.float32)", "return _f64(p)"),
    "router bias subtracted": ("l = l + np.repeat(b, S, axis=0)",
                               "l = l - np.repeat(b, S, axis=0)"),
    # combine weights and order
    "combine weight dropped": ("out[rows] += w[e][:, None] * y", "out[rows] += y"),
    "route_scale dropped": ("out[e] = route_scale * w[e] / tot[idx[e]]",
                            "out[e] = w[e] / tot[idx[e]]"),
    "token lists in descending expert order": ("lst = sorted(per_tok[t])",
                                               "lst = sorted(per_tok[t], reverse=True)"),
    # section 6.3: the block's gated residual
    "gate not clamped": ("np.tanh(np.clip(_f64(gate2), -2.0, 2.0))", "np.tanh(_f64(gate2))"),
    "clamp after tanh": ("np.tanh(np.clip(_f64(gate2), -2.0, 2.0))",
                         "np.clip(np.tanh(_f64(gate2)), -2.0, 2.0)"),
    "gate row by token modulo segments": (
        "seg = np.arange(out.shape[0]) // (out.shape[0] // n_segments)",
        "seg = np.arange(out.shape[0]) % n_segments"),
    "residual subtracted": ("return _f64(residual) + out", "return _f64(residual) - out"),
    # section 6.2: the gate reads the unmodulated hidden states, the experts x
    "router ignores its own input": (
        "logits = router_logits(x if router_x is None else router_x, W_r, router_bias, "
        "n_segments)",
        "logits = router_logits(x, W_r, router_bias, n_segments)"),
    "experts transform the router input": (
        "y = swiglu_ffn(x[rows], W1[e], W3[e], W2[e])",
        "y = swiglu_ffn((x if router_x is None else _f64(router_x))[rows], W1[e], W3[e], "
        "W2[e])"),
}


def _mutant_module(name):
    old, new = MUTANTS[name]
    assert old in SRC, f"{name}: the oracle no longer contains {old!r}"
    mod = types.ModuleType("nmoe_oracle_mutant")
    exec(compile(SRC.replace(old, new), f"<oracle: {name}>", "exec"), mod.__dict__)
    return mod


def _pins():
    """(label, zero-argument callable) for every non-slow pin, parametrised cases
    expanded."""
    out = []
    for fname, fn in inspect.getmembers(P, inspect.isfunction):
        if not fname.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        if any(m.name == "slow" for m in marks):
            continue
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            out.append((fname, fn))
            continue
        assert len(params) == 1
        argname, values = params[0].args[0], params[0].args[1]
        assert "," not in argname
        for i, v in enumerate(values):
            out.append((f"{fname}[{i}]", lambda fn=fn, a=argname, v=v: fn(**{a: v})))
    return out


@pytest.mark.parametrize("name", list(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, monkeypatch):
    monkeypatch.setattr(P, "O", _mutant_module(name))
    for label, pin in _pins():
        try:
            pin()
        except Exception:
            return  # caught
    pytest.fail(f"no pin catches the mistake '{name}'")


def test_the_unmutated_oracle_passes_every_pin():
    for label, pin in _pins():
        pin()

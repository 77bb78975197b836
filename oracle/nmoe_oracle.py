"""CPU oracle for the expert-choice MoE feed-forward layer (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code, table or helper with the CUDA library.

What it computes is the MoE layer of NucleusMoE-Image's single-stream DiT block as
described in "Diffusers 中 NucleusMoE-Image 文生图流水线：单流 DiT + MoE 专家层 +
Qwen3-VL 文本编码的全链路解析" (trdm.cn), section 6.2 "expert-choice routing + shared
expert", and section 6 (packed SwiGLU experts, ``gate_up_proj`` of shape
(experts, hidden, 2*moe_intermediate_dim)). In that section:

  * a gate Linear (no bias) scores every token against every expert; the score is a
    softmax (default here) or a sigmoid, giving each expert's affinity for each token;
    the scores are viewed per expert (transposed to experts x tokens);
  * each expert takes its top ``capacity`` tokens, so every expert gets exactly
    ``capacity`` tokens per group;
  * the chosen rows go through that expert's SwiGLU FFN (fused gate/up projection,
    then down projection);
  * the weighted expert outputs are scattered (added) back onto their tokens; the page
    weights them by the token's score, optionally normalised by the total score of the
    token's selections and multiplied by ``route_scale``.

Readings taken where the page is silent:
  * softmax runs over the experts of one token;
  * selection runs over a flat token axis, or per segment when ``n_segments > 1``
    (the page's per-sample selection); C is the per-segment capacity;
  * ties are broken by the lower token index; scores are compared as fp32 values
    (the fp64 softmax rounded to fp32 once), which is what both sides decide on;
  * the chosen tokens of an expert are listed in ascending token order;
  * the first half of the fused gate/up weight is the gate (goes through SiLU), the
    second half is the up projection: h = silu(x W1) * (x W3), y = h W2;
  * combine weight = the token's score for that expert (``"raw"``), or
    route_scale * score / sum of the token's selected scores (``"normalized"``); a
    token chosen by no expert outputs exactly zero; contributions are summed in
    ascending expert order;
  * the page's router input cat([timestep, hidden]) is exactly a per-segment additive
    logit bias ``router_bias[s, e] = temb_s . W_gate[:d_t, e]``
    (see :func:`router_logits_concat` for the literal form);
  * the gate reads the unmodulated hidden states while the experts transform the
    block's input: ``router_x`` gives the router its own input; by default both are x;
  * the shared expert (section 6.2: one SwiGLU feed-forward over every token, the
    routed outputs added onto its output) has its own width F_shared, which the page
    does not give;
  * the block around the layer (section 6.3: the modulation gates pass through
    clamp(-2, 2) and then tanh) adds the layer output to its residual stream as
    ``residual + tanh(clamp(gate2, -2, 2)) * ffn_out``, with one gate vector of d
    values per segment (sample); see :func:`gated_residual`.

Every floating-point step is done in fp64 on the exact values of the inputs.
"""

from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=F64)


# -- router (section 6.2: gate Linear, then softmax or sigmoid) -----------------------

def router_logits(x, W_r, router_bias=None, n_segments: int = 1) -> np.ndarray:
    """logits[t, e] = sum_k x[t, k] W_r[k, e] (+ router_bias[segment(t), e])."""
    x = _f64(x)
    l = x @ _f64(W_r)
    if router_bias is not None:
        T = x.shape[0]
        S = T // n_segments
        b = _f64(router_bias).reshape(n_segments, -1)
        l = l + np.repeat(b, S, axis=0)
    return l


def router_logits_concat(temb, x, W_gate, n_segments: int = 1) -> np.ndarray:
    """The page's literal router: Linear(cat([timestep expanded, hidden])), no bias.

    temb [n_segments, d_t] is broadcast to every token of its segment;
    W_gate [d_t + d, E] maps the concatenated row to expert logits.
    """
    x = _f64(x)
    T = x.shape[0]
    S = T // n_segments
    t_rows = np.repeat(_f64(temb), S, axis=0)
    return np.concatenate([t_rows, x], axis=1) @ _f64(W_gate)


def scores_from_logits(logits, score_fn: str = "softmax") -> np.ndarray:
    """fp64 affinity of every expert for every token."""
    l = _f64(logits)
    if score_fn == "softmax":
        m = l.max(axis=1, keepdims=True)
        e = np.exp(l - m)
        return e / e.sum(axis=1, keepdims=True)
    if score_fn == "sigmoid":
        return 1.0 / (1.0 + np.exp(-l))
    raise ValueError(score_fn)


def round_f32(p) -> np.ndarray:
    """The fp32 scores: each fp64 score rounded once to the nearest fp32."""
    return _f64(p).astype(np.float32)


# -- expert-choice top-C (section 6.2: each expert takes its top `capacity` tokens) ----

def select(scores32, C: int, n_segments: int = 1) -> np.ndarray:
    """idx[e, :] = the tokens expert e chooses, ascending token index.

    Within each segment of T / n_segments tokens, expert e orders the tokens by
    (score descending, token index ascending) and keeps the first C. The result has
    n_segments * C entries per expert.
    """
    s = np.asarray(scores32, dtype=np.float32)
    T, E = s.shape
    S = T // n_segments
    if not (1 <= C <= S):
        raise ValueError("capacity out of range")
    idx = np.empty((E, n_segments * C), dtype=np.int64)
    for e in range(E):
        chosen = []
        for g in range(n_segments):
            col = s[g * S:(g + 1) * S, e].astype(F64)
            tok = np.arange(g * S, (g + 1) * S)
            order = np.lexsort((tok, -col))  # primary: -score, secondary: token
            chosen.append(np.sort(tok[order[:C]]))
        idx[e] = np.concatenate(chosen)
    return idx


def token_lists(idx, T: int):
    """CSR of the selection: tok_ptr[T+1], tok_ent[] with entries e * Ce + slot.

    Ce = idx.shape[1] (entries per expert). Each token lists its (expert, slot)
    pairs in ascending expert order.
    """
    idx = np.asarray(idx)
    E, Ce = idx.shape
    per_tok = [[] for _ in range(T)]
    for e in range(E):
        for slot in range(Ce):
            per_tok[int(idx[e, slot])].append(e * Ce + slot)
    tok_ptr = np.zeros(T + 1, dtype=np.int64)
    ent = []
    for t in range(T):
        lst = sorted(per_tok[t])  # e * Ce + slot ascends with e
        tok_ptr[t + 1] = tok_ptr[t] + len(lst)
        ent.extend(lst)
    return tok_ptr, np.asarray(ent, dtype=np.int64)


# -- experts (section 6: packed SwiGLU experts) --------------------------------------

def silu(g):
    g = _f64(g)
    return g / (1.0 + np.exp(-g))


def swiglu_ffn(rows, W1e, W3e, W2e) -> np.ndarray:
    """y = (silu(rows W1e) * (rows W3e)) W2e."""
    rows = _f64(rows)
    h = silu(rows @ _f64(W1e)) * (rows @ _f64(W3e))
    return h @ _f64(W2e)


# -- combine weights and the layer ----------------------------------------------------

def combine_weights(p, idx, mode: str = "raw", route_scale: float = 1.0) -> np.ndarray:
    """w[e, slot] for every selected (expert, slot).

    raw:        w = p[t, e]
    normalized: w = route_scale * p[t, e] / sum_{e' selecting t} p[t, e']
    """
    p = _f64(p)
    idx = np.asarray(idx)
    E, Ce = idx.shape
    w = np.empty((E, Ce), dtype=F64)
    for e in range(E):
        w[e] = p[idx[e], e]
    if mode == "raw":
        return w
    if mode != "normalized":
        raise ValueError(mode)
    T = p.shape[0]
    tot = np.zeros(T, dtype=F64)
    for e in range(E):
        np.add.at(tot, idx[e], p[idx[e], e])
    out = np.empty_like(w)
    for e in range(E):
        out[e] = route_scale * w[e] / tot[idx[e]]
    return out


def gated_residual(residual, gate2, ffn_out, n_segments: int = 1) -> np.ndarray:
    """Section 6.3: residual + tanh(clamp(gate2, -2, 2)) * ffn_out, the gate row of each
    token's segment (gate2 [n_segments, d]; None means a gate of one)."""
    out = np.asarray(ffn_out, dtype=F64)
    if gate2 is not None:
        g = np.tanh(np.clip(_f64(gate2), -2.0, 2.0))
        seg = np.arange(out.shape[0]) // (out.shape[0] // n_segments)
        out = g[seg] * out
    return _f64(residual) + out


def layer(x, W_r, W1, W3, W2, C: int, *, score_fn: str = "softmax",
          combine: str = "raw", route_scale: float = 1.0, n_segments: int = 1,
          router_bias=None, selection=None, shared=None, residual=None,
          gate2=None, router_x=None) -> dict:
    """The whole MoE FFN layer.

    ``selection`` injects an expert-choice selection (idx[E, n_segments*C]) instead of
    the oracle's own, so that outputs can be compared given the same integer decisions.
    ``shared`` = (Ws1 [d,Fs], Ws3 [d,Fs], Ws2 [Fs,d]) adds a shared SwiGLU expert that
    every token goes through (section 6.2), onto which the routed outputs are added.
    ``residual`` [T,d] (and ``gate2`` [n_segments,d]) add the result to the block's
    residual stream through the gate (section 6.3, :func:`gated_residual`).
    ``router_x`` [T,d], when given, is what the router scores (section 6.2: the gate
    reads the unmodulated hidden states, the experts the block's modulated input x).

    Returns dict(out [T,d] fp64, p fp64 [T,E], scores32 [T,E], idx, w).
    """
    x = _f64(x)
    T, d = x.shape
    E = np.asarray(W_r).shape[1]
    logits = router_logits(x if router_x is None else router_x, W_r, router_bias, n_segments)
    p = scores_from_logits(logits, score_fn)
    s32 = round_f32(p)
    idx = select(s32, C, n_segments) if selection is None else np.asarray(selection)
    w = combine_weights(p, idx, combine, route_scale)
    out = np.zeros((T, d), dtype=F64)
    if shared is not None:
        out += swiglu_ffn(x, *shared)
    # ascending expert order: each token's contributions are added e = 0, 1, ...
    for e in range(E):
        rows = idx[e]
        y = swiglu_ffn(x[rows], W1[e], W3[e], W2[e])
        out[rows] += w[e][:, None] * y  # rows within one expert are distinct
    if residual is not None:
        out = gated_residual(residual, gate2, out, n_segments)
    return dict(out=out, p=p, scores32=s32, idx=idx, w=w)


def layer_rows(x, W_r, W1, W3, W2, C: int, tokens, *, score_fn: str = "softmax",
               combine: str = "raw", route_scale: float = 1.0, n_segments: int = 1,
               router_bias=None, selection=None, shared=None, residual=None,
               gate2=None, router_x=None) -> dict:
    """The layer output for the listed tokens only (for workloads too large to run
    whole). Router, scores and selection still cover every token."""
    x = _f64(x)
    E = np.asarray(W_r).shape[1]
    logits = router_logits(x if router_x is None else router_x, W_r, router_bias, n_segments)
    p = scores_from_logits(logits, score_fn)
    s32 = round_f32(p)
    idx = select(s32, C, n_segments) if selection is None else np.asarray(selection)
    w = combine_weights(p, idx, combine, route_scale)
    tokens = np.asarray(tokens)
    out = np.zeros((len(tokens), x.shape[1]), dtype=F64)
    if shared is not None:
        out += swiglu_ffn(x[tokens], *shared)
    pos = {int(t): i for i, t in enumerate(tokens)}
    for e in range(E):
        hit = [(slot, pos[int(t)]) for slot, t in enumerate(idx[e]) if int(t) in pos]
        if not hit:
            continue
        slots = np.array([h[0] for h in hit])
        where = np.array([h[1] for h in hit])
        y = swiglu_ffn(x[idx[e][slots]], np.asarray(W1[e]), np.asarray(W3[e]),
                       np.asarray(W2[e]))
        out[where] += w[e][slots][:, None] * y
    if residual is not None:
        T = x.shape[0]
        g = np.ones((len(tokens), x.shape[1])) if gate2 is None else \
            np.tanh(np.clip(_f64(gate2), -2.0, 2.0))[tokens // (T // n_segments)]
        out = _f64(residual)[tokens] + g * out
    return dict(out=out, p=p, scores32=s32, idx=idx, w=w)

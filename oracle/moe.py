"""Routed-expert MoE block over a frozen NF4 fused stack with per-expert LoRA.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Plain float64 numpy,
written as a loop over the experts, one at a time, which is how the pages
say the method's own plain forward is built ("How do I QLoRA-train the fused
experts of a MoE", §"Why it happens").

What is computed (same page, §"The abstraction that fails, and what replaces
it" and §"Why it happens"; readings where the pages are silent are marked):

* routing: per token the ``k`` largest float32 router logits, ties to the
  lower expert id, slots ordered by descending logit; routing weights are a
  softmax over those ``k`` logits.  The router is frozen and its logits are
  inputs, so routing is constant in the backward.
* grouping (reading): the slots of expert ``e`` in ascending flat slot index
  ``t*k + j``.
* per routed slot (token t, expert e, weight w), with ``s = alpha / r``:
  ``gu = W_gu[e] x + s B_gu[e] (A_gu[e] x)``; ``g = gu[:I]``,
  ``u = gu[I:]`` (reading: gate rows first, then up rows);
  ``a = silu(g) * u``; ``yd = W_d[e] a + s B_d[e] (A_d[e] a)``;
  ``y[t] += w * yd``.  The LoRA delta enters before the activation.
* backward with upstream ``dY``, base frozen (no base gradient), router
  constant: ``dyw = w dY[t]``; ``da = W_d[e]^T dyw + s A_d[e]^T (B_d[e]^T dyw)``;
  ``dg = da * u * sig(g) * (1 + g (1 - sig(g)))``; ``du = da * silu(g)``;
  ``dx[t] += W_gu[e]^T dgu + s A_gu[e]^T (B_gu[e]^T dgu)``; and the adapter
  gradients ``dB_gu[e] += s dgu (A_gu[e] x)^T``, ``dA_gu[e] += s (B_gu[e]^T dgu) x^T``,
  ``dB_d[e] += s dyw (A_d[e] a)^T``, ``dA_d[e] += s (B_d[e]^T dyw) a^T``.
  The base weights are dequantised again in the backward (§"Why it
  happens": the backward decodes the 4-bit base again).

Pins (tests/test_oracle_moe.py): the adapter layout consumed here (one A/B
pair on the fused gate_up stack, one on down) reproduces the trainable-
parameter counts the pages print for a real model (section "Measured
result"); B = 0 gives exactly the base-only block;
a per-token, per-expert brute-force loop; dense-delta equivalence with
``W + s B A`` materialised; E = 1, k = 1 against torch's SiLU, matmul and
autograd; central finite differences of every gradient; routing against
torch.topk/softmax and a stable library sort.  Router backward (for a trained
router): central finite differences of the block's loss in the logits, torch
autograd through topk + softmax, and the softmax invariants (selected entries
of a row sum to 0, unselected entries exactly 0, k = 1 gives 0).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Iterable, Optional

import numpy as np

from .nf4 import dequantize_nf4_matrix


@dataclass
class Experts:
    """Frozen NF4 stacks plus the per-expert LoRA factors (float64 copies).

    ``gate_up_nf4`` uint8 [E, 2I, H/2], ``gate_up_absmax`` float32
    [E, 2I, H/64], ``down_nf4`` uint8 [E, H, I/2], ``down_absmax`` float32
    [E, H, I/64]; ``A_gu`` [E, r, H], ``B_gu`` [E, 2I, r], ``A_d`` [E, r, I],
    ``B_d`` [E, H, r].
    """

    gate_up_nf4: np.ndarray
    gate_up_absmax: np.ndarray
    down_nf4: np.ndarray
    down_absmax: np.ndarray
    A_gu: np.ndarray
    B_gu: np.ndarray
    A_d: np.ndarray
    B_d: np.ndarray

    @property
    def E(self) -> int:
        return self.gate_up_nf4.shape[0]

    @property
    def H(self) -> int:
        return self.down_nf4.shape[1]

    @property
    def I(self) -> int:  # noqa: E743
        return self.gate_up_nf4.shape[1] // 2

    @property
    def r(self) -> int:
        return self.A_gu.shape[1]


def expert_weights(experts: Experts, e: int):
    """Dequantised base of expert ``e``: (W_gu [2I, H], W_d [H, I]) float64."""
    w_gu = dequantize_nf4_matrix(experts.gate_up_nf4[e], experts.gate_up_absmax[e])
    w_d = dequantize_nf4_matrix(experts.down_nf4[e], experts.down_absmax[e])
    return w_gu, w_d


def route_topk(logits: np.ndarray, k: int):
    """Top-k experts per token and the softmax over the selected logits.

    Returns ``ids`` int32 [T, k] (descending logit, ties to the lower id) and
    ``w`` float64 [T, k].
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # A stable sort of the negated logits keeps equal logits in ascending id order.
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    ids = order.astype(np.int32)
    sel = np.take_along_axis(logits, order, axis=1).astype(np.float64)
    z = np.exp(sel - sel[:, :1])
    w = z / z.sum(axis=1, keepdims=True)
    return ids, w


def group_by_expert(ids: np.ndarray, E: int) -> Dict[str, np.ndarray]:
    """Group the flat slots ``t*k + j`` by expert, stable in slot order.

    Returns ``counts`` [E], ``starts`` [E+1] (exclusive prefix sum),
    ``slots`` [N] (the slots in grouped order) and ``rank`` [N] (the position
    of each slot inside its expert's group).
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    N = flat.shape[0]
    counts = np.zeros(E, dtype=np.int64)
    rank = np.zeros(N, dtype=np.int64)
    for f in range(N):  # one pass in slot order: the running count is the rank
        e = flat[f]
        rank[f] = counts[e]
        counts[e] += 1
    starts = np.zeros(E + 1, dtype=np.int64)
    starts[1:] = np.cumsum(counts)
    slots = np.empty(N, dtype=np.int64)
    slots[starts[flat] + rank] = np.arange(N)
    return {"counts": counts, "starts": starts, "slots": slots, "rank": rank}


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


def expert_forward(X, w_gu, w_d, A_gu, B_gu, A_d, B_d, s):
    """One expert on the rows ``X`` [n, H]; returns the intermediates."""
    I = w_d.shape[1]
    p_gu = X @ A_gu.T                       # A_gu x        [n, r]
    gu = X @ w_gu.T + s * (p_gu @ B_gu.T)   # pre-activation [n, 2I]
    g, u = gu[:, :I], gu[:, I:]
    a = _silu(g) * u                        # act(gate) * up
    p_d = a @ A_d.T                         # A_d a          [n, r]
    yd = a @ w_d.T + s * (p_d @ B_d.T)      # expert output  [n, H]
    return {"p_gu": p_gu, "gu": gu, "act": a, "p_d": p_d, "yd": yd}


def expert_backward(X, dyw, fwd, w_gu, w_d, A_gu, B_gu, A_d, B_d, s):
    """Backward of one expert for upstream ``dyw`` [n, H] (already weighted)."""
    I = w_d.shape[1]
    g, u = fwd["gu"][:, :I], fwd["gu"][:, I:]
    a = fwd["act"]
    q_d = dyw @ B_d                          # B_d^T dyw      [n, r]
    da = dyw @ w_d + s * (q_d @ A_d)         # d act          [n, I]
    sg = _sigmoid(g)
    dg = da * u * sg * (1.0 + g * (1.0 - sg))
    du = da * _silu(g)
    dgu = np.concatenate([dg, du], axis=1)   # [n, 2I]
    q_gu = dgu @ B_gu                        # B_gu^T dgu     [n, r]
    dX = dgu @ w_gu + s * (q_gu @ A_gu)      # [n, H]
    return {
        "q_d": q_d,
        "dact": da,
        "dgu": dgu,
        "q_gu": q_gu,
        "dX": dX,
        "dB_gu": s * dgu.T @ fwd["p_gu"],    # [2I, r]
        "dA_gu": s * q_gu.T @ X,             # [r, H]
        "dB_d": s * dyw.T @ fwd["p_d"],      # [H, r]
        "dA_d": s * q_d.T @ a,               # [r, I]
    }


def _lora(experts: Experts, e: int):
    f = lambda z: np.asarray(z[e], dtype=np.float64)  # noqa: E731
    return f(experts.A_gu), f(experts.B_gu), f(experts.A_d), f(experts.B_d)


def moe_forward(x, logits, experts: Experts, k: int, alpha: float,
                tokens: Optional[Iterable[int]] = None):
    """Forward of the block.  ``x`` [T, H] (values), ``logits`` [T, E] float32.

    With ``tokens`` given, only those tokens' outputs are computed (every
    expert a selected token is routed to).  Returns a dict with ``ids``,
    ``w``, ``y`` [T, H] (rows of unselected tokens are zero) and, keyed by
    flat slot, the per-slot intermediates ``gu``, ``act``, ``p_gu``, ``p_d``,
    ``yd``.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    s = float(alpha) / experts.r
    ids, w = route_topk(logits, k)
    flat = ids.reshape(-1)
    want = np.ones(T, dtype=bool)
    if tokens is not None:
        want[:] = False
        want[np.asarray(list(tokens), dtype=np.int64)] = True
    y = np.zeros((T, H), dtype=np.float64)
    per_slot = {"gu": {}, "act": {}, "p_gu": {}, "p_d": {}, "yd": {}}
    for e in range(experts.E):
        slots = np.flatnonzero((flat == e) & want[np.arange(flat.size) // k])
        if slots.size == 0:
            continue
        w_gu, w_d = expert_weights(experts, e)
        res = expert_forward(x[slots // k], w_gu, w_d, *_lora(experts, e), s)
        for i, f in enumerate(slots):
            t, j = divmod(int(f), k)
            y[t] += w[t, j] * res["yd"][i]
            for key in per_slot:
                per_slot[key][int(f)] = res[key][i]
    out = {"ids": ids, "w": w, "y": y}
    out.update(per_slot)
    return out


def moe_backward(x, logits, dY, experts: Experts, k: int, alpha: float,
                 tokens: Optional[Iterable[int]] = None,
                 grad_experts: Optional[Iterable[int]] = None):
    """Backward of the block for upstream ``dY`` [T, H].

    ``dx`` is computed for ``tokens`` (all when None); the adapter gradients
    ``dA_gu`` [E, r, H], ``dB_gu`` [E, 2I, r], ``dA_d`` [E, r, I],
    ``dB_d`` [E, H, r] for ``grad_experts`` (all when None), each summed over
    every token routed to that expert.  Experts with no tokens get exactly
    zero gradients.  Per-slot ``dgu``, ``q_gu``, ``q_d``, ``dx_slot`` are
    returned keyed by flat slot for the slots that were evaluated.
    """
    x = np.asarray(x, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    T, H = x.shape
    E, I, r = experts.E, experts.I, experts.r
    s = float(alpha) / r
    ids, w = route_topk(logits, k)
    flat = ids.reshape(-1)
    tok_of = np.arange(flat.size) // k
    want_tok = np.ones(T, dtype=bool)
    if tokens is not None:
        want_tok[:] = False
        want_tok[np.asarray(list(tokens), dtype=np.int64)] = True
    want_exp = np.ones(E, dtype=bool)
    if grad_experts is not None:
        want_exp[:] = False
        want_exp[np.asarray(list(grad_experts), dtype=np.int64)] = True
    dx = np.zeros((T, H))
    grads = {
        "dA_gu": np.zeros((E, r, H)), "dB_gu": np.zeros((E, 2 * I, r)),
        "dA_d": np.zeros((E, r, I)), "dB_d": np.zeros((E, H, r)),
    }
    per_slot = {"dgu": {}, "q_gu": {}, "q_d": {}, "dx_slot": {}}
    for e in range(E):
        sel = flat == e
        if not want_exp[e]:
            sel &= want_tok[tok_of]
        slots = np.flatnonzero(sel)
        if slots.size == 0:
            continue
        # The base is dequantised again here, as in the method's backward.
        w_gu, w_d = expert_weights(experts, e)
        lora = _lora(experts, e)
        X = x[slots // k]
        fwd = expert_forward(X, w_gu, w_d, *lora, s)
        wj = w[slots // k, slots % k]
        dyw = wj[:, None] * dY[slots // k]
        res = expert_backward(X, dyw, fwd, w_gu, w_d, *lora, s)
        for i, f in enumerate(slots):
            t = int(f) // k
            if want_tok[t]:
                dx[t] += res["dX"][i]
            per_slot["dgu"][int(f)] = res["dgu"][i]
            per_slot["q_gu"][int(f)] = res["q_gu"][i]
            per_slot["q_d"][int(f)] = res["q_d"][i]
            per_slot["dx_slot"][int(f)] = res["dX"][i]
        if want_exp[e]:
            for key in grads:
                grads[key][e] = res[key]
    out = {"ids": ids, "w": w, "dx": dx}
    out.update(grads)
    out.update(per_slot)
    return out


def topk_softmax_backward(logits, k: int, dY, yd, tokens: Optional[Iterable[int]] = None):
    """Router-logit gradient from the per-slot expert outputs ``yd``.

    ``yd`` is indexed by flat slot ``t * k + j`` (an array [T*k, H] or a
    mapping); ``ids`` and ``w`` are the top-k routing of ``logits``.  The
    steps are the two of :func:`router_backward`: ``dw[t, j] = <dY[t],
    yd[t*k + j]>``, then the softmax-over-top-k backward.  Only the rows in
    ``tokens`` (every row when None) are computed; the others stay zero.
    """
    ids, w = route_topk(logits, k)
    dY = np.asarray(dY, dtype=np.float64)
    T = dY.shape[0]
    E = np.asarray(logits).shape[1]
    rows = range(T) if tokens is None else sorted(set(int(t) for t in tokens))
    d_logits = np.zeros((T, E), dtype=np.float64)
    dw = np.zeros((T, k), dtype=np.float64)
    for t in rows:
        for j in range(k):
            dw[t, j] = float(np.dot(dY[t], np.asarray(yd[t * k + j], dtype=np.float64)))
        d_logits[t, ids[t]] = w[t] * (dw[t] - float(np.dot(w[t], dw[t])))
    return {"d_logits": d_logits, "dw": dw, "ids": ids, "w": w}


def router_backward(x, logits, dY, experts: Experts, k: int, alpha: float,
                    tokens: Optional[Iterable[int]] = None):
    """Gradient of the loss with respect to the router logits, for a trained router.

    The router is frozen by default; with it trained ("How do I QLoRA-train
    the fused experts of a MoE", section "The abstraction that fails, and what
    replaces it": ``TRAIN_ROUTER=1``), the logits receive a gradient through
    the routing weights only -- the top-k selection is piecewise constant.
    With ``yd[t, j]`` the output of the j-th selected expert for token t
    (before weighting) and upstream ``dY``:

    * ``dw[t, j] = <dY[t], yd[t, j]>`` (since ``y[t] = sum_j w[t, j] yd[t, j]``);
    * softmax over the k selected logits:
      ``dlogits[t, ids[t, j]] = w[t, j] * (dw[t, j] - sum_i w[t, i] dw[t, i])``;
    * every unselected expert's logit gets exactly 0.

    Returns ``d_logits`` [T, E] float64 (rows of unselected tokens zero) and
    ``dw`` [T, k].
    """
    fwd = moe_forward(x, logits, experts, k, alpha, tokens=tokens)
    return topk_softmax_backward(logits, k, dY, fwd["yd"], tokens=tokens)

"""Pins of the oracle's routing, grouping, forward and backward (CPU only)."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from grouped_nf4_expert_b200 import inputs


def _experts(prob, lora_dtype=np.float64):
    f = lambda b: inputs.bits_to_f32(b).astype(lora_dtype)  # noqa: E731
    return oracle.Experts(prob.gate_up_nf4, prob.gate_up_absmax, prob.down_nf4,
                          prob.down_absmax, f(prob.A_gu), f(prob.B_gu), f(prob.A_d), f(prob.B_d))


@pytest.fixture(scope="module")
def tiny():
    prob = inputs.make_problem(inputs.CONFIGS["tiny"])
    return prob, _experts(prob), inputs.bits_to_f32(prob.x).astype(np.float64)


# ---------------------------------------------------------------- routing

def test_route_matches_torch_topk_softmax():
    rng = np.random.default_rng(0)
    logits = rng.standard_normal((500, 37)).astype(np.float32)
    ids, w = oracle.route_topk(logits, 5)
    tl = torch.from_numpy(logits)
    vals, idx = torch.topk(tl, 5, dim=1, sorted=True)
    assert np.array_equal(ids, idx.numpy().astype(np.int32))
    ref = torch.softmax(vals.double(), dim=1).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-14, atol=0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)


def test_route_ties_go_to_lower_id_and_order_is_descending():
    logits = np.array([[0.5, 2.0, 2.0, -1.0, 2.0],
                       [0.0, 0.0, 0.0, 0.0, 0.0],
                       [-0.0, 0.0, 1.0, -3.0, 0.0]], dtype=np.float32)
    ids, w = oracle.route_topk(logits, 3)
    assert ids.tolist() == [[1, 2, 4], [0, 1, 2], [2, 0, 1]]
    np.testing.assert_allclose(w[1], [1 / 3] * 3, rtol=1e-15)


def test_route_rejects_bad_k():
    with pytest.raises(ValueError):
        oracle.route_topk(np.zeros((2, 3), np.float32), 4)


def test_grouping_is_a_stable_sort():
    rng = np.random.default_rng(1)
    ids = rng.integers(0, 9, (300, 3)).astype(np.int32)
    ids[:, 1] = (ids[:, 0] + 1) % 9  # distinct within a token like real routing
    g = oracle.group_by_expert(ids, 10)
    flat = ids.reshape(-1)
    ref = np.argsort(flat, kind="stable")
    assert np.array_equal(g["slots"], ref)
    assert np.array_equal(g["counts"], np.bincount(flat, minlength=10))
    assert g["counts"][9] == 0 and g["starts"][-1] == flat.size
    assert np.array_equal(np.sort(g["slots"]), np.arange(flat.size))
    for f in range(flat.size):
        assert g["slots"][g["starts"][flat[f]] + g["rank"][f]] == f


# ---------------------------------------------------------------- forward pins

def test_b_zero_gives_base_block_exactly():
    prob = inputs.make_problem(inputs.CONFIGS["tiny_b0"])
    ex = _experts(prob)
    base = oracle.Experts(ex.gate_up_nf4, ex.gate_up_absmax, ex.down_nf4, ex.down_absmax,
                          np.zeros_like(ex.A_gu), ex.B_gu, np.zeros_like(ex.A_d), ex.B_d)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    a = oracle.moe_forward(x, prob.logits, ex, 2, 16.0)
    b = oracle.moe_forward(x, prob.logits, base, 2, 16.0)
    assert np.any(ex.A_gu != 0)
    assert np.array_equal(a["y"], b["y"])


def _silu(v):
    return v / (1 + np.exp(-v))


def test_bruteforce_per_token_per_expert_loop(tiny):
    prob, ex, x = tiny
    cfg = prob.cfg
    s = cfg.alpha / cfg.r
    out = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha)
    # Independent brute force: every token against every expert, a dense
    # gate over all E with zeros outside the top-k, matrix-vector products.
    T, E, I = cfg.T, cfg.E, cfg.I
    W = [oracle.expert_weights(ex, e) for e in range(E)]
    y = np.zeros((T, cfg.H))
    for t in range(T):
        lg = prob.logits[t].astype(np.float64)
        top = sorted(range(E), key=lambda e: (-prob.logits[t, e], e))[: cfg.top_k]
        z = np.array([np.exp(lg[e] - lg[top[0]]) for e in top])
        gate = np.zeros(E)
        gate[top] = z / z.sum()
        for e in range(E):
            wgu, wd = W[e]
            hv = wgu.dot(x[t]) + s * ex.B_gu[e].dot(ex.A_gu[e].dot(x[t]))
            av = _silu(hv[:I]) * hv[I:]
            yv = wd.dot(av) + s * ex.B_d[e].dot(ex.A_d[e].dot(av))
            y[t] += gate[e] * yv
    np.testing.assert_allclose(out["y"], y, rtol=1e-11, atol=1e-13)


def test_dense_delta_equivalence_with_torch(tiny):
    prob, ex, x = tiny
    cfg = prob.cfg
    s = cfg.alpha / cfg.r
    out = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha)
    ids, w = out["ids"], out["w"]
    xt = torch.from_numpy(x)
    y = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for e in range(cfg.E):
        wgu, wd = (torch.from_numpy(m) for m in oracle.expert_weights(ex, e))
        wgu = wgu + s * torch.from_numpy(ex.B_gu[e]) @ torch.from_numpy(ex.A_gu[e])
        wd = wd + s * torch.from_numpy(ex.B_d[e]) @ torch.from_numpy(ex.A_d[e])
        h = F.linear(xt, wgu)
        yd = F.linear(F.silu(h[:, : cfg.I]) * h[:, cfg.I:], wd)
        gate = torch.from_numpy(((ids == e) * w).sum(1))
        y += gate[:, None] * yd
    np.testing.assert_allclose(out["y"], y.numpy(), rtol=1e-10, atol=1e-12)


def test_token_subset_matches_full(tiny):
    prob, ex, x = tiny
    full = oracle.moe_forward(x, prob.logits, ex, 2, 16.0)
    sub = oracle.moe_forward(x, prob.logits, ex, 2, 16.0, tokens=[3, 17, 30])
    np.testing.assert_allclose(sub["y"][[3, 17, 30]], full["y"][[3, 17, 30]], rtol=1e-12, atol=1e-15)
    assert np.all(sub["y"][0] == 0)


# ---------------------------------------------------------------- backward pins

def _dense_torch_block(x, ex, s, I):
    """E = 1, k = 1: the block is a dense SwiGLU MLP with LoRA on both projections."""
    wgu, wd = (torch.from_numpy(m) for m in oracle.expert_weights(ex, 0))
    X = torch.from_numpy(x).requires_grad_(True)
    A_gu = torch.from_numpy(ex.A_gu[0].copy()).requires_grad_(True)
    B_gu = torch.from_numpy(ex.B_gu[0].copy()).requires_grad_(True)
    A_d = torch.from_numpy(ex.A_d[0].copy()).requires_grad_(True)
    B_d = torch.from_numpy(ex.B_d[0].copy()).requires_grad_(True)
    h = F.linear(X, wgu) + s * F.linear(F.linear(X, A_gu), B_gu)
    a = F.silu(h[:, :I]) * h[:, I:]
    y = F.linear(a, wd) + s * F.linear(F.linear(a, A_d), B_d)
    return y, (X, A_gu, B_gu, A_d, B_d)


def test_single_expert_reduces_to_dense_swiglu_mlp_with_torch_autograd():
    cfg = inputs.Config("e1k1", E=1, H=64, I=128, top_k=1, T=24, r=8, alpha=16.0,
                        routing="normal", seed=21)
    prob = inputs.make_problem(cfg)
    ex = _experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    s = cfg.alpha / cfg.r
    y, leaves = _dense_torch_block(x, ex, s, cfg.I)
    (y * torch.from_numpy(dY)).sum().backward()
    fo = oracle.moe_forward(x, prob.logits, ex, 1, cfg.alpha)
    bo = oracle.moe_backward(x, prob.logits, dY, ex, 1, cfg.alpha)
    np.testing.assert_allclose(fo["y"], y.detach().numpy(), rtol=1e-11, atol=1e-13)
    X, A_gu, B_gu, A_d, B_d = leaves
    for mine, ref in [(bo["dx"], X.grad), (bo["dA_gu"][0], A_gu.grad), (bo["dB_gu"][0], B_gu.grad),
                      (bo["dA_d"][0], A_d.grad), (bo["dB_d"][0], B_d.grad)]:
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-13)


def _loss(x, logits, dY, ex, k, alpha):
    return float(np.sum(oracle.moe_forward(x, logits, ex, k, alpha)["y"] * dY))


def test_finite_differences_all_gradients(tiny):
    prob, ex, x = tiny
    cfg = prob.cfg
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    bo = oracle.moe_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha)
    rng = np.random.default_rng(7)
    eps = 1e-4

    def check(name, grad, perturb):
        v = rng.standard_normal(grad.shape)
        v /= np.linalg.norm(v)  # unit direction: truncation error O(eps^2)
        lp = perturb(eps * v)
        lm = perturb(-eps * v)
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(grad * v))
        assert np.linalg.norm(grad) > 1e-3, name
        assert abs(fd - an) <= 1e-7 * np.linalg.norm(grad), (name, fd, an)

    def with_lora(key, dv):
        kw = {f: getattr(ex, f) for f in ("gate_up_nf4", "gate_up_absmax", "down_nf4", "down_absmax",
                                          "A_gu", "B_gu", "A_d", "B_d")}
        kw[key] = kw[key] + dv
        return _loss(x, prob.logits, dY, oracle.Experts(**kw), cfg.top_k, cfg.alpha)

    check("dx", bo["dx"], lambda dv: _loss(x + dv, prob.logits, dY, ex, cfg.top_k, cfg.alpha))
    check("dA_gu", bo["dA_gu"], lambda dv: with_lora("A_gu", dv))
    check("dB_gu", bo["dB_gu"], lambda dv: with_lora("B_gu", dv))
    check("dA_d", bo["dA_d"], lambda dv: with_lora("A_d", dv))
    check("dB_d", bo["dB_d"], lambda dv: with_lora("B_d", dv))
    # and a few single coordinates of dx
    for (t, h) in [(0, 0), (5, 33), (31, 63)]:
        d = np.zeros_like(x)
        d[t, h] = eps
        fd = (_loss(x + d, prob.logits, dY, ex, 2, 16.0) - _loss(x - d, prob.logits, dY, ex, 2, 16.0)) / (2 * eps)
        assert abs(fd - bo["dx"][t, h]) <= 1e-6 * max(1.0, abs(fd))


def test_b_zero_gives_zero_dA_and_empty_expert_zero_grads():
    prob = inputs.make_problem(inputs.CONFIGS["tiny_b0"])
    ex = _experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    logits = prob.logits.copy()
    logits[:, 3] = -1e30  # expert 3 never routed
    bo = oracle.moe_backward(x, logits, dY, ex, 2, 16.0)
    assert np.all(bo["dA_gu"] == 0) and np.all(bo["dA_d"] == 0)
    assert np.any(bo["dB_gu"][0] != 0) and np.any(bo["dB_d"][0] != 0)
    for key in ("dB_gu", "dB_d"):
        assert np.all(bo[key][3] == 0)


def test_backward_subsets_match_full(tiny):
    prob, ex, x = tiny
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    full = oracle.moe_backward(x, prob.logits, dY, ex, 2, 16.0)
    sub = oracle.moe_backward(x, prob.logits, dY, ex, 2, 16.0, tokens=[1, 2], grad_experts=[2])
    np.testing.assert_allclose(sub["dx"][[1, 2]], full["dx"][[1, 2]], rtol=1e-12, atol=1e-15)
    for key in ("dA_gu", "dB_gu", "dA_d", "dB_d"):
        np.testing.assert_allclose(sub[key][2], full[key][2], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- router backward

def test_router_backward_finite_differences(tiny):
    # d/d(logits) of L = sum_t <dY_t, y_t> against central differences of the
    # forward: the selected logits move the softmax weights; an unselected
    # logit moved by less than its distance to the k-th selected one changes nothing.
    prob, ex, x = tiny
    cfg = prob.cfg
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    rb = oracle.router_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha)
    lg = np.asarray(prob.logits, dtype=np.float32)
    srt = np.sort(lg, axis=1)[:, ::-1]
    gap = srt[:, cfg.top_k - 1] - srt[:, cfg.top_k]
    eps = np.float32(2.0 ** -10)
    checked = 0
    for t in np.flatnonzero(gap > 64 * eps)[:6]:
        for e in range(cfg.E):
            lp, lm = lg.copy(), lg.copy()
            lp[t, e] = lg[t, e] + eps
            lm[t, e] = lg[t, e] - eps
            h = float(lp[t, e]) - float(lm[t, e])  # the representable float32 step
            fd = (_loss(x, lp, dY, ex, cfg.top_k, cfg.alpha) - _loss(x, lm, dY, ex, cfg.top_k, cfg.alpha)) / h
            an = rb["d_logits"][t, e]
            assert abs(fd - an) <= 1e-4 * max(1.0, np.abs(rb["d_logits"][t]).max()), (t, e, fd, an)
            checked += 1
    assert checked >= 4 * cfg.E
    assert np.abs(rb["d_logits"]).max() > 1e-3


def test_router_backward_invariants(tiny):
    prob, ex, x = tiny
    cfg = prob.cfg
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    rb = oracle.router_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha)
    dl, ids = rb["d_logits"], rb["ids"]
    # softmax shift invariance: the selected entries of a row sum to zero
    assert np.allclose(dl.sum(axis=1), 0.0, atol=1e-12 * max(1.0, np.abs(dl).max()))
    # unselected experts get exact zeros
    mask = np.zeros_like(dl, dtype=bool)
    np.put_along_axis(mask, ids.astype(np.int64), True, axis=1)
    assert np.all(dl[~mask] == 0.0)
    # dw is the plain dot product of dY with each selected expert's output
    fwd = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha)
    t, j = 3, 1
    assert rb["dw"][t, j] == float(np.dot(dY[t], fwd["yd"][t * cfg.top_k + j]))
    # one expert per token: the routing weight is constant 1, no gradient
    rb1 = oracle.router_backward(x, prob.logits, dY, ex, 1, cfg.alpha)
    assert np.all(rb1["d_logits"] == 0.0)
    # token subsets agree with the full computation
    sub = oracle.router_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha, tokens=[0, 7, 19])
    assert np.allclose(sub["d_logits"][[0, 7, 19]], dl[[0, 7, 19]], rtol=1e-12, atol=0)  # BLAS blocking only
    assert np.all(sub["d_logits"][1] == 0.0)



def test_topk_softmax_backward_against_torch_autograd():
    # The same gradient from torch's own topk + softmax + autograd (float64),
    # for arbitrary per-slot outputs yd: L = sum_t sum_j w_tj <dY_t, yd_tj>.
    rng = np.random.default_rng(11)
    T, E, k, H = 24, 12, 4, 40
    logits = rng.standard_normal((T, E)).astype(np.float32)
    dY = rng.standard_normal((T, H))
    yd = rng.standard_normal((T * k, H))
    got = oracle.topk_softmax_backward(logits, k, dY, yd)
    lt = torch.tensor(logits, dtype=torch.float64, requires_grad=True)
    vals, idx = torch.topk(lt, k, dim=1)
    w = torch.softmax(vals, dim=1)
    dw = (torch.tensor(dY)[:, None, :] * torch.tensor(yd).view(T, k, H)).sum(-1)
    (w * dw).sum().backward()
    assert np.array_equal(got["ids"], idx.numpy())
    assert np.allclose(got["d_logits"], lt.grad.numpy(), rtol=1e-12, atol=1e-13)
    assert np.allclose(got["dw"], dw.detach().numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- adapter layout (printed counts)

def _golden_ints(name):
    from conftest import golden_path
    out = {}
    for line in open(golden_path(name)):
        line = line.strip()
        if line and not line.startswith("#"):
            key, val = line.split()
            out[key] = int(val)
    return out


def test_adapter_layout_matches_the_printed_trainable_parameter_counts():
    # The pages print the trainable-parameter count of the per-expert adapter on a real model. The
    # oracle's layout -- one A/B pair on the fused gate_up stack (A_gu [r, H], B_gu [2I, r]) and one on
    # down (A_d [r, I], B_d [H, r]) -- must reproduce it; the oracle is run on those shapes so that
    # the count is of the arrays it consumes.
    g = _golden_ints("granite_trainable_params.txt")
    r, L, H, I, E = g["rank"], g["layers"], g["hidden"], g["intermediate"], g["experts"]
    q_out, kv_out = g["heads"] * g["head_dim"], g["kv_heads"] * g["head_dim"]
    attention = L * r * ((H + q_out) + 2 * (H + kv_out) + (q_out + H))  # q, k, v, o
    assert attention == g["attention_only"]
    cfg = inputs.Config("granite_layer", E=E, H=H, I=I, top_k=8, T=2, r=r, alpha=16.0, routing="normal", seed=7)
    prob = inputs.make_problem(cfg)
    ex = _experts(prob)
    out = oracle.moe_forward(inputs.bits_to_f32(prob.x).astype(np.float64), prob.logits, ex, cfg.top_k,
                             cfg.alpha, tokens=[0])
    assert np.isfinite(out["y"][0]).all()
    per_layer = ex.A_gu.size + ex.B_gu.size + ex.A_d.size + ex.B_d.size
    assert attention + L * per_layer == g["attention_and_experts"]
    # layouts the count rules out: adapter on gate_up alone; separate gate and up adapters
    assert attention + L * E * r * (H + 2 * I) != g["attention_and_experts"]
    assert attention + L * E * r * (2 * (H + I) + (I + H)) != g["attention_and_experts"]

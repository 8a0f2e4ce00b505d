"""The seeded input generator follows the recipe the design states (CPU only).

Checked on the generator's own output, against the distributions it claims:
Gumbel-top-k logits sample experts with Zipf(s) popularity, block absmax is
distributed as the maximum |w| of 64 normal weights, NF4 codes are uniform,
activations and LoRA factors have the stated scales, a data-parallel rank gets
its own batch over the same weights, and everything is reproducible.
"""

import numpy as np
from scipy import stats

from grouped_nf4_expert_b200 import inputs

ZIPF = inputs.Config("zipf16", E=16, H=64, I=64, top_k=2, T=200_000, r=8, alpha=16.0, routing="zipf", seed=21)


def test_zipf_logits_pick_the_first_expert_with_zipf_probabilities():
    # argmax of log p + Gumbel noise is a draw from p (the Gumbel-max property); the popularity order
    # is a fixed permutation of the experts
    lg = inputs.router_logits(ZIPF)
    first = np.argmax(lg, axis=1)
    freq = np.bincount(first, minlength=ZIPF.E) / len(first)
    p_sorted = np.arange(1, ZIPF.E + 1, dtype=np.float64) ** -ZIPF.zipf_s
    p_sorted /= p_sorted.sum()
    np.testing.assert_allclose(np.sort(freq)[::-1], p_sorted, atol=4 * np.sqrt(p_sorted[0] / len(first)))
    # not the identity order: the most popular expert is wherever the seeded permutation put it
    assert list(np.argsort(-freq)) != list(range(ZIPF.E))


def test_normal_logits_spread_the_load_evenly():
    cfg = inputs.Config("even", E=16, H=64, I=64, top_k=4, T=50_000, r=8, alpha=16.0, routing="normal", seed=22)
    lg = inputs.router_logits(cfg)
    ids = np.argsort(-lg, axis=1)[:, :cfg.top_k]
    share = np.bincount(ids.ravel(), minlength=cfg.E) / ids.size
    np.testing.assert_allclose(share, 1.0 / cfg.E, atol=0.004)


def test_block_absmax_is_the_max_of_64_normal_magnitudes():
    cfg = inputs.Config("w", E=4, H=4096, I=64, top_k=1, T=1, r=8, alpha=16.0, routing="normal", seed=23)
    prob = inputs.make_problem(cfg)
    got = prob.gate_up_absmax.ravel().astype(np.float64) / cfg.sigma_w
    # CDF of max |N(0,1)| over 64 draws: (2 Phi(m) - 1)^64
    cdf = lambda m: (2.0 * stats.norm.cdf(m) - 1.0) ** 64  # noqa: E731
    assert stats.kstest(got, cdf).pvalue > 1e-3


def test_nf4_codes_are_uniform_over_the_16_levels():
    cfg = inputs.Config("c", E=2, H=2048, I=256, top_k=1, T=1, r=8, alpha=16.0, routing="normal", seed=24)
    prob = inputs.make_problem(cfg)
    b = prob.gate_up_nf4.ravel()
    for codes in (b >> 4, b & 15):
        counts = np.bincount(codes, minlength=16)
        assert stats.chisquare(counts).pvalue > 1e-3


def test_activation_and_adapter_scales():
    cfg = inputs.Config("s", E=4, H=512, I=256, top_k=2, T=2000, r=16, alpha=32.0, routing="normal", seed=25)
    prob = inputs.make_problem(cfg)
    f = inputs.bits_to_f32
    for name, arr, std in [("x", prob.x, 1.0), ("dY", prob.dY, 1.0), ("A_gu", prob.A_gu, 1 / np.sqrt(cfg.H)),
                           ("A_d", prob.A_d, 1 / np.sqrt(cfg.I)), ("B_gu", prob.B_gu, 0.01),
                           ("B_d", prob.B_d, 0.01)]:
        v = f(arr).astype(np.float64).ravel()
        assert abs(v.mean()) < 5 * std / np.sqrt(v.size), name
        assert abs(v.std() / std - 1) < 0.02, name
    b0 = inputs.make_problem(inputs.CONFIGS["tiny_b0"])
    assert not b0.B_gu.any() and not b0.B_d.any()


def test_ranks_draw_their_own_batch_over_the_same_weights_reproducibly():
    cfg = inputs.CONFIGS["tiny"]
    a, a2, b = inputs.make_problem(cfg), inputs.make_problem(cfg), inputs.make_problem(cfg, data_rank=1)
    for name in ("x", "logits", "dY", "gate_up_nf4", "gate_up_absmax", "down_nf4", "down_absmax", "A_gu", "B_gu",
                 "A_d", "B_d"):
        assert np.array_equal(getattr(a, name), getattr(a2, name)), name
    for name in ("x", "logits", "dY"):
        assert not np.array_equal(getattr(a, name), getattr(b, name)), name
    for name in ("gate_up_nf4", "gate_up_absmax", "down_nf4", "down_absmax", "A_gu", "B_gu", "A_d", "B_d"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name

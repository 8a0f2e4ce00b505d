"""The algorithmic work counts bench.py divides by (the roofline numerators), checked against
operation-by-operation tallies of the block on small shapes."""

import importlib.util
import os

from grouped_nf4_expert_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)

CFG = inputs.Config("count", E=4, H=64, I=192, top_k=2, T=5, r=8, alpha=16.0, routing="normal", seed=1)


def _matmuls():
    """Every matrix product of one training step as (rows, reduction, cols), per routed slot."""
    H, I, r = CFG.H, CFG.I, CFG.r
    fwd = [(1, H, 2 * I), (1, H, r), (1, r, 2 * I),      # W_gu x, A_gu x, B_gu p
           (1, I, H), (1, I, r), (1, r, H)]              # W_d act, A_d act, B_d p
    dgrad = [(1, H, I), (1, H, r), (1, r, I),            # W_d^T dyw, B_d^T dyw, A_d^T q
             (1, 2 * I, H), (1, 2 * I, r), (1, r, H)]    # W_gu^T dgu, B_gu^T dgu, A_gu^T q
    wgrad = [(2 * I, 1, r), (r, 1, H), (H, 1, r), (r, 1, I)]  # outer products summed over slots
    return fwd, dgrad, wgrad


def test_step_flops_is_the_sum_of_the_step_matmuls():
    fwd, dgrad, wgrad = _matmuls()
    macs = sum(a * b * c for a, b, c in fwd + dgrad + wgrad) * CFG.N
    assert bench.step_flops(CFG) == 2 * macs
    assert bench.fwd_flops(CFG) == 2 * CFG.N * sum(a * b * c for a, b, c in fwd)


def test_gemm_flops_cover_the_base_products_and_their_k_r_terms():
    H, I, r, N = CFG.H, CFG.I, CFG.r, CFG.N
    g = bench.nf4_gemm_flops(CFG)
    assert g["nf4_gemm_fwd_gate_up"] == 2 * N * (H * 2 * I + r * 2 * I)
    assert g["nf4_gemm_fwd_down"] == 2 * N * (I * H + r * H)
    assert g["nf4_gemm_dgrad_down"] == 2 * N * (H * I + r * I)
    assert g["nf4_gemm_dgrad_gate_up"] == 2 * N * (2 * I * H + r * H)
    # the four launches hold every base product of the step
    assert sum(g.values()) - 2 * N * r * (2 * I + H + I + H) == 2 * N * 6 * H * I


def test_stream_bytes_are_codes_and_scales_of_touched_experts():
    H, I = CFG.H, CFG.I
    for touched in (1, 3):
        b = bench.stream_bytes(CFG, touched)
        assert b["nf4_stream_fwd_gate_up"] == touched * (2 * I * H // 2 + 2 * I * (H // 64) * 4)
        assert b["nf4_stream_fwd_down"] == touched * (H * I // 2 + H * (I // 64) * 4)


def test_router_backward_and_quantiser_bytes():
    T, k, H, E = CFG.T, CFG.top_k, CFG.H, CFG.E
    per_token = k * H * 2 + H * 2 + k * (4 + 4 + 4) + E * 4  # k rows, dY row, ids/weights/rows, d(logits) row
    assert bench.router_bwd_bytes(CFG) == T * per_token
    n = 128  # two blocks
    assert bench.quantize_bytes(n) == n * 2 + n // 2 + 2 * 4

"""The algorithmic work counts bench.py divides by (the roofline numerators), checked against
operation-by-operation tallies of the block on small shapes; and the reference arm's JSON line."""

import importlib.util
import os

from grouped_nf4_expert_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)

CFG = inputs.Config("count", E=4, H=64, I=192, top_k=2, T=5, r=8, alpha=16.0, routing="normal", seed=1,
                    passes=("fwd", "dgrad", "wgrad"))


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
    # workloads without some passes count only the passes they run
    import dataclasses
    fd = dataclasses.replace(CFG, passes=("fwd", "dgrad"))
    assert bench.step_flops(fd) == 2 * CFG.N * sum(a * b * c for a, b, c in fwd + dgrad)
    assert bench.step_flops(dataclasses.replace(CFG, passes=("fwd",))) == bench.fwd_flops(CFG)


def test_gemm_flop_total_counts_only_the_launched_modes():
    g = bench.nf4_gemm_flops(CFG)
    kern = {"nf4_gemm_fwd_gate_up": (3, 1.0), "nf4_gemm_fwd_down": (3, 1.0), "combine_y": (3, 1.0)}
    assert bench.nf4_gemm_flop_total(g, kern) == 3 * (g["nf4_gemm_fwd_gate_up"] + g["nf4_gemm_fwd_down"])
    kern.update({"nf4_gemm_dgrad_down": (3, 1.0), "nf4_gemm_dgrad_gate_up": (3, 1.0)})
    assert bench.nf4_gemm_flop_total(g, kern) == 3 * sum(g.values())


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


def _run_bench(extra_env, *args):
    import json
    import subprocess
    import sys
    env = dict(os.environ, **extra_env)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env, cwd=ROOT,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_one_contract_line_on_rank_0_only():
    args = ("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1")
    (line,) = _run_bench({"RANK": "0"}, *args)
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    for key in ("metric", "value", "n_gpus", "steps", "warmup", "ms_per_step", "scaling", "vs_baseline", "dtype",
                "data", "config"):
        assert key in line, key
    assert line["steps"] == 2 and line["warmup"] == 1 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "workload" in line["config"]
    assert _run_bench({"RANK": "1"}, *args) == []   # other ranks exit 0 without work

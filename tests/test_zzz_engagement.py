"""Engagement: each call runs exactly the kernels its design names (GPU).

The pages ask for the fast path's engagement to be asserted, not just its
results: here the library's own launch record (the per-kernel profiler and the
launch counter) shows, per call, which kernels ran and how often -- the grouped
tensor-core GEMMs for training-sized batches, the weight-streaming kernels for
decode-sized ones, the fused row gathers, and the serving call of a decode-sized
batch: routing plus one persistent launch for everything else.
Collected after the parity tests.
"""

import pytest

import test_gpu_parity as gp
from grouped_nf4_expert_b200 import build, e4b, inputs
from grouped_nf4_expert_b200 import device as dv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    e4b.lib()


def _launched(call):
    """{kernel name: launches} of the library kernels `call` launches."""
    e4b.e4b_profiler_read()  # drop anything recorded before
    n0 = e4b.e4b_launch_count()
    e4b.e4b_profiler_enable(True)
    try:
        call()
    finally:
        e4b.e4b_profiler_enable(False)
    got = {name: n for name, (n, _) in e4b.e4b_profiler_read().items()}
    assert sum(got.values()) == e4b.e4b_launch_count() - n0
    return got


def _training_calls(cfg, streaming):
    d = dv.upload(inputs.make_problem(cfg))
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    assert (cfg.N <= 16 * cfg.E) == streaming
    fwd = "nf4_stream" if streaming else "nf4_gemm"
    assert _launched(lambda: blk.e4b_route_permute(d.logits, d.x, gather=False)) == {
        "route_topk": 1, "route_scan": 1, "route_rank": 1}
    assert _launched(lambda: blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora(), x=d.x)) == {
        "gather_proj_x": 1, fwd + "_fwd_gate_up": 1, "lora_proj": 1, fwd + "_fwd_down": 1, "combine_y": 1}
    assert _launched(lambda: blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), d.dY)) == {
        "gather_proj_dyw": 1, "nf4_gemm_dgrad_down": 1, "lora_proj": 1, "nf4_gemm_dgrad_gate_up": 1,
        "combine_dx": 1}
    assert _launched(blk.e4b_lora_wgrad) == {"lora_wgrad": 1}
    # the routing call that also permutes the rows adds the gather; the forward then projects them
    assert _launched(lambda: blk.e4b_route_permute(d.logits, d.x)) == {
        "route_topk": 1, "route_scan": 1, "route_rank": 1, "gather_x": 1}
    assert _launched(lambda: blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora())) == {
        "lora_proj": 2, fwd + "_fwd_gate_up": 1, fwd + "_fwd_down": 1, "combine_y": 1}
    assert blk.check_device_error() == e4b.E4B_OK


def test_training_sized_batch_runs_the_grouped_tensor_core_gemms():
    _training_calls(gp.SMALL["medium"], streaming=False)


def test_decode_sized_batch_forward_runs_the_weight_streaming_kernels():
    _training_calls(gp.SMALL["stream_r24"], streaming=True)


def test_serving_call_is_routing_plus_one_launch_for_a_decode_batch():
    cfg = inputs.CONFIGS["decode"]
    d = dv.upload(inputs.make_problem(cfg))
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    assert _launched(lambda: blk.e4b_moe_serve_fwd(d.logits, d.x, d.base(), d.lora())) == {
        "route_small": 1, "nf4_serve": 1}
    assert blk.check_device_error() == e4b.E4B_OK


def test_serving_call_above_64_tokens_routes_in_three_launches_then_one():
    # more than one routing block of tokens: the multi-block routing kernels, then the same single launch
    cfg = gp.SMALL["stream_zipf_r64"]
    assert cfg.T > 64 and cfg.N <= 16 * cfg.E
    d = dv.upload(inputs.make_problem(cfg))
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    assert _launched(lambda: blk.e4b_moe_serve_fwd(d.logits, d.x, d.base(), d.lora())) == {
        "route_topk": 1, "route_scan": 1, "route_rank": 1, "nf4_serve": 1}
    assert blk.check_device_error() == e4b.E4B_OK

"""The largest expert count the library admits, E = 1024 (GPU).

Routing keeps up to 32 logits per lane at this size and most experts get a
handful of slots (or none), so nearly every 128-row group is mostly padding.
Checked against the oracle: the training calls (routing, forward, input
gradient, weight gradients) on a Zipf-skewed batch, and the serving call on a
decode-sized batch (one-CTA routing).  The file is named to be collected last.
"""

import numpy as np
import pytest

import oracle
import test_gpu_parity as gp
from grouped_nf4_expert_b200 import build, e4b, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    e4b.lib()


TRAIN = inputs.Config("max_experts", E=1024, H=64, I=64, top_k=8, T=600, r=8, alpha=16.0, routing="zipf",
                      seed=61)
SERVE = inputs.Config("max_experts_decode", E=1024, H=128, I=64, top_k=8, T=16, r=16, alpha=32.0,
                      routing="normal", seed=62)


def test_max_expert_count_training_calls():
    gp._check_block(TRAIN, True)


def test_max_expert_count_serving_call():
    prob, _, blk = gp._serve(SERVE)
    gp._check_serve_routing(prob, blk)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, gp.oracle_experts(prob), SERVE.top_k, SERVE.alpha)
    assert gp.rel_err(gp.f64(blk.y), fo["y"]) <= gp.TOL

"""Binding-level checks that need a GPU (collected after the parity tests).

The binding refuses mismatched tensors in Python before any library launch,
and a block's four LoRA gradients are views of one flat buffer, which a
data-parallel step reduces with one collective.
"""

import pytest

from grouped_nf4_expert_b200 import build, e4b, inputs
from grouped_nf4_expert_b200 import device as dv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    e4b.lib()


def test_binding_refuses_mismatched_tensors_before_any_launch():
    # wrong dtype, layout, size or problem: refused in Python, nothing launched
    cfg = inputs.CONFIGS["tiny"]
    d = dv.upload(inputs.make_problem(cfg))
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    n0 = e4b.e4b_launch_count()
    with pytest.raises(TypeError, match="logits: dtype"):
        blk.e4b_route_permute(d.logits.double(), d.x)
    with pytest.raises(ValueError, match="x: must be contiguous"):
        blk.e4b_route_permute(d.logits, d.x.t())
    with pytest.raises(ValueError, match="dY: .* elements, the call needs"):
        blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), d.dY[: cfg.T // 2])
    small = inputs.Config("small_e", E=2, H=cfg.H, I=cfg.I, top_k=1, T=8, r=cfg.r, alpha=cfg.alpha,
                          routing="normal", seed=3)
    ds = dv.upload(inputs.make_problem(small))
    with pytest.raises(ValueError, match="base.gate_up_nf4: .* the dims need"):
        blk.e4b_grouped_nf4_lora_fwd(ds.base(), d.lora(), x=d.x)
    with pytest.raises(ValueError, match="lora.A_gu: .* the dims need"):
        blk.e4b_moe_serve_fwd(d.logits, d.x, d.base(), ds.lora())
    assert e4b.e4b_launch_count() == n0


def test_lora_gradients_are_views_of_one_flat_buffer():
    # a data-parallel step reduces the four gradients with one collective over this buffer
    cfg = inputs.CONFIGS["train"]
    blk = e4b.Block(dv.dims_of(cfg), 1)
    grads = (blk.dA_gu, blk.dB_gu, blk.dA_d, blk.dB_d)
    addr = blk.lora_grads.data_ptr()
    for g in grads:
        assert g.is_contiguous() and g.data_ptr() % 16 == 0
        assert g.data_ptr() == addr
        addr += g.numel() * 2
    assert addr == blk.lora_grads.data_ptr() + blk.lora_grads.numel() * 2

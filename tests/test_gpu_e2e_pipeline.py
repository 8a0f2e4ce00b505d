"""The end-to-end measurement's training loop delivers the library's results.

`bench.py` times the training workloads end to end as a loop in which step
i+1's inputs are copied in and step i's results copied out on two copy streams
(inputs and results double-buffered on the device).  The results that reach
pinned host memory must be exactly the ones the library computed for that
step: the calls are deterministic and every step sees the same inputs, so the
last copied-out set equals the outputs left on the device, bit for bit.
"""

import importlib.util
import os
import types

import numpy as np
import pytest
import torch

from grouped_nf4_expert_b200 import e4b, inputs
from grouped_nf4_expert_b200 import device as dv

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,steps", [("tiny", 3), ("tiny", 4)])
def test_pipelined_end_to_end_copies_out_the_step_results(name, steps):
    bench = _bench_module()
    cfg = inputs.CONFIGS[name]
    dev = torch.device("cuda", 0)
    prob = inputs.make_problem(cfg)
    d = dv.upload(prob, dev)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T, dev)
    base, lora = d.base(), d.lora()
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)  # noqa: E731
    ins = (pin(d.x), pin(d.logits), pin(d.dY))
    for h, t in zip(ins, (d.x, d.logits, d.dY)):
        h.copy_(t)
    outs = [blk.y, blk.dx, blk.lora_grads]
    houts = [pin(t) for t in outs]
    for h in houts:
        h.fill_(0)
    ctx = types.SimpleNamespace(dev=dev, world=1, sync_all=lambda: torch.cuda.synchronize(dev))
    ms = bench.pipelined_e2e(ctx, steps, blk, base, lora, d, ins, outs, houts, True, (blk.lora_grads,))
    assert ms > 0
    assert blk.check_device_error() == e4b.E4B_OK
    # `houts` is the first host set: it holds the results of the last even step; the device holds the
    # last step's, computed from the same inputs
    for h, t in zip(houts, outs):
        assert np.array_equal(h.view(torch.int16).numpy(), t.view(torch.int16).cpu().numpy())
        assert h.view(torch.int16).abs().sum().item() > 0

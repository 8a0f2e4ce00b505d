"""Data-parallel path on CPU: two gloo ranks, each with its own token batch.

After the all-reduce, every rank's LoRA gradients must equal the gradients of
the union of both batches (the gradients are sums over tokens), computed by
the oracle in one process.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from grouped_nf4_expert_b200 import inputs
from grouped_nf4_expert_b200 import parallel

CFG = inputs.Config("dp", E=4, H=64, I=64, top_k=2, T=12, r=8, alpha=16.0, routing="normal", seed=51)
KEYS = ("dA_gu", "dB_gu", "dA_d", "dB_d")


def _experts(prob):
    f = lambda b: inputs.bits_to_f32(b).astype(np.float64)  # noqa: E731
    return oracle.Experts(prob.gate_up_nf4, prob.gate_up_absmax, prob.down_nf4, prob.down_absmax,
                          f(prob.A_gu), f(prob.B_gu), f(prob.A_d), f(prob.B_d))


def _rank_grads(rank):
    prob = inputs.make_problem(CFG, data_rank=rank)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    bo = oracle.moe_backward(x, prob.logits, dY, _experts(prob), CFG.top_k, CFG.alpha)
    return [bo[k] for k in KEYS]


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = _rank_grads(rank)
        grads = [torch.from_numpy(g.copy()) for g in mine]
        parallel.allreduce_lora_grads(grads)
        # as the training step does it: the four gradients as views of one flat buffer, one collective
        flat = torch.cat([torch.from_numpy(g).reshape(-1) for g in mine])
        views, o = [], 0
        for g in mine:
            views.append(flat[o:o + g.size].view(g.shape))
            o += g.size
        parallel.allreduce_lora_grads([flat])
        out_q.put((rank, [g.numpy() for g in grads], [v.numpy().copy() for v in views]))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_allreduce_equals_union_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results, flat_results = {}, {}
    for _ in range(world):
        rank, per_tensor, flat_views = q.get(timeout=240)
        results[rank], flat_results[rank] = per_tensor, flat_views
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # union batch: both ranks' tokens in one oracle call
    pa, pb = inputs.make_problem(CFG, data_rank=0), inputs.make_problem(CFG, data_rank=1)
    union = inputs.make_problem(CFG, T=2 * CFG.T)
    union.x = np.concatenate([pa.x, pb.x])
    union.logits = np.concatenate([pa.logits, pb.logits])
    union.dY = np.concatenate([pa.dY, pb.dY])
    x = inputs.bits_to_f32(union.x).astype(np.float64)
    dY = inputs.bits_to_f32(union.dY).astype(np.float64)
    bo = oracle.moe_backward(x, union.logits, dY, _experts(union), CFG.top_k, CFG.alpha)
    for r in range(world):
        for k, got, got_flat in zip(KEYS, results[r], flat_results[r]):
            np.testing.assert_allclose(got, bo[k], rtol=1e-10, atol=1e-12)
            np.testing.assert_array_equal(got_flat, got)
    # the ranks really had different batches
    assert not np.array_equal(pa.x, pb.x)

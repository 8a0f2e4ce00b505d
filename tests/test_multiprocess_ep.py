"""Expert-parallel plumbing on CPU: two gloo ranks, each owning half of the experts.

Each rank routes its own tokens over all experts, sends every routed slot's row
to the rank owning that expert, computes its experts' outputs for the rows it
received (top-1 onto the received expert, weight 1), and gets the outputs back
for the weighted combine; the backward sends w * dY rows the same way.  The
local expert computation here is the oracle (this test checks the exchange,
not the kernels): every rank's y and dx must equal the oracle's full block on
its tokens, and each owner's LoRA gradients must equal the union batch's
gradients of its experts.
"""

import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import oracle
from grouped_nf4_expert_b200 import inputs
from grouped_nf4_expert_b200 import parallel

CFG = inputs.Config("ep", E=4, H=64, I=64, top_k=2, T=13, r=8, alpha=16.0, routing="zipf", seed=57)
# four ranks, two experts each, skewed routing and few tokens: some rank pairs exchange no rows
CFG4 = inputs.Config("ep4", E=8, H=64, I=64, top_k=3, T=5, r=8, alpha=16.0, routing="zipf", seed=58)
KEYS = ("dA_gu", "dB_gu", "dA_d", "dB_d")


def _experts(prob, sl=slice(None)):
    f = lambda b: inputs.bits_to_f32(b).astype(np.float64)  # noqa: E731
    return oracle.Experts(prob.gate_up_nf4[sl], prob.gate_up_absmax[sl], prob.down_nf4[sl], prob.down_absmax[sl],
                          f(prob.A_gu[sl]), f(prob.B_gu[sl]), f(prob.A_d[sl]), f(prob.B_d[sl]))


def _onehot_logits(local_ids, n):
    lg = np.full((len(local_ids), n), -1e30, dtype=np.float32)
    lg[np.arange(len(local_ids)), local_ids] = 0.0
    return lg


def _worker(rank, world, port, out_q, cfg_name="ep"):
    global CFG
    CFG = CFG4 if cfg_name == "ep4" else CFG
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        prob = inputs.make_problem(CFG, data_rank=rank)
        e_loc = CFG.E // world
        local = _experts(prob, slice(rank * e_loc, (rank + 1) * e_loc))
        x = inputs.bits_to_f32(prob.x).astype(np.float64)
        dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
        ids, w = oracle.route_topk(prob.logits, CFG.top_k)
        ids_t, w_t = torch.from_numpy(ids.astype(np.int64)), torch.from_numpy(w)
        # the owner's computation for received rows: top-1 onto the local expert, weight 1 (the oracle)
        seen = {}

        def local_forward(rows, local_ids):
            seen["x"], seen["ids"] = rows.numpy(), local_ids.numpy()
            if not len(local_ids):
                return torch.zeros((0, CFG.H), dtype=torch.float64)
            lg = _onehot_logits(local_ids.numpy(), e_loc)
            return torch.from_numpy(oracle.moe_forward(rows.numpy(), lg, local, 1, CFG.alpha)["y"])

        def local_backward(dyw_rows, local_ids):
            assert np.array_equal(local_ids.numpy(), seen["ids"])  # same rows, same order as the forward
            if not len(local_ids):
                seen["grads"] = [np.zeros_like(getattr(local, a)) for a in ("A_gu", "B_gu", "A_d", "B_d")]
                return torch.zeros((0, CFG.H), dtype=torch.float64)
            lg = _onehot_logits(local_ids.numpy(), e_loc)
            bo = oracle.moe_backward(seen["x"], lg, dyw_rows.numpy(), local, 1, CFG.alpha)
            seen["grads"] = [bo[k] for k in KEYS]
            return torch.from_numpy(bo["dx"])

        y, _ = parallel.ep_block_forward(ids_t, w_t, torch.from_numpy(x), CFG.E, local_forward)
        dx = parallel.ep_block_backward(ids_t, w_t, torch.from_numpy(dY), CFG.E, local_backward)
        # rows that crossed between ranks (counted from the routing, as the dispatch plans them)
        owner = parallel.expert_owner(ids_t.reshape(-1), CFG.E, world)
        sent = int((owner != rank).sum())
        counts = torch.bincount(owner, minlength=world)
        recv = torch.empty_like(counts)
        dist.all_to_all_single(recv, counts)
        recvd = int(recv.sum() - recv[rank])
        out_q.put((rank, y.double().numpy(), dx.double().numpy(), seen["grads"], sent, recvd))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_expert_parallel_equals_full_block():
    _run_and_check(2, CFG, "ep", require_exchange=True)


def test_four_rank_expert_parallel_with_empty_exchanges():
    # the case really has a rank that sends no rows to another
    counts = []
    for r in range(4):
        ids, _ = oracle.route_topk(inputs.make_problem(CFG4, data_rank=r).logits, CFG4.top_k)
        counts.append(np.bincount(ids.reshape(-1) // (CFG4.E // 4), minlength=4))
    assert (np.array(counts) == 0).any()
    _run_and_check(4, CFG4, "ep4", require_exchange=False)


def _run_and_check(world, cfg, cfg_name, require_exchange):
    global CFG
    CFG = cfg
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, cfg_name)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, *rest = q.get(timeout=240)
        results[rank] = rest
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    probs = [inputs.make_problem(CFG, data_rank=r) for r in range(world)]
    full = _experts(probs[0])
    grads_union = {k: 0.0 for k in KEYS}
    for r, prob in enumerate(probs):
        x = inputs.bits_to_f32(prob.x).astype(np.float64)
        dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
        fo = oracle.moe_forward(x, prob.logits, full, CFG.top_k, CFG.alpha)
        bo = oracle.moe_backward(x, prob.logits, dY, full, CFG.top_k, CFG.alpha)
        y, dx, _, sent, recvd = results[r]
        np.testing.assert_allclose(y, fo["y"], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dx, bo["dx"], rtol=1e-10, atol=1e-12)
        if require_exchange:
            assert sent > 0 and recvd > 0  # rows really crossed between the ranks
        for k in KEYS:
            grads_union[k] = grads_union[k] + bo[k]
    e_loc = CFG.E // world
    for r in range(world):
        for k, got in zip(KEYS, results[r][2]):
            np.testing.assert_allclose(got, grads_union[k][r * e_loc:(r + 1) * e_loc], rtol=1e-10, atol=1e-12)


def test_expert_owner_blocks():
    ids = torch.arange(8)
    assert parallel.expert_owner(ids, 8, 2).tolist() == [0, 0, 0, 0, 1, 1, 1, 1]
    assert parallel.expert_owner(ids, 8, 4).tolist() == [0, 0, 1, 1, 2, 2, 3, 3]
    try:
        parallel.expert_owner(ids, 6, 4)
        raise AssertionError("E not divisible by the ranks must be refused")
    except ValueError:
        pass

"""Multi-GPU plumbing, one process per GPU over torch.distributed (NCCL over NVLink on GPUs; the
tests use gloo on CPU).

Data parallel: every rank runs the whole block on its own tokens.  The frozen NF4 base is
replicated and has no gradient, so the only exchange of a training step is the sum of the four
LoRA gradient tensors over all ranks (:func:`allreduce_lora_grads`).

Expert parallel: the experts are split across the ranks and the routed rows travel to their
experts' owners and back (:func:`ep_dispatch`, :func:`ep_return`, :func:`ep_combine`,
:func:`ep_block_forward`, :func:`ep_block_backward`); the owner computes through the library with
:func:`ep_local_forward` / :func:`ep_local_backward`.
"""

from __future__ import annotations


def allreduce_lora_grads(grads, group=None):
    """Sums each gradient tensor over all ranks of ``group``, in place.  A
    :class:`~grouped_nf4_expert_b200.e4b.Block` holds its four LoRA gradients as views of one flat
    buffer (``Block.lora_grads``): passing that buffer sums all four in one collective."""
    import torch.distributed as dist
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    return grads


# ----------------------------------------------------------------------------------------------------
# Expert parallel: the experts are split into `world` contiguous blocks of E / world, rank r owning
# block r (its slice of the NF4 stacks and LoRA factors).  Every rank routes its own tokens over all E
# experts; each routed slot's row travels to the rank owning its expert (all-to-all), the owner runs
# the block on its experts with every received row routed to exactly that expert (top-1, weight 1),
# and the expert outputs travel back to be combined with the routing weights.  The backward sends
# w * dY rows the same way and returns each slot's input gradient; the LoRA gradients of an expert
# live on its owner only (no reduction).  Remote rows land in local memory before any compute.
# ----------------------------------------------------------------------------------------------------

class EpPlan:
    """Send order and counts of one dispatch (kept for the return trip)."""

    def __init__(self, order, send_counts, recv_counts, k):
        self.order = order              # slot indices f = t*k + j, grouped by owner rank (stable)
        self.send_counts = send_counts  # [world] slots sent to each rank
        self.recv_counts = recv_counts  # [world] rows received from each rank
        self.k = k


def expert_owner(ids, E: int, world: int):
    """Rank owning each expert id (contiguous blocks of E / world experts)."""
    if E % world:
        raise ValueError("expert parallel needs E divisible by the number of ranks")
    return ids // (E // world)


def _a2a_rows(rows, send_counts, recv_counts, group=None):
    """All-to-all of the rows of a 2-D tensor (split sizes in rows); bf16 travels as int16."""
    import torch
    import torch.distributed as dist
    as16 = rows.dtype == torch.bfloat16
    src = rows.view(torch.int16) if as16 else rows
    out = src.new_empty((int(sum(recv_counts)),) + tuple(src.shape[1:]))
    dist.all_to_all_single(out, src.contiguous(), output_split_sizes=list(recv_counts),
                           input_split_sizes=list(send_counts), group=group)
    return out.view(torch.bfloat16) if as16 else out


def ep_dispatch(ids, rows, E: int, group=None):
    """Sends each routed slot's row to the owner of its expert.

    ``ids`` [T, k] global expert ids (descending logit per token, as routing writes them), ``rows``
    [T, H] (per token) or [T*k, H] (per slot).  Returns ``(recv_rows, recv_local_ids, plan)``: the rows
    this rank received (grouped by source rank, in the sender's slot order) and their local expert ids.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    T, k = ids.shape
    flat = ids.reshape(-1).to(torch.int64)
    owner = expert_owner(flat, E, world)
    order = torch.sort(owner, stable=True).indices
    send_counts = torch.bincount(owner, minlength=world)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    send_counts, recv_counts = send_counts.tolist(), recv_counts.tolist()
    src = rows[order // k] if rows.shape[0] == T and k > 1 else rows[order]
    recv_rows = _a2a_rows(src, send_counts, recv_counts, group)
    local_ids = (flat[order] - owner[order] * (E // world)).to(torch.int32).unsqueeze(1)
    recv_ids = _a2a_rows(local_ids, send_counts, recv_counts, group).squeeze(1)
    return recv_rows, recv_ids, EpPlan(order, send_counts, recv_counts, k)


def ep_return(rows, plan: EpPlan, group=None):
    """Sends per-row results back to the slots they came from: [T*k, H] in slot order."""
    back = _a2a_rows(rows, plan.recv_counts, plan.send_counts, group)
    out = back.new_empty(back.shape)
    out[plan.order] = back
    return out


def ep_combine(slot_rows, w):
    """y[t] = sum_j w[t, j] * slot_rows[t*k + j], summed in slot order in fp32 (fp64 for fp64 rows)."""
    import torch
    T, k = w.shape
    dt = torch.promote_types(torch.float32, slot_rows.dtype)
    acc = torch.zeros((T, slot_rows.shape[1]), dtype=dt, device=slot_rows.device)
    rows = slot_rows.to(dt).view(T, k, -1)
    for j in range(k):
        acc += w[:, j:j + 1].to(dt) * rows[:, j]
    return acc


def ep_local_forward(dims_local, rows, local_ids, base_local, lora_local):
    """The owner's experts on the rows it received: every row routed top-1 to its local expert with
    weight 1, through the library's forward, so the block output of a row is its expert's output.

    ``dims_local``: :class:`~grouped_nf4_expert_b200.e4b.Dims` with E the local expert count (top_k
    is taken as 1); ``rows`` bf16 [R, H] and ``local_ids`` [R] on the GPU; ``base_local`` /
    ``lora_local`` the owner's slices of the stacks.  Returns the :class:`e4b.Block` holding the
    outputs (``y`` [R, H]) and the activations a backward needs.
    """
    import torch
    from . import e4b
    d = e4b.Dims(E=dims_local.E, H=dims_local.H, I=dims_local.I, top_k=1, r=dims_local.r,
                 alpha=dims_local.alpha)
    R = rows.shape[0]
    blk = e4b.Block(d, R, rows.device)
    logits = torch.full((max(R, 1), d.E), -1e30, dtype=torch.float32, device=rows.device)[:R]
    logits[torch.arange(R, device=rows.device), local_ids.long()] = 0.0
    blk.e4b_route_permute(logits, rows, gather=False)
    blk.e4b_grouped_nf4_lora_fwd(base_local, lora_local, x=rows)
    return blk


def ep_local_backward(blk, dyw_rows, base_local, lora_local):
    """The owner's backward for the rows it received: ``dyw_rows`` bf16 [R, H] are the received
    w * dY rows (the routing weight applied by the sender), run through the library's input
    gradient and LoRA weight gradients with the top-1, weight-1 routing of :func:`ep_local_forward`
    (``blk`` is the block it returned).  Returns ``blk``: ``dx`` [R, H] holds each row's input
    gradient (to be sent back), ``dA_gu``/``dB_gu``/``dA_d``/``dB_d`` the owner's expert gradients."""
    blk.e4b_grouped_nf4_lora_dgrad(base_local, lora_local, dyw_rows)
    blk.e4b_lora_wgrad()
    return blk


def ep_block_forward(ids, w, x, E: int, local_forward, group=None):
    """Expert-parallel forward of this rank's tokens.

    ``ids``/``w`` [T, k]: this rank's routing over all E experts; ``x`` [T, H].  ``local_forward(rows,
    local_ids)`` computes the owner's expert outputs for the rows it received (for instance through
    :func:`ep_local_forward`: its block's ``y``).  Returns ``(y, state)``: y [T, H] in fp32 (fp64 for
    fp64 rows), and the state :func:`ep_block_backward` needs.
    """
    rows, local_ids, plan = ep_dispatch(ids, x, E, group)
    yd = local_forward(rows, local_ids)
    y = ep_combine(ep_return(yd, plan, group), w)
    return y, (rows, local_ids)


def ep_block_backward(ids, w, dY, E: int, local_backward, group=None):
    """Expert-parallel input gradient of this rank's tokens: w * dY rows go to the owners,
    ``local_backward(dyw_rows, local_ids)`` returns each received row's input gradient (the owner
    keeps its experts' LoRA gradients), and the rows come back summed per token: dx [T, H]."""
    import torch
    T, k = w.shape
    dt = torch.promote_types(torch.float32, dY.dtype)  # the product in fp32, rounded once (as the library)
    dyw = (w.to(dt).unsqueeze(2) * dY.to(dt).unsqueeze(1)).to(dY.dtype).reshape(T * k, -1)
    rows, local_ids, plan = ep_dispatch(ids, dyw, E, group)
    dx_rows = local_backward(rows, local_ids)
    return ep_combine(ep_return(dx_rows, plan, group), torch.ones_like(w))

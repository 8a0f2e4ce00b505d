"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Indices and NF4 dequantisation must match bit for bit; bf16 values must
satisfy max|gpu - oracle| / max|oracle| <= 1e-2 (fp32 accumulation on the
GPU, float64 in the oracle); where the oracle is exactly zero the GPU must be
exactly zero.  Small cases compare every element; the full-size workloads
compare sampled tokens and experts the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import oracle
from grouped_nf4_expert_b200 import build, e4b, inputs
from grouped_nf4_expert_b200 import device as dv

pytestmark = pytest.mark.gpu

TOL = 1e-2

SMALL = {
    "tiny": inputs.CONFIGS["tiny"],
    "tiny_b0": inputs.CONFIGS["tiny_b0"],
    # several tiles per dimension, ragged groups, K loops of several stages
    "medium": inputs.Config("medium", E=8, H=256, I=384, top_k=2, T=300, r=16, alpha=32.0,
                            routing="normal", seed=31),
    # Zipf skew: experts spanning several 128-row tiles next to nearly empty ones; r = 64
    "medium_zipf_r64": inputs.Config("medium_zipf_r64", E=32, H=512, I=256, top_k=4, T=700, r=64,
                                     alpha=128.0, routing="zipf", seed=32),
    # r = 24 (padded to 32), H and I not multiples of 128 (half-empty output tiles)
    "medium_r24": inputs.Config("medium_r24", E=6, H=192, I=320, top_k=3, T=257, r=24, alpha=48.0,
                                routing="normal", seed=33),
    # decode-sized batches (T*k <= 16*E) take the weight-streaming forward:
    # Zipf skew puts several 32-slot tiles on the popular experts; r = 64
    "stream_zipf_r64": inputs.Config("stream_zipf_r64", E=64, H=256, I=192, top_k=8, T=100, r=64,
                                     alpha=128.0, routing="zipf", seed=34),
    # r = 24, H not a multiple of 128 (half-empty down tile), a few slots per expert
    "stream_r24": inputs.Config("stream_r24", E=16, H=192, I=128, top_k=2, T=64, r=24, alpha=48.0,
                                routing="normal", seed=35),
}


@pytest.fixture(scope="session", autouse=True)
def _built():
    build.build()
    e4b.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    m = np.abs(ref).max() if ref.size else 0.0
    if m == 0.0:
        return 0.0 if np.all(gpu == 0) else np.inf
    return float(np.abs(gpu - ref).max() / m)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_experts(prob):
    f = lambda b: inputs.bits_to_f32(b).astype(np.float64)  # noqa: E731
    return oracle.Experts(prob.gate_up_nf4, prob.gate_up_absmax, prob.down_nf4, prob.down_absmax,
                          f(prob.A_gu), f(prob.B_gu), f(prob.A_d), f(prob.B_d))


def run(cfg, fwd=True, dgrad=True, wgrad=True, prob=None, fused_gather=True):
    # fused_gather: x_perm is written by the forward (with its first projection), else by the routing call
    prob = prob if prob is not None else inputs.make_problem(cfg)
    d = dv.upload(prob)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    fused = fused_gather and fwd
    blk.e4b_route_permute(d.logits, d.x, gather=not fused)
    if fwd:
        blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora(), x=d.x if fused else None)
    if dgrad:
        blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), d.dY)
    if wgrad:
        blk.e4b_lora_wgrad()
    assert blk.check_device_error() == e4b.E4B_OK
    return prob, d, blk


def check_routing(prob, blk):
    cfg = prob.cfg
    ids, w = oracle.route_topk(prob.logits, cfg.top_k)
    g = oracle.group_by_expert(ids, cfg.E)
    assert np.array_equal(blk.topk_ids.cpu().numpy(), ids)
    np.testing.assert_allclose(blk.topk_w.cpu().numpy(), w, rtol=4e-6, atol=1e-7)
    assert np.array_equal(blk.counts.cpu().numpy(), g["counts"])
    offsets = blk.offsets.cpu().numpy().astype(np.int64)
    padded = (g["counts"] + 127) // 128 * 128
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), padded)
    flat = ids.reshape(-1)
    ros = blk.row_of_slot.cpu().numpy().astype(np.int64)
    assert np.array_equal(ros - offsets[flat], g["rank"])
    used = int(offsets[-1])
    sor = blk.slot_of_row.cpu().numpy()[:used]
    assert np.array_equal(sor[ros], np.arange(flat.size))
    pad = np.ones(used, dtype=bool)
    pad[ros] = False
    assert np.all(sor[pad] == -1)
    xp = bits(blk.x_perm)[:used]
    assert np.array_equal(xp[ros], prob.x[np.arange(flat.size) // cfg.top_k])
    assert np.all(xp[pad] == 0)
    tiles = blk.tiles.cpu().numpy()
    assert tiles[0] == padded.sum() // 128 and tiles[1] == used
    return ros


# --------------------------------------------------------------------- decode

def test_nf4_dequant_bit_exact():
    rng = np.random.default_rng(0)
    n = 64 * 8192
    packed = rng.integers(0, 256, n // 2, dtype=np.uint8)
    packed[:256] = np.arange(256, dtype=np.uint8)
    absmax = rng.uniform(0.0, 0.2, n // 64).astype(np.float32)
    absmax[:12] = np.array([0.0, 1.0, 1e-30, 3e38, 0.5, 2.0 ** -126, 1e-45, 7.5, -0.3, 2.0 ** -149, 1e20, 0.02],
                           dtype=np.float32)
    want, _ = oracle.dequantize_nf4(packed.reshape(1, -1), absmax.reshape(1, -1))
    dp = torch.from_numpy(packed).cuda()
    da = torch.from_numpy(absmax).cuda()
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_nf4_dequant(dp, da, out)
    torch.cuda.synchronize()
    got = bits(out)
    assert np.array_equal(got, want[0]), np.flatnonzero(got != want[0])[:10]


def _quantize_gpu(w_bits):
    w = torch.from_numpy(w_bits.view(np.int16)).cuda().view(torch.bfloat16)
    packed = torch.empty(w.numel() // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(w.numel() // 64, dtype=torch.float32, device="cuda")
    e4b.e4b_nf4_quantize(w, packed, absmax)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), absmax.cpu().numpy()


def test_nf4_quantize_bit_exact_special_blocks():
    # codes are integers decided in float32 on both sides: they must agree bit for bit
    rng = np.random.default_rng(3)
    lv = oracle.nf4_table().astype(np.float32)
    blocks = [np.zeros(64, np.float32),                                   # zero block -> code 7, absmax 0
              np.r_[np.zeros(63), 0.25].astype(np.float32),              # a single nonzero
              rng.standard_normal(64).astype(np.float32) * 1e-38,        # subnormal scale
              rng.standard_normal(64).astype(np.float32) * 1e37,         # huge scale
              -np.abs(rng.standard_normal(64)).astype(np.float32),      # all negative
              np.r_[1.0, -1.0, np.zeros(62)].astype(np.float32)]         # the two extreme levels
    # exact midpoints between adjacent levels (scaled by a power of two: w / absmax stays exact)
    mids = (lv[:-1] + lv[1:]) / np.float32(2.0)
    blk = np.zeros(64, np.float32)
    blk[0] = 1.0
    blk[1:16] = mids
    blocks.append(blk * np.float32(0.5))
    for scale in (0.02, 1.0, 3.0):
        blocks += [(rng.standard_normal(64) * scale).astype(np.float32) for _ in range(200)]
    # every bf16 value of [-amax, amax] next to a block maximum amax, for amax = 1 (x = w exactly) and
    # amax = 1.5, 0.3 (x rounded by the division): every decision near every midpoint is taken
    for amax in (1.0, 1.5, 0.3):
        top = int(oracle.bf16_round_bits(np.array([amax], np.float32))[0])
        vals = np.r_[np.arange(0, top + 1), np.arange(0x8000, 0x8000 + top + 1)].astype(np.uint16)
        vals = inputs.bits_to_f32(vals)
        vals = np.r_[vals, np.zeros((-vals.size) % 63, np.float32)].reshape(-1, 63)
        blocks += list(np.c_[np.full((vals.shape[0], 1), inputs.bits_to_f32(np.array([top], np.uint16))[0]),
                             vals].astype(np.float32))
    w = np.stack(blocks).reshape(-1)
    w_bits = oracle.bf16_round_bits(w)                # the bf16 weights both sides see
    w32 = inputs.bits_to_f32(w_bits)
    want_p, want_a = oracle.quantize_nf4(w32.reshape(1, -1))
    got_p, got_a = _quantize_gpu(w_bits)
    assert np.array_equal(got_p, want_p[0]), np.flatnonzero(got_p != want_p[0])[:10]
    assert np.array_equal(got_a.view(np.uint32), want_a[0].view(np.uint32))


def _near_boundary_blocks(n_amax=400, seed=7):
    # Blocks whose w / absmax (IEEE float32) falls within 2^-17 of a level or of a midpoint between two
    # adjacent levels: the decisions a fast approximate quotient could get wrong.
    lv = oracle.nf4_table().astype(np.float64)
    pts = np.r_[lv, (lv[:-1] + lv[1:]) / 2.0]
    rng = np.random.default_rng(seed)
    tops = np.unique(oracle.bf16_round_bits(rng.uniform(0.01, 10.0, n_amax).astype(np.float32)))
    blocks, hits = [], 0
    for top in tops:
        a = inputs.bits_to_f32(np.array([top], np.uint16))[0]
        vals = inputs.bits_to_f32(np.r_[np.arange(1, top), np.arange(0x8001, 0x8000 + top)].astype(np.uint16))
        x = (vals / a).astype(np.float64)  # float32 division, then exact widening
        near = np.abs(x[:, None] - pts[None, :]).min(axis=1) <= 2.0 ** -17
        v = vals[near][:63]
        if v.size:
            hits += v.size
            blocks.append(np.r_[a, v, np.zeros(63 - v.size, np.float32)].astype(np.float32))
    return blocks, hits


def test_nf4_quantize_bit_exact_near_decision_boundaries():
    blocks, hits = _near_boundary_blocks()
    assert hits >= 500
    w_bits = oracle.bf16_round_bits(np.stack(blocks).reshape(-1))
    want_p, want_a = oracle.quantize_nf4(inputs.bits_to_f32(w_bits).reshape(1, -1))
    got_p, got_a = _quantize_gpu(w_bits)
    assert np.array_equal(got_p, want_p[0]), np.flatnonzero(got_p != want_p[0])[:10]
    assert np.array_equal(got_a.view(np.uint32), want_a[0].view(np.uint32))


def test_nf4_quantize_full_size_stack_sampled_blocks():
    # a gate_up-sized stack of the fine-grained workload (128 x 1536 x 2048 bf16, 805 MB), checked on sampled blocks
    E, R, K = 128, 1536, 2048
    g = torch.Generator(device="cuda").manual_seed(5)
    w = (torch.randn(E * R * K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    packed = torch.empty(w.numel() // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(w.numel() // 64, dtype=torch.float32, device="cuda")
    e4b.e4b_nf4_quantize(w, packed, absmax)
    torch.cuda.synchronize()
    nblk = w.numel() // 64
    idx = torch.from_numpy(np.sort(np.random.default_rng(6).choice(nblk, 20000, replace=False))).cuda()
    wb = w.view(-1, 64)[idx].view(torch.int16).cpu().numpy().view(np.uint16)
    want_p, want_a = oracle.quantize_nf4(inputs.bits_to_f32(wb))
    got_p = packed.view(-1, 32)[idx].cpu().numpy()
    got_a = absmax[idx].cpu().numpy()
    assert np.array_equal(got_p, want_p)
    assert np.array_equal(got_a.view(np.uint32), want_a.reshape(-1).view(np.uint32))


# --------------------------------------------------------------------- routing

@pytest.mark.parametrize("name", list(SMALL))
def test_routing_bit_exact_small(name):
    prob, _, blk = run(SMALL[name], fwd=False, dgrad=False, wgrad=False)
    check_routing(prob, blk)


@pytest.mark.parametrize("name", ["finegrained", "decode", "train"])
def test_routing_bit_exact_workloads(name):
    prob, _, blk = run(inputs.CONFIGS[name], fwd=False, dgrad=False, wgrad=False)
    check_routing(prob, blk)


def test_routing_ties_and_deterministic():
    cfg = inputs.Config("ties", E=16, H=64, I=64, top_k=4, T=500, r=8, alpha=16.0, routing="normal", seed=41)
    prob = inputs.make_problem(cfg)
    prob.logits[:] = np.round(prob.logits * 2) / 2  # many exact ties
    prob.logits[7, :] = 0.0
    prob.logits[8, 3] = np.nan
    _, _, a = run(cfg, fwd=False, dgrad=False, wgrad=False, prob=prob)
    check_routing(prob, a)
    _, _, b = run(cfg, fwd=False, dgrad=False, wgrad=False, prob=prob)
    for t in ("topk_ids", "topk_w", "row_of_slot", "slot_of_row", "offsets", "tiles"):
        assert torch.equal(getattr(a, t), getattr(b, t)), t


# --------------------------------------------------------------------- full block, small sizes

# Degenerate shapes: one token (a 128-row tile holding 2 rows), every expert selected (k = E),
# a single expert, and k = 32 (the combine's long path) with H not a multiple of 128.
EDGE = {
    "one_token": inputs.Config("one_token", E=4, H=64, I=64, top_k=2, T=1, r=8, alpha=16.0,
                               routing="normal", seed=51),
    "k_equals_E": inputs.Config("k_equals_E", E=8, H=128, I=128, top_k=8, T=40, r=16, alpha=32.0,
                                routing="normal", seed=52),
    "one_expert": inputs.Config("one_expert", E=1, H=128, I=192, top_k=1, T=200, r=8, alpha=16.0,
                                routing="normal", seed=53),
    "k32_ragged": inputs.Config("k32_ragged", E=40, H=192, I=64, top_k=32, T=45, r=8, alpha=16.0,
                                routing="zipf", seed=54),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_block_parity_edge_shapes(name):
    _check_block(EDGE[name], True)


def test_zero_tokens_is_a_no_op_with_zero_gradients():
    cfg = inputs.Config("zero", E=4, H=64, I=64, top_k=2, T=0, r=8, alpha=16.0, routing="normal", seed=55)
    prob = inputs.make_problem(cfg)
    d = dv.upload(prob)
    blk = e4b.Block(dv.dims_of(cfg), 0)
    for t in (blk.dA_gu, blk.dB_gu, blk.dA_d, blk.dB_d):
        t.fill_(1.0)
    # [0, .] token tensors still need valid aligned pointers
    x = torch.zeros((1, cfg.H), dtype=torch.bfloat16, device="cuda")
    logits = torch.zeros((1, cfg.E), dtype=torch.float32, device="cuda")
    blk.e4b_route_permute(logits, x, gather=False)
    blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora(), x=x)
    blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), x)
    blk.e4b_lora_wgrad()
    blk.e4b_moe_serve_fwd(logits, x, d.base(), d.lora())
    torch.cuda.synchronize()
    assert blk.check_device_error() == e4b.E4B_OK
    for t in (blk.dA_gu, blk.dB_gu, blk.dA_d, blk.dB_d):
        assert torch.count_nonzero(t).item() == 0


@pytest.mark.parametrize("name,fused", [(n, True) for n in SMALL] + [("medium", False), ("stream_r24", False)])
def test_block_parity_small(name, fused):
    _check_block(SMALL[name], fused)


def _check_block(cfg, fused):
    _check_block_prob(cfg, None, fused)


def _check_block_prob(cfg, prob, fused=True):
    prob, _, blk = run(cfg, fused_gather=fused, prob=prob)
    ros = check_routing(prob, blk)
    ex = oracle_experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    s = cfg.alpha / cfg.r
    fo = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha)
    bo = oracle.moe_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha)
    slots = np.array(sorted(fo["gu"].keys()))
    rows = ros[slots]
    errs = {}
    errs["y"] = rel_err(f64(blk.y), fo["y"])
    for key, buf, scale in [("gu", blk.gu, 1.0), ("act", blk.act, 1.0), ("p_gu", blk.p_gu, s),
                            ("p_d", blk.p_d, s), ("yd", blk.y_perm, 1.0)]:
        errs[key] = rel_err(f64(buf)[rows], np.stack([fo[key][f] for f in slots]) * scale)
    errs["dx"] = rel_err(f64(blk.dx), bo["dx"])
    w = bo["w"].reshape(-1)
    errs["dyw"] = rel_err(f64(blk.dyw)[rows], w[slots, None] * dY[slots // cfg.top_k])
    for key, buf, scale in [("dgu", blk.dgu, 1.0), ("q_gu", blk.q_gu, s), ("q_d", blk.q_d, s),
                            ("dx_slot", blk.dx_perm, 1.0)]:
        errs[key] = rel_err(f64(buf)[rows], np.stack([bo[key][f] for f in slots]) * scale)
    for key, buf in [("dA_gu", blk.dA_gu), ("dB_gu", blk.dB_gu), ("dA_d", blk.dA_d), ("dB_d", blk.dB_d)]:
        errs[key] = rel_err(f64(buf), bo[key])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("name", ["tiny", "medium", "stream_r24"])
def test_block_parity_on_quantised_normal_stacks(name):
    # The workloads' recipe for the frozen base: dense weights ~ N(0, 0.02), NF4-quantised (64-element
    # blocks, fp32 absmax).  The GPU quantiser must produce the oracle quantiser's bytes exactly; the
    # block then runs on those bytes and is compared with the oracle element by element.
    cfg = SMALL[name] if name in SMALL else inputs.CONFIGS[name]
    prob = inputs.make_problem(cfg)
    gu_w, dn_w = inputs.dense_expert_weights(cfg)
    want = {}
    for key, wbits in (("gate_up", gu_w), ("down", dn_w)):
        packed, absmax = oracle.quantize_nf4(inputs.bits_to_f32(wbits))
        got_p, got_a = _quantize_gpu(wbits.reshape(-1))
        assert np.array_equal(got_p, packed.reshape(-1)), key
        assert np.array_equal(got_a.view(np.uint32), absmax.reshape(-1).view(np.uint32)), key
        want[key] = (packed, absmax)
    prob.gate_up_nf4, prob.gate_up_absmax = want["gate_up"]
    prob.down_nf4, prob.down_absmax = want["down"]
    # every code occurs (quantised normals, not a narrow subset)
    codes = np.concatenate([prob.gate_up_nf4.reshape(-1) >> 4, prob.gate_up_nf4.reshape(-1) & 15])
    assert np.unique(codes).size == 16
    _check_block_prob(cfg, prob)


def test_b_zero_delta_is_exactly_zero_on_gpu():
    cfg = inputs.CONFIGS["tiny_b0"]
    prob = inputs.make_problem(cfg)
    _, _, a = run(cfg, dgrad=False, wgrad=False, prob=prob)
    base_only = inputs.make_problem(cfg)
    base_only.A_gu[:] = 0
    base_only.A_d[:] = 0
    _, _, b = run(cfg, dgrad=False, wgrad=False, prob=base_only)
    assert np.array_equal(bits(a.y), bits(b.y))
    assert np.array_equal(bits(a.gu), bits(b.gu))


def test_empty_expert_gets_exact_zero_gradients():
    cfg = SMALL["medium"]
    prob = inputs.make_problem(cfg)
    prob.logits[:, 5] = -1e30
    _, _, blk = run(cfg, prob=prob)
    assert blk.counts[5].item() == 0
    for t in (blk.dA_gu, blk.dB_gu, blk.dA_d, blk.dB_d):
        assert torch.count_nonzero(t[5]).item() == 0
        assert torch.count_nonzero(t[0]).item() > 0


def test_frozen_base_bytes_unchanged_and_outputs_deterministic():
    cfg = SMALL["medium_zipf_r64"]
    prob = inputs.make_problem(cfg)
    d = dv.upload(prob)
    before = [t.clone() for t in (d.gate_up_nf4, d.gate_up_absmax, d.down_nf4, d.down_absmax)]
    outs = []
    for _ in range(2):
        blk = e4b.Block(dv.dims_of(cfg), cfg.T)
        blk.e4b_route_permute(d.logits, d.x)
        blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora())
        blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), d.dY)
        blk.e4b_lora_wgrad()
        assert blk.check_device_error() == e4b.E4B_OK
        outs.append([t.clone() for t in (blk.y, blk.dx, blk.dA_gu, blk.dB_gu, blk.dA_d, blk.dB_d)])
    for t0, t1 in zip(before, (d.gate_up_nf4, d.gate_up_absmax, d.down_nf4, d.down_absmax)):
        assert torch.equal(t0, t1)
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_watchdog_times_out_cleanly_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    e4b.e4b_workspace_init(ws)
    e4b.e4b_debug_watchdog(ws, 2_000_000)  # 2 ms
    assert e4b.e4b_check_device_error(ws) == e4b.E4B_ERR_DEVICE_TIMEOUT
    e4b.e4b_workspace_init(ws)
    assert e4b.e4b_check_device_error(ws) == e4b.E4B_OK
    prob, _, blk = run(inputs.CONFIGS["tiny"], dgrad=False, wgrad=False)
    assert torch.isfinite(blk.y.float()).all()


# --------------------------------------------------------------------- full-size workloads, sampled

def _sample_tokens(T, n, seed):
    return np.sort(np.random.default_rng(seed).choice(T, size=n, replace=False))


def _unit_covering_slots(prob, seed):
    """Routed slots chosen so that every work unit of the GPU path holds one of them.

    From the oracle's own routing: the slots of each expert in grouped
    (stable) order, one random slot from each 128-row tile of the expert's
    group (each 256-row unit of the grouped GEMM therefore holds two, a
    128-row tail unit one) and the expert's last slot (the ragged end of its
    group).  Every expert with a routed slot contributes.
    """
    cfg = prob.cfg
    ids, _ = oracle.route_topk(prob.logits, cfg.top_k)
    g = oracle.group_by_expert(ids, cfg.E)
    rng = np.random.default_rng(seed)
    chosen = set()
    for e in range(cfg.E):
        cnt = int(g["counts"][e])
        if cnt == 0:
            continue
        members = g["slots"][g["starts"][e]:g["starts"][e] + cnt]
        for lo in range(0, cnt, 128):
            chosen.add(int(members[rng.integers(lo, min(cnt, lo + 128))]))
        chosen.add(int(members[cnt - 1]))
    return np.array(sorted(chosen), dtype=np.int64)


def _per_row_err(gpu_rows, ref_rows):
    """max over rows of max|gpu - oracle| / max|oracle| within the row (a row that is exactly zero in
    the oracle must be exactly zero on the GPU)."""
    gpu_rows = np.asarray(gpu_rows, np.float64)
    ref_rows = np.asarray(ref_rows, np.float64)
    assert gpu_rows.shape == ref_rows.shape
    m = np.abs(ref_rows).max(axis=1)
    d = np.abs(gpu_rows - ref_rows).max(axis=1)
    err = np.where(m > 0, d / np.where(m > 0, m, 1.0), np.where(d == 0, 0.0, np.inf))
    return float(err.max()), int(err.argmax())


def _check_slots(blk, cfg, slots, fo, bo=None, dY=None):
    """Per-slot intermediates of the sampled slots, row by row, and the block outputs of their tokens."""
    ros = blk.row_of_slot.cpu().numpy().astype(np.int64)
    rows = torch.from_numpy(ros[slots]).cuda()
    s = cfg.alpha / cfg.r
    toks = np.unique(slots // cfg.top_k)
    errs = {}
    pick = lambda buf: f64(buf[rows])  # noqa: E731
    for key, buf, scale in [("gu", blk.gu, 1.0), ("act", blk.act, 1.0), ("p_gu", blk.p_gu, s),
                            ("p_d", blk.p_d, s), ("y_perm", blk.y_perm, 1.0)]:
        okey = "yd" if key == "y_perm" else key
        errs[key] = _per_row_err(pick(buf), np.stack([fo[okey][int(f)] for f in slots]) * scale)
    errs["y"] = _per_row_err(f64(blk.y)[toks], fo["y"][toks])
    if bo is not None:
        w = bo["w"].reshape(-1)
        errs["dyw"] = _per_row_err(pick(blk.dyw), w[slots, None] * dY[slots // cfg.top_k])
        for key, buf, scale in [("dgu", blk.dgu, 1.0), ("q_gu", blk.q_gu, s), ("q_d", blk.q_d, s),
                                ("dx_perm", blk.dx_perm, 1.0)]:
            okey = "dx_slot" if key == "dx_perm" else key
            errs[key] = _per_row_err(pick(buf), np.stack([bo[okey][int(f)] for f in slots]) * scale)
        errs["dx"] = _per_row_err(f64(blk.dx)[toks], bo["dx"][toks])
    bad = {k: v for k, v in errs.items() if not v[0] <= TOL}
    assert not bad, ("(max row error, sampled row index)", bad, errs)


@pytest.mark.parametrize("name", ["finegrained", "train"])
def test_workload_fwd_dgrad_every_unit_sampled(name):
    # Full size (E128 H2048 I768 top-8, 8192 tokens, Zipf routing): one slot of every 128-row tile of
    # every expert's group and each group's last slot, so a wrong work unit of any kernel (a heavy
    # expert's 29th unit, a 128-row tail unit, the lightest expert) fails; checked row by row.
    cfg = inputs.CONFIGS[name]
    prob, _, blk = run(cfg, wgrad=False)
    slots = _unit_covering_slots(prob, 100)
    ex = oracle_experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    toks = np.unique(slots // cfg.top_k)
    fo = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha, tokens=toks)
    bo = oracle.moe_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha, tokens=toks, grad_experts=[])
    ids = oracle.route_topk(prob.logits, cfg.top_k)[0].reshape(-1)
    assert set(ids[slots].tolist()) == set(np.flatnonzero(blk.counts.cpu().numpy()).tolist())
    _check_slots(blk, cfg, slots, fo, bo, dY)


def test_train_workload_wgrad_sampled_experts():
    cfg = inputs.CONFIGS["train"]
    prob, _, blk = run(cfg)
    counts = blk.counts.cpu().numpy()
    order = np.argsort(-counts, kind="stable")
    nz = order[counts[order] > 0]
    # the heaviest, the median and the lightest expert, and five more at random
    rng = np.random.default_rng(104)
    experts = sorted({int(nz[0]), int(nz[len(nz) // 2]), int(nz[-1])} |
                     set(int(e) for e in rng.choice(nz, 5, replace=False)))
    ex = oracle_experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    bo = oracle.moe_backward(x, prob.logits, dY, ex, cfg.top_k, cfg.alpha, tokens=[], grad_experts=experts)
    for key, buf in [("dA_gu", blk.dA_gu), ("dB_gu", blk.dB_gu), ("dA_d", blk.dA_d), ("dB_d", blk.dB_d)]:
        for e in experts:
            assert rel_err(f64(buf[e]), bo[key][e]) <= TOL, (key, e)


def test_decode_workload_full():
    # every routed slot of the decode batch, row by row (the weight-streaming forward)
    cfg = inputs.CONFIGS["decode"]
    prob, _, blk = run(cfg, dgrad=False, wgrad=False)
    ex = oracle_experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha)
    assert rel_err(f64(blk.y), fo["y"]) <= TOL
    _check_slots(blk, cfg, np.arange(cfg.T * cfg.top_k), fo)


def test_mixtral_workload_forward_every_unit_sampled():
    # E8 H4096 I14336 top-2, 4096 tokens (the largest groups): one slot of every 128-row tile of each
    # expert's group and each group's last slot, checked row by row (gu, act, p, y_perm, y).
    cfg = inputs.CONFIGS["mixtral"]
    prob, _, blk = run(cfg, dgrad=False, wgrad=False)
    slots = _unit_covering_slots(prob, 101)
    ex = oracle_experts(prob)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, ex, cfg.top_k, cfg.alpha, tokens=np.unique(slots // cfg.top_k))
    _check_slots(blk, cfg, slots, fo)


@pytest.mark.parametrize("name", ["finegrained", "train", "decode"])
def test_repeated_full_size_runs_are_bit_identical(name):
    # Any ordering race in the pipelined kernels shows up as run-to-run
    # differences: the training-step workload exercises the 2-SM NF4 GEMM with
    # its code ring, the decode batch the weight-streaming forward.
    cfg = inputs.CONFIGS[name]
    prob = inputs.make_problem(cfg)
    d = dv.upload(prob)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    backward = "dgrad" in cfg.passes
    ref = None
    for _ in range(6 if name == "finegrained" else 3):
        blk.e4b_route_permute(d.logits, d.x, gather=False)
        blk.e4b_grouped_nf4_lora_fwd(d.base(), d.lora(), x=d.x)
        if backward:
            blk.e4b_grouped_nf4_lora_dgrad(d.base(), d.lora(), d.dY)
            blk.e4b_lora_wgrad()
        assert blk.check_device_error() == e4b.E4B_OK
        outs = (blk.y, blk.dx, blk.gu, blk.dgu, blk.dA_gu, blk.dB_d) if backward else (blk.y, blk.gu, blk.act)
        cur = [t.clone() for t in outs]
        if ref is None:
            ref = cur
        else:
            for a, b in zip(ref, cur):
                assert torch.equal(a, b)

# --------------------------------------------------------------------- router backward (trained router)

RBWD_TOL = 1e-4  # fp32 sums of exact bf16 products against float64


def _router_bwd_gpu(blk, d, T, E, k):
    d_logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    dw = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    blk.e4b_router_backward(d.dY, d_logits, dw)
    torch.cuda.synchronize()
    return d_logits.cpu().numpy(), dw.cpu().numpy()


def _check_router_rows(dl_gpu, dw_gpu, ref, rows, tol):
    assert rel_err(dl_gpu[rows], ref["d_logits"][rows]) <= tol
    assert rel_err(dw_gpu[rows], ref["dw"][rows]) <= tol
    mask = np.zeros(ref["d_logits"].shape, dtype=bool)
    np.put_along_axis(mask, ref["ids"].astype(np.int64), True, axis=1)
    sel = mask[rows]
    assert np.all(dl_gpu[rows][~sel] == 0.0)  # every unselected logit exactly 0
    assert np.all(np.isfinite(dl_gpu[rows][sel]))


@pytest.mark.parametrize("name", list(SMALL) + ["k1", "k32"])
def test_router_backward_given_expert_outputs(name):
    # The kernel alone: seeded per-slot expert outputs placed in y_perm, every row compared.
    cfg = {"k1": inputs.Config("k1", E=8, H=128, I=64, top_k=1, T=70, r=8, alpha=16.0, routing="normal", seed=41),
           "k32": inputs.Config("k32", E=40, H=192, I=64, top_k=32, T=45, r=8, alpha=16.0, routing="normal",
                                seed=42)}.get(name) or SMALL[name]
    prob, d, blk = run(cfg, fwd=False, dgrad=False, wgrad=False)
    ros = check_routing(prob, blk)
    T, E, k, H = cfg.T, cfg.E, cfg.top_k, cfg.H
    yd = inputs.bf16_bits(np.random.default_rng(900 + cfg.seed).standard_normal((T * k, H), dtype=np.float32))
    blk.y_perm[torch.from_numpy(ros).cuda()] = torch.from_numpy(yd.view(np.int16)).cuda().view(torch.bfloat16)
    dl, dw = _router_bwd_gpu(blk, d, T, E, k)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    ref = oracle.topk_softmax_backward(prob.logits, k, dY, inputs.bits_to_f32(yd).astype(np.float64))
    _check_router_rows(dl, dw, ref, np.arange(T), RBWD_TOL)
    if k == 1:
        assert np.all(dl == 0.0)


def test_router_backward_full_size_sampled_tokens():
    # train workload (E128 H2048 top-8, 8192 tokens): the whole launch, sampled rows compared
    cfg = inputs.CONFIGS["train"]
    prob, d, blk = run(cfg, fwd=False, dgrad=False, wgrad=False)
    ros = blk.row_of_slot.cpu().numpy().astype(np.int64)
    T, E, k, H = cfg.T, cfg.E, cfg.top_k, cfg.H
    yd = inputs.bf16_bits(np.random.default_rng(950).standard_normal((T * k, H), dtype=np.float32))
    blk.y_perm[torch.from_numpy(ros).cuda()] = torch.from_numpy(yd.view(np.int16)).cuda().view(torch.bfloat16)
    dl, dw = _router_bwd_gpu(blk, d, T, E, k)
    toks = _sample_tokens(T, 64, 102)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    ref = oracle.topk_softmax_backward(prob.logits, k, dY, {int(f): inputs.bits_to_f32(yd[f]).astype(np.float64)
                                                            for t in toks for f in range(t * k, t * k + k)},
                                       tokens=toks)
    _check_router_rows(dl, dw, ref, toks, RBWD_TOL)
    # properties at any size: every row has at most k nonzeros, all finite, sum ~ 0
    assert np.all(np.isfinite(dl)) and np.all((dl != 0).sum(axis=1) <= k)
    assert np.abs(dl.sum(axis=1)).max() <= 1e-4 * np.abs(dl).max()


@pytest.mark.parametrize("name", ["medium", "stream_zipf_r64"])
def test_router_backward_through_the_forward(name):
    # End to end: the GPU forward's y_perm feeds the router backward; against the oracle's own forward.
    cfg = SMALL[name]
    prob, d, blk = run(cfg, dgrad=False, wgrad=False)
    dl, dw = _router_bwd_gpu(blk, d, cfg.T, cfg.E, cfg.top_k)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    ref = oracle.router_backward(x, prob.logits, dY, oracle_experts(prob), cfg.top_k, cfg.alpha)
    _check_router_rows(dl, dw, ref, np.arange(cfg.T), TOL)


def test_router_backward_train_workload_sampled_tokens():
    cfg = inputs.CONFIGS["train"]
    prob, d, blk = run(cfg, dgrad=False, wgrad=False)
    dl, dw = _router_bwd_gpu(blk, d, cfg.T, cfg.E, cfg.top_k)
    toks = _sample_tokens(cfg.T, 12, 103)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    ref = oracle.router_backward(x, prob.logits, dY, oracle_experts(prob), cfg.top_k, cfg.alpha, tokens=toks)
    _check_router_rows(dl, dw, ref, toks, TOL)


# --------------------------------------------------------------------- serving forward

SERVE = ["tiny", "stream_r24", "stream_zipf_r64", "medium"]  # medium: a prefill-sized batch (training forward)


def _serve(cfg, prob=None, keep_gu=False):
    # keep_gu=False: no gu buffer, as a decode-sized serving call passes it
    prob = prob if prob is not None else inputs.make_problem(cfg)
    d = dv.upload(prob)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    blk.e4b_moe_serve_fwd(d.logits, d.x, d.base(), d.lora(), keep_gu=keep_gu)
    assert blk.check_device_error() == e4b.E4B_OK
    torch.cuda.synchronize()
    return prob, d, blk


def _check_serve_routing(prob, blk):
    cfg = prob.cfg
    ids, w = oracle.route_topk(prob.logits, cfg.top_k)
    g = oracle.group_by_expert(ids, cfg.E)
    assert np.array_equal(blk.topk_ids.cpu().numpy(), ids)
    np.testing.assert_allclose(blk.topk_w.cpu().numpy(), w, rtol=4e-6, atol=1e-7)
    assert np.array_equal(blk.counts.cpu().numpy(), g["counts"])
    offsets = blk.offsets.cpu().numpy().astype(np.int64)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), (g["counts"] + 127) // 128 * 128)
    ros = blk.row_of_slot.cpu().numpy().astype(np.int64)
    assert np.array_equal(ros - offsets[ids.reshape(-1)], g["rank"])
    return ros


@pytest.mark.parametrize("name", SERVE)
def test_serve_forward_parity(name):
    cfg = SMALL[name]
    prob, _, blk = _serve(cfg, keep_gu=(name == "medium"))
    ros = _check_serve_routing(prob, blk)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, oracle_experts(prob), cfg.top_k, cfg.alpha)
    slots = np.arange(cfg.N)
    rows = ros[slots]
    s = cfg.alpha / cfg.r
    errs = {"y": rel_err(f64(blk.y), fo["y"])}
    for key, buf, scale in [("act", blk.act, 1.0), ("p_gu", blk.p_gu, s), ("p_d", blk.p_d, s),
                            ("yd", blk.y_perm, 1.0)]:
        errs[key] = rel_err(f64(buf)[rows], np.stack([fo[key][f] for f in slots]) * scale)
    assert np.array_equal(bits(blk.x_perm)[rows], prob.x[slots // cfg.top_k])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, (bad, errs)


def test_serve_decode_workload_full_and_gu_optional():
    cfg = inputs.CONFIGS["decode"]
    prob = inputs.make_problem(cfg)
    _, _, a = _serve(cfg, prob, keep_gu=False)
    _check_serve_routing(prob, a)
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, oracle_experts(prob), cfg.top_k, cfg.alpha)
    assert rel_err(f64(a.y), fo["y"]) <= TOL
    assert np.all(bits(a.gu) == 0)  # never written without keep_gu
    _, _, b = _serve(cfg, prob, keep_gu=True)
    assert np.array_equal(bits(a.y), bits(b.y))  # gu is a by-product only
    ros = b.row_of_slot.cpu().numpy().astype(np.int64)
    gu = np.stack([fo["gu"][f] for f in range(cfg.N)])
    assert rel_err(f64(b.gu)[ros], gu) <= TOL


def test_serve_forward_cuda_graph_replay_is_bit_identical():
    # the call allocates nothing and never synchronises: capture it once, replay it on new inputs
    cfg = inputs.CONFIGS["decode"]
    p1 = inputs.make_problem(cfg)
    p2 = inputs.make_problem(cfg, data_rank=1)  # another batch over the same weights
    d1, d2 = dv.upload(p1), dv.upload(p2)
    blk = e4b.Block(dv.dims_of(cfg), cfg.T)
    base, lora = d1.base(), d1.lora()
    xs, ls = d1.x.clone(), d1.logits.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        blk.e4b_moe_serve_fwd(ls, xs, base, lora, keep_gu=False)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        blk.e4b_moe_serve_fwd(ls, xs, base, lora, keep_gu=False)
    outs = []
    for d in (d2, d1, d2):
        xs.copy_(d.x)
        ls.copy_(d.logits)
        graph.replay()
        torch.cuda.synchronize()
        outs.append(bits(blk.y).copy())
    eager = []
    for d in (d2, d1):
        blk.e4b_moe_serve_fwd(d.logits, d.x, base, lora, keep_gu=False)
        torch.cuda.synchronize()
        eager.append(bits(blk.y).copy())
    assert blk.check_device_error() == e4b.E4B_OK
    assert np.array_equal(outs[0], eager[0]) and np.array_equal(outs[2], eager[0])
    assert np.array_equal(outs[1], eager[1]) and not np.array_equal(outs[0], outs[1])
    del graph


# --------------------------------------------------------------------- expert parallel (owner side)

def test_expert_parallel_owner_forward_and_backward():
    # The owner's computation for rows it received: top-1 onto the given local experts, weight 1,
    # through the library; each output row must be that expert's output for the row (the oracle's yd).
    from grouped_nf4_expert_b200 import parallel
    cfg = SMALL["medium"]
    prob = inputs.make_problem(cfg)
    d = dv.upload(prob)
    ids, _ = oracle.route_topk(prob.logits, cfg.top_k)
    flat = ids.reshape(-1)
    lo, hi = 2, 6  # this owner's experts
    slots = np.flatnonzero((flat >= lo) & (flat < hi))
    rows = d.x[torch.from_numpy(slots // cfg.top_k).cuda()].contiguous()
    local_ids = torch.from_numpy((flat[slots] - lo).astype(np.int32)).cuda()
    sl = slice(lo, hi)
    base = e4b.nf4_experts(d.gate_up_nf4[sl].contiguous(), d.gate_up_absmax[sl].contiguous(),
                           d.down_nf4[sl].contiguous(), d.down_absmax[sl].contiguous())
    keep = [d.A_gu[sl].contiguous(), d.B_gu[sl].contiguous(), d.A_d[sl].contiguous(), d.B_d[sl].contiguous()]
    blk = parallel.ep_local_forward(e4b.Dims(E=hi - lo, H=cfg.H, I=cfg.I, top_k=1, r=cfg.r, alpha=cfg.alpha),
                                    rows, local_ids, base, e4b.lora_factors(*keep))
    assert blk.check_device_error() == e4b.E4B_OK
    x = inputs.bits_to_f32(prob.x).astype(np.float64)
    fo = oracle.moe_forward(x, prob.logits, oracle_experts(prob), cfg.top_k, cfg.alpha)
    want = np.stack([fo["yd"][int(f)] for f in slots])
    assert rel_err(f64(blk.y), want) <= TOL
    # the owner's backward: received w * dY rows -> each row's input gradient and its experts' gradients
    _, w = oracle.route_topk(prob.logits, cfg.top_k)
    dY = inputs.bits_to_f32(prob.dY).astype(np.float64)
    wf = w.reshape(-1)
    dyw_bits = oracle.bf16_round_bits((wf[slots, None] * dY[slots // cfg.top_k]).astype(np.float32))
    dyw = torch.from_numpy(dyw_bits.view(np.int16)).cuda().view(torch.bfloat16)
    parallel.ep_local_backward(blk, dyw, base, e4b.lora_factors(*keep))
    assert blk.check_device_error() == e4b.E4B_OK
    # the oracle on the same rows: top-1 onto the local experts, weight 1, upstream = the bf16 rows sent
    sub = oracle_experts(prob)
    sub = oracle.Experts(*(getattr(sub, f)[sl] for f in ("gate_up_nf4", "gate_up_absmax", "down_nf4",
                                                          "down_absmax", "A_gu", "B_gu", "A_d", "B_d")))
    lg = np.full((len(slots), hi - lo), -1e30, dtype=np.float32)
    lg[np.arange(len(slots)), flat[slots] - lo] = 0.0
    bo = oracle.moe_backward(x[slots // cfg.top_k], lg, inputs.bits_to_f32(dyw_bits).astype(np.float64), sub, 1,
                             cfg.alpha)
    assert rel_err(f64(blk.dx), bo["dx"]) <= TOL
    for key, buf in [("dA_gu", blk.dA_gu), ("dB_gu", blk.dB_gu), ("dA_d", blk.dA_d), ("dB_d", blk.dB_d)]:
        assert rel_err(f64(buf), bo[key]) <= TOL, key

"""The allocation-free routing entry point agrees with the workspace one.

``e4b_route_permute_noalloc`` serves callers that cannot allocate device
memory (for instance while a CUDA graph is being captured, or inside an engine
plugin limited to pre-planned memory), so it keeps its scratch in a fixed
array inside the library instead of a caller workspace.  This test calls it
through the C ABI twice in a row, on two different batches, and checks each
result against ``e4b_route_permute`` on the same inputs: routing ids, counts,
offsets, permutation and the permuted rows must be identical, and the routing
weights within the parity tests' tolerance (they come out bit-identical).
The work lists in ``tiles`` are compared up to the counts in their header:
entries past the counts are not defined by a routing call.
A third call writes the routing tables only (no permuted rows), through the
binding.  It also checks that a problem too large for the fixed array is refused.
This file is named to be collected after every other test file.
"""

import ctypes

import numpy as np
import pytest
import torch

from grouped_nf4_expert_b200 import build, e4b, inputs
from grouped_nf4_expert_b200 import device as dv

pytestmark = pytest.mark.gpu


def _live_tiles(blk, T, k, E):
    """The entries of the routing work lists that a routing call defines.

    ``tiles`` holds a header ([0] 128-row m-tiles, [1] rows used, [2] 256-row
    m-units, [3] 32-slot streaming tiles) and then four lists sized for the
    largest batch; a call writes each list only up to its count, so entries
    past the counts keep whatever the buffer held before.
    """
    t = blk.tiles.cpu().numpy()
    N = T * k
    mt_cap = (N + 127) // 128 + E
    hdr = 8
    mt_off = hdr
    order_off = hdr + 2 * mt_cap
    mu_off = order_off + E
    st_off = mu_off + 3 * mt_cap
    n_mt, n_mu, n_st = int(t[0]), int(t[2]), int(t[3])
    return {
        "header": t[:4].copy(),
        "m-tiles": t[mt_off:mt_off + 2 * n_mt].copy(),
        "expert order": t[order_off:order_off + E].copy(),
        "m-units": t[mu_off:mu_off + 3 * n_mu].copy(),
        "streaming tiles": t[st_off:st_off + 3 * n_st].copy(),
    }


def _assert_same_tiles(a, b, T, k, E, what):
    la, lb = _live_tiles(a, T, k, E), _live_tiles(b, T, k, E)
    for key in la:
        np.testing.assert_array_equal(la[key], lb[key], err_msg="%s: tiles %s" % (what, key))


def _noalloc_fn():
    fn = e4b.lib().e4b_route_permute_noalloc
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.POINTER(e4b.MoeDims), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.POINTER(e4b.Routing), ctypes.c_void_p, ctypes.c_void_p]
    return fn


def test_noalloc_routing_matches_workspace_routing_twice_in_a_row():
    build.build()
    fn = _noalloc_fn()
    cfg = inputs.CONFIGS["finegrained"]
    dims = dv.dims_of(cfg)
    ref = e4b.Block(dims, cfg.T)   # e4b_route_permute with its workspace
    out = e4b.Block(dims, cfg.T)   # buffers for the allocation-free variant
    stream = torch.cuda.current_stream().cuda_stream
    for batch in (0, 1):           # two calls in a row, different tokens and logits
        prob = inputs.make_problem(cfg, data_rank=batch)
        d = dv.upload(prob)
        ref.e4b_route_permute(d.logits, d.x)
        st = fn(ctypes.byref(out._dims_c), cfg.T, d.logits.data_ptr(), d.x.data_ptr(), ctypes.byref(out._routing),
                out.x_perm.data_ptr(), stream)
        assert st == e4b.E4B_OK, e4b.STATUS.get(st, st)
        torch.cuda.synchronize()
        for name in ("topk_ids", "counts", "offsets", "row_of_slot"):
            assert torch.equal(getattr(out, name), getattr(ref, name)), (batch, name)
        _assert_same_tiles(out, ref, cfg.T, cfg.top_k, cfg.E, "batch %d" % batch)
        used = int(ref.offsets[-1].item())
        assert torch.equal(out.slot_of_row[:used], ref.slot_of_row[:used]), batch
        assert torch.equal(out.x_perm[:used], ref.x_perm[:used]), batch
        np.testing.assert_allclose(out.topk_w.cpu().numpy(), ref.topk_w.cpu().numpy(), rtol=1e-6, atol=0)
    # tables only (no x_perm), through the binding: the same tables again
    tab = e4b.Block(dims, cfg.T)
    tab.e4b_route_permute_noalloc(d.logits, None, gather=False)
    torch.cuda.synchronize()
    for name in ("topk_ids", "counts", "offsets", "row_of_slot"):
        assert torch.equal(getattr(tab, name), getattr(ref, name)), name
    # `tab` is a fresh buffer and `ref` saw two batches: only the defined
    # entries of the work lists are comparable
    _assert_same_tiles(tab, ref, cfg.T, cfg.top_k, cfg.E, "tables only")


def test_noalloc_refuses_problems_beyond_its_fixed_scratch():
    fn = _noalloc_fn()
    dims = e4b.Dims(E=1024, H=64, I=64, top_k=2, r=8, alpha=16.0).c()
    T = 256 * 600   # 2 * ceil(T / tokens-per-routing-block) * 1024 experts > 1,048,576 entries
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    routing = e4b.Routing(*([x.data_ptr()] * 7))
    st = fn(ctypes.byref(dims), T, x.data_ptr(), x.data_ptr(), ctypes.byref(routing), x.data_ptr(), None)
    assert st == e4b.E4B_ERR_UNSUPPORTED

"""The C-ABI library builds, loads and exports what include/e4b.h declares (CPU only).

No compute entry point is called with valid arguments here: every call below
fails host-side validation before any CUDA call, which is what is tested.
"""

import ctypes

import numpy as np
import pytest

from conftest import read_golden_floats
from grouped_nf4_expert_b200 import build as e4b_build
from grouped_nf4_expert_b200 import e4b


@pytest.fixture(scope="module")
def so():
    e4b_build.build()
    return e4b.lib()


def test_exports_every_declared_symbol(so):
    names = e4b.header_symbols()
    assert len(names) >= 12
    for required in ("e4b_route_permute", "e4b_grouped_nf4_lora_fwd", "e4b_grouped_nf4_lora_dgrad",
                     "e4b_lora_wgrad", "e4b_nf4_dequant", "e4b_get_sizes"):
        assert required in names
    for n in names:
        assert hasattr(so, n), n


def test_levels_are_the_published_nf4_table(so):
    lv = np.array(e4b.e4b_nf4_levels(), dtype=np.float32)
    pub = np.array(read_golden_floats("nf4_levels_qlora.txt"), dtype=np.float32)
    assert np.array_equal(lv.view(np.uint32), pub.view(np.uint32))


def test_status_strings(so):
    for code, name in e4b.STATUS.items():
        assert so.e4b_status_string(code).decode().startswith(name)
    assert b"e4b" in so.e4b_version()


def test_sizes_for_the_workloads(so):
    d = e4b.Dims(E=128, H=2048, I=768, top_k=8, r=64, alpha=128.0)
    s = e4b.e4b_get_sizes(d, 8192)
    assert s.slots == 65536
    assert s.rows_cap % 128 == 0 and s.rows_cap >= 65536 + 128 * 127
    assert s.workspace_bytes >= 256
    s0 = e4b.e4b_get_sizes(d, 0)
    assert s0.slots == 0


@pytest.mark.parametrize("field,value,status", [
    ("H", 96, e4b.E4B_ERR_UNSUPPORTED), ("I", 0, e4b.E4B_ERR_UNSUPPORTED), ("top_k", 0, e4b.E4B_ERR_UNSUPPORTED),
    ("top_k", 5, e4b.E4B_ERR_UNSUPPORTED), ("r", 12, e4b.E4B_ERR_UNSUPPORTED), ("r", 72, e4b.E4B_ERR_UNSUPPORTED),
    ("E", 0, e4b.E4B_ERR_UNSUPPORTED), ("E", 2048, e4b.E4B_ERR_UNSUPPORTED),
    ("blocksize", 32, e4b.E4B_ERR_UNSUPPORTED), ("act", 1, e4b.E4B_ERR_UNSUPPORTED),
    ("alpha", float("nan"), e4b.E4B_ERR_INVALID_ARG),
])
def test_bad_dims_are_refused(so, field, value, status):
    d = e4b.MoeDims(4, 64, 128, 2, 8, 16.0, 64, 0)
    setattr(d, field, value)
    out = e4b.Sizes()
    assert so.e4b_get_sizes(ctypes.byref(d), 32, ctypes.byref(out)) == status


def test_negative_tokens_refused(so):
    d = e4b.MoeDims(4, 64, 128, 2, 8, 16.0, 64, 0)
    out = e4b.Sizes()
    assert so.e4b_get_sizes(ctypes.byref(d), -1, ctypes.byref(out)) == e4b.E4B_ERR_INVALID_ARG


def _fake(n=64):
    # Host memory standing in for device pointers: validation reads only the
    # addresses, never the memory, and fails before any CUDA call.
    buf = (ctypes.c_uint8 * (n * 16 + 16))()
    base = (ctypes.addressof(buf) + 15) & ~15
    return buf, [base + 16 * i for i in range(n)]


def test_null_and_misaligned_pointers_refused(so):
    keep, p = _fake()
    d = e4b.MoeDims(4, 64, 128, 2, 8, 16.0, 64, 0)
    T = 32
    sz = e4b.Sizes()
    assert so.e4b_get_sizes(ctypes.byref(d), T, ctypes.byref(sz)) == 0
    routing = e4b.Routing(*p[0:7])
    ws, wsb = p[10], sz.workspace_bytes
    # valid-looking call shape but a null logits pointer
    assert so.e4b_route_permute(ctypes.byref(d), T, None, p[8], ctypes.byref(routing), p[9], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG
    # misaligned x
    assert so.e4b_route_permute(ctypes.byref(d), T, p[7], p[8] + 2, ctypes.byref(routing), p[9], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG
    # workspace too small
    assert so.e4b_route_permute(ctypes.byref(d), T, p[7], p[8], ctypes.byref(routing), p[9], ws, 16,
                                None) == e4b.E4B_ERR_WORKSPACE_TOO_SMALL
    # routing struct with a null member
    bad = e4b.Routing(*p[0:6], None)
    assert so.e4b_route_permute(ctypes.byref(d), T, p[7], p[8], ctypes.byref(bad), p[9], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG
    base = e4b.Nf4Experts(p[11], p[12], None, p[14])
    lora = e4b.Lora(*p[15:19])
    fwd = e4b.FwdBuffers(*p[19:25])
    assert so.e4b_grouped_nf4_lora_fwd(ctypes.byref(d), T, ctypes.byref(routing), ctypes.byref(base),
                                       ctypes.byref(lora), None, ctypes.byref(fwd), p[25], ws, wsb,
                                       None) == e4b.E4B_ERR_INVALID_ARG
    # a misaligned x to gather from
    assert so.e4b_grouped_nf4_lora_fwd(ctypes.byref(d), T, ctypes.byref(routing),
                                       ctypes.byref(e4b.Nf4Experts(*p[11:15])), ctypes.byref(lora), p[8] + 2,
                                       ctypes.byref(fwd), p[25], ws, wsb, None) == e4b.E4B_ERR_INVALID_ARG
    # routing tables only (no x_perm): x is not needed; nothing to do for T == 0
    assert so.e4b_route_permute(ctypes.byref(d), 0, p[7], None, ctypes.byref(routing), None, ws, wsb,
                                None) == e4b.E4B_OK
    # the allocation-free variant validates the same way, before any CUDA call
    na = so.e4b_route_permute_noalloc
    assert na(ctypes.byref(d), 0, None, None, None, None, None) == e4b.E4B_OK
    assert na(ctypes.byref(d), T, p[7], p[8] + 2, ctypes.byref(routing), p[9], None) == e4b.E4B_ERR_INVALID_ARG
    assert na(ctypes.byref(d), T, p[7], None, None, None, None) == e4b.E4B_ERR_INVALID_ARG
    big = e4b.Dims(E=1024, H=64, I=64, top_k=2, r=8, alpha=16.0).c()
    assert na(ctypes.byref(big), 256 * 600, p[7], None, ctypes.byref(routing), None,
              None) == e4b.E4B_ERR_UNSUPPORTED
    bwd = e4b.BwdBuffers(*p[26:30], p[30] + 8)
    base_ok = e4b.Nf4Experts(*p[11:15])
    assert so.e4b_grouped_nf4_lora_dgrad(ctypes.byref(d), T, ctypes.byref(routing), ctypes.byref(base_ok),
                                         ctypes.byref(lora), ctypes.byref(fwd), p[31], ctypes.byref(bwd), p[32],
                                         ws, wsb, None) == e4b.E4B_ERR_INVALID_ARG
    bwd_ok = e4b.BwdBuffers(*p[26:31])
    assert so.e4b_lora_wgrad(ctypes.byref(d), T, ctypes.byref(routing), ctypes.byref(fwd), ctypes.byref(bwd_ok),
                             p[33], None, p[35], p[36], ws, wsb, None) == e4b.E4B_ERR_INVALID_ARG
    # serving forward: gu optional only for decode-sized batches; unaligned inputs; T == 0 launches nothing
    nogu = e4b.FwdBuffers(p[19], p[20], None, p[22], p[23], p[24])
    big = 33  # 66 routed slots > 16 * E
    wsb_big = e4b.Sizes()
    assert so.e4b_get_sizes(ctypes.byref(d), big, ctypes.byref(wsb_big)) == e4b.E4B_OK
    assert wsb_big.workspace_bytes <= wsb
    assert so.e4b_moe_serve_fwd(ctypes.byref(d), big, p[7], p[8], ctypes.byref(routing), ctypes.byref(base_ok),
                                ctypes.byref(lora), ctypes.byref(nogu), p[25], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_moe_serve_fwd(ctypes.byref(d), T, p[7] + 4, p[8], ctypes.byref(routing), ctypes.byref(base_ok),
                                ctypes.byref(lora), ctypes.byref(nogu), p[25], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_moe_serve_fwd(ctypes.byref(d), T, p[7], p[8], ctypes.byref(routing), ctypes.byref(base),
                                ctypes.byref(lora), ctypes.byref(nogu), p[25], ws, wsb,
                                None) == e4b.E4B_ERR_INVALID_ARG  # base with a null member
    assert so.e4b_moe_serve_fwd(ctypes.byref(d), 0, p[7], p[8], ctypes.byref(routing), ctypes.byref(base_ok),
                                ctypes.byref(lora), ctypes.byref(nogu), p[25], ws, wsb, None) == e4b.E4B_OK
    # router backward: unaligned or missing tensors; dw optional; T == 0 launches nothing
    assert so.e4b_router_backward(ctypes.byref(d), T, ctypes.byref(routing), p[24] + 2, p[31], p[37], None,
                                  None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_router_backward(ctypes.byref(d), T, ctypes.byref(routing), p[24], None, p[37], None,
                                  None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_router_backward(ctypes.byref(d), T, ctypes.byref(routing), p[24], p[31], p[37], p[38] + 4,
                                  None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_router_backward(ctypes.byref(d), T, ctypes.byref(bad), p[24], p[31], p[37], None,
                                  None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_router_backward(ctypes.byref(d), 0, ctypes.byref(routing), p[24], p[31], p[37], None,
                                  None) == e4b.E4B_OK
    # unsupported dims are refused before pointers are looked at
    d.r = 12
    assert so.e4b_lora_wgrad(ctypes.byref(d), T, ctypes.byref(routing), ctypes.byref(fwd), ctypes.byref(bwd_ok),
                             p[33], p[34], p[35], p[36], ws, wsb, None) == e4b.E4B_ERR_UNSUPPORTED


def test_dequant_and_watchdog_argument_checks(so):
    keep, p = _fake()
    assert so.e4b_nf4_dequant(p[0], p[1], 100, p[2], None) == e4b.E4B_ERR_INVALID_ARG  # not a multiple of 64
    assert so.e4b_nf4_dequant(p[0] + 1, p[1], 64, p[2], None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_nf4_dequant(p[0], p[1], 0, p[2], None) == e4b.E4B_OK  # nothing to do
    assert so.e4b_nf4_quantize(p[0], 100, p[1], p[2], None) == e4b.E4B_ERR_INVALID_ARG  # not a multiple of 64
    assert so.e4b_nf4_quantize(p[0] + 2, 64, p[1], p[2], None) == e4b.E4B_ERR_INVALID_ARG  # unaligned weights
    assert so.e4b_nf4_quantize(p[0], 64, p[1] + 1, p[2], None) == e4b.E4B_ERR_INVALID_ARG  # unaligned codes
    assert so.e4b_nf4_quantize(p[0], 64, p[1], p[2] + 2, None) == e4b.E4B_ERR_INVALID_ARG  # unaligned absmax
    assert so.e4b_nf4_quantize(p[0], 0, p[1], p[2], None) == e4b.E4B_OK  # nothing to do
    assert so.e4b_debug_watchdog(p[0], 256, 0, None) == e4b.E4B_ERR_INVALID_ARG
    assert so.e4b_debug_watchdog(p[0], 8, 1000, None) == e4b.E4B_ERR_INVALID_ARG


def test_binding_pointer_of_empty_views_is_their_storage_address():
    # torch reports address 0 for empty tensors; the binding passes where the view would start, so
    # that a T = 0 call sees valid (aligned) pointers rather than NULL
    import torch
    buf = torch.zeros(64)
    assert e4b._ptr(buf[:0]) == buf.data_ptr()
    assert e4b._ptr(buf[16:16]) == buf.data_ptr() + 16 * 4
    assert e4b._ptr(buf[4:]) == buf.data_ptr() + 16
    assert e4b._ptr(None) is None


def test_binding_checks_tensors_before_calling_the_library():
    # The binding refuses what raw addresses cannot carry (dtype, layout, size, device) before any
    # library call; CPU tensors exercise every check up to the device one.
    import torch
    n = 256
    packed = torch.zeros(n // 2, dtype=torch.uint8)
    absmax = torch.zeros(n // 64, dtype=torch.float32)
    out = torch.zeros(n, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="out: dtype"):
        e4b.e4b_nf4_dequant(packed, absmax, out.float())
    with pytest.raises(ValueError, match="packed: 64 elements, the call needs 128"):
        e4b.e4b_nf4_dequant(packed[:64], absmax, out)
    with pytest.raises(ValueError, match="absmax: must be contiguous"):
        e4b.e4b_nf4_dequant(packed, torch.zeros(8, dtype=torch.float32)[::2], out)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        e4b.e4b_nf4_dequant(packed, absmax, out)
    with pytest.raises(ValueError, match="w: a tensor is required"):
        e4b.e4b_nf4_quantize(None, packed, absmax)
    with pytest.raises(ValueError, match="absmax: 2 elements, the call needs 4"):
        e4b.e4b_nf4_quantize(out, packed, absmax[:2])
    with pytest.raises(TypeError, match="gate_up_nf4: dtype"):
        e4b.nf4_experts(absmax, absmax, packed, absmax)
    with pytest.raises(TypeError, match="expected a torch.Tensor"):
        e4b.lora_factors(np.zeros(4), out, out, out)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        e4b.lora_factors(out, out, out, out)


def test_binding_checks_struct_sizes_against_the_dims():
    class Fake:  # what nf4_experts / lora_factors record
        _device = "cuda:0"
        _numel = {"A_gu": 100}
    e4b._check_struct(Fake(), {"A_gu": 100}, "cuda:0", "lora")
    with pytest.raises(ValueError, match="lora.A_gu: 100 elements, the dims need 101"):
        e4b._check_struct(Fake(), {"A_gu": 101}, "cuda:0", "lora")
    with pytest.raises(ValueError, match="on cuda:0, the problem is on cuda:1"):
        e4b._check_struct(Fake(), {"A_gu": 1}, "cuda:1", "lora")
    e4b._check_struct(e4b.Lora(), {"A_gu": 10 ** 9}, "cuda:0", "lora")  # built field by field: not checked


def test_binding_signatures_match_the_header_prototypes():
    # every prototype in include/e4b.h has a ctypes signature with the same number of arguments
    import re
    text = re.sub(r"/\*.*?\*/", "", open(e4b.HEADER).read(), flags=re.S)
    protos = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(e4b_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.M | re.S)
    assert len(protos) == len(e4b.header_symbols())
    for name, args in protos:
        a = args.strip()
        n = 0 if a in ("", "void") else a.count(",") + 1
        assert name in e4b._SIGNATURES, name
        assert len(e4b._SIGNATURES[name][1]) == n, name


def test_binding_structs_match_the_header_structs_field_by_field():
    # a field out of order would hand the library one buffer in place of another
    import re
    text = re.sub(r"/\*.*?\*/", "", open(e4b.HEADER).read(), flags=re.S)
    structs = {}
    for body, name in re.findall(r"typedef\s+struct\s*\{(.*?)\}\s*(\w+)\s*;", text, flags=re.S):
        fields = []
        for decl in filter(None, (d.strip() for d in body.split(";"))):
            decl = re.sub(r"\[[^\]]*\]", "", decl)
            fields += [re.findall(r"\w+", part)[-1] for part in decl.split(",")]
        structs[name] = fields
    pairs = {"e4b_moe_dims": e4b.MoeDims, "e4b_nf4_experts": e4b.Nf4Experts, "e4b_lora": e4b.Lora,
             "e4b_routing": e4b.Routing, "e4b_fwd_buffers": e4b.FwdBuffers, "e4b_bwd_buffers": e4b.BwdBuffers,
             "e4b_sizes": e4b.Sizes, "e4b_kernel_time": e4b.KernelTime}
    assert set(structs) == set(pairs)
    for cname, cls in pairs.items():
        assert [f[0] for f in cls._fields_] == structs[cname], cname


def test_buffer_capacities_hold_every_routing_outcome(so):
    # rows_cap and tiles_cap (e4b_get_sizes) must hold the padded groups and the three device work lists
    # for ANY split of the N slots over the E experts; the worst splits leave one slot over a tile edge
    # in as many experts as possible.  Work-list layout: an 8-int header, 2 ints per 128-row m-tile,
    # E ints of expert order, 3 per 256-row m-unit and 3 per 32-slot streaming tile, the m-unit and
    # streaming regions sized 3 and 12 ints per m-tile of capacity.
    rng = np.random.default_rng(5)
    for _ in range(300):
        E = int(rng.integers(1, 1025))
        k = int(rng.integers(1, min(E, 32) + 1))
        T = int(rng.integers(0, 5000))
        N = T * k
        d = e4b.Dims(E=E, H=64, I=64, top_k=k, r=8, alpha=16.0)
        s = e4b.e4b_get_sizes(d, T)
        mt_cap = (s.tiles_cap - 8 - E) // 17
        assert s.tiles_cap == 8 + 17 * mt_cap + E
        splits = [rng.multinomial(N, np.ones(E) / E)]
        worst = np.zeros(E, dtype=np.int64)   # as many experts as possible hold 1 slot past an edge
        m = min(E, N)
        worst[:m] = 1
        worst[0] += N - m
        splits.append(worst)
        for c in splits:
            assert c.sum() == N
            mt = int(((c + 127) // 128).sum())
            mu = int((((c + 127) // 128 + 1) // 2).sum())
            st = int(((c + 31) // 32).sum())
            assert int(((c + 127) // 128 * 128).sum()) <= s.rows_cap
            assert mt <= mt_cap and mu <= mt_cap and st <= 4 * mt_cap


def test_binding_fails_loudly_without_the_library(monkeypatch):
    # no fallback: with libe4b.so absent the binding raises instead of computing anything elsewhere
    monkeypatch.setattr(e4b, "_LIB", None)
    monkeypatch.setattr(e4b, "LIB_PATH", e4b.LIB_PATH + ".missing")
    with pytest.raises(RuntimeError, match="not built"):
        e4b.lib()
    with pytest.raises(RuntimeError, match="not built"):
        e4b.e4b_get_sizes(e4b.Dims(E=4, H=64, I=64, top_k=2, r=8, alpha=16.0), 8)

"""Python binding of the C ABI in ``include/e4b.h`` (ctypes; argument marshalling only).

Every function here forwards to the entry point of the same name in
``libe4b.so``; all computation runs in that library's CUDA kernels.  Tensors
are torch CUDA tensors (PyTorch supplies device memory and streams).  A
non-OK status raises :class:`E4BError`.  There is no fallback: if the library
is missing, :func:`lib` raises.

The library sees raw device addresses only, so before each call the binding
checks what the addresses cannot carry: every tensor is a contiguous CUDA
tensor of the dtype the header names, on one device, holding at least the
elements the call reads or writes (``TypeError`` / ``ValueError`` otherwise).
Alignment, shapes the build refuses and workspace size are the library's own
checks.
"""

from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libe4b.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "e4b.h")

c_i32, c_i64, c_f32, c_vp, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

STATUS = {0: "E4B_OK", 1: "E4B_ERR_INVALID_ARG", 2: "E4B_ERR_UNSUPPORTED",
          3: "E4B_ERR_WORKSPACE_TOO_SMALL", 4: "E4B_ERR_CUDA", 5: "E4B_ERR_DEVICE_TIMEOUT"}
E4B_OK, E4B_ERR_INVALID_ARG, E4B_ERR_UNSUPPORTED = 0, 1, 2
E4B_ERR_WORKSPACE_TOO_SMALL, E4B_ERR_CUDA, E4B_ERR_DEVICE_TIMEOUT = 3, 4, 5
ROW_ALIGN = 128


class E4BError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().e4b_status_string(status).decode()
        super().__init__("%s failed: %s" % (where, msg))


class MoeDims(ctypes.Structure):
    _fields_ = [("E", c_i32), ("H", c_i32), ("I", c_i32), ("top_k", c_i32), ("r", c_i32),
                ("alpha", c_f32), ("blocksize", c_i32), ("act", c_i32)]


class Nf4Experts(ctypes.Structure):
    _fields_ = [("gate_up_nf4", c_vp), ("gate_up_absmax", c_vp), ("down_nf4", c_vp), ("down_absmax", c_vp)]


class Lora(ctypes.Structure):
    _fields_ = [("A_gu", c_vp), ("B_gu", c_vp), ("A_d", c_vp), ("B_d", c_vp)]


class Routing(ctypes.Structure):
    _fields_ = [("topk_ids", c_vp), ("topk_w", c_vp), ("counts", c_vp), ("offsets", c_vp),
                ("row_of_slot", c_vp), ("slot_of_row", c_vp), ("tiles", c_vp)]


class FwdBuffers(ctypes.Structure):
    _fields_ = [("x_perm", c_vp), ("p_gu", c_vp), ("gu", c_vp), ("act", c_vp), ("p_d", c_vp), ("y_perm", c_vp)]


class BwdBuffers(ctypes.Structure):
    _fields_ = [("dyw", c_vp), ("q_d", c_vp), ("dgu", c_vp), ("q_gu", c_vp), ("dx_perm", c_vp)]


class Sizes(ctypes.Structure):
    _fields_ = [("slots", c_i64), ("rows_cap", c_i64), ("tiles_cap", c_i64), ("workspace_bytes", c_sz)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", c_i64), ("total_ms", ctypes.c_double)]


_LIB: Optional[ctypes.CDLL] = None

_SIGNATURES = {
    "e4b_status_string": (ctypes.c_char_p, [c_i32]),
    "e4b_version": (ctypes.c_char_p, []),
    "e4b_nf4_levels": (None, [ctypes.POINTER(c_f32)]),
    "e4b_get_sizes": (c_i32, [ctypes.POINTER(MoeDims), c_i32, ctypes.POINTER(Sizes)]),
    "e4b_workspace_init": (c_i32, [c_vp, c_sz, c_vp]),
    "e4b_check_device_error": (c_i32, [c_vp, c_vp]),
    "e4b_route_permute": (c_i32, [ctypes.POINTER(MoeDims), c_i32, c_vp, c_vp, ctypes.POINTER(Routing), c_vp,
                                  c_vp, c_sz, c_vp]),
    "e4b_route_permute_noalloc": (c_i32, [ctypes.POINTER(MoeDims), c_i32, c_vp, c_vp, ctypes.POINTER(Routing),
                                          c_vp, c_vp]),
    "e4b_grouped_nf4_lora_fwd": (c_i32, [ctypes.POINTER(MoeDims), c_i32, ctypes.POINTER(Routing),
                                         ctypes.POINTER(Nf4Experts), ctypes.POINTER(Lora), c_vp,
                                         ctypes.POINTER(FwdBuffers), c_vp, c_vp, c_sz, c_vp]),
    "e4b_grouped_nf4_lora_dgrad": (c_i32, [ctypes.POINTER(MoeDims), c_i32, ctypes.POINTER(Routing),
                                           ctypes.POINTER(Nf4Experts), ctypes.POINTER(Lora),
                                           ctypes.POINTER(FwdBuffers), c_vp, ctypes.POINTER(BwdBuffers), c_vp,
                                           c_vp, c_sz, c_vp]),
    "e4b_lora_wgrad": (c_i32, [ctypes.POINTER(MoeDims), c_i32, ctypes.POINTER(Routing),
                               ctypes.POINTER(FwdBuffers), ctypes.POINTER(BwdBuffers), c_vp, c_vp, c_vp, c_vp,
                               c_vp, c_sz, c_vp]),
    "e4b_moe_serve_fwd": (c_i32, [ctypes.POINTER(MoeDims), c_i32, c_vp, c_vp, ctypes.POINTER(Routing),
                                  ctypes.POINTER(Nf4Experts), ctypes.POINTER(Lora), ctypes.POINTER(FwdBuffers), c_vp,
                                  c_vp, c_sz, c_vp]),
    "e4b_router_backward": (c_i32, [ctypes.POINTER(MoeDims), c_i32, ctypes.POINTER(Routing), c_vp, c_vp, c_vp,
                                    c_vp, c_vp]),
    "e4b_nf4_dequant": (c_i32, [c_vp, c_vp, c_i64, c_vp, c_vp]),
    "e4b_nf4_quantize": (c_i32, [c_vp, c_i64, c_vp, c_vp, c_vp]),
    "e4b_debug_watchdog": (c_i32, [c_vp, c_sz, c_i64, c_vp]),
    "e4b_profiler_enable": (c_i32, [c_i32]),
    "e4b_profiler_read": (c_i32, [ctypes.POINTER(KernelTime), c_i32, ctypes.POINTER(c_i32)]),
    "e4b_launch_count": (c_i64, []),
}


def lib() -> ctypes.CDLL:
    """Loads ``libe4b.so`` (built in-tree by ``grouped_nf4_expert_b200.build``)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libe4b.so is not built; run `python -m grouped_nf4_expert_b200.build`")
        so = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(so, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = so
    return _LIB


def header_symbols():
    """Names of the entry points ``include/e4b.h`` declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:const\s+)?[\w\s\*]*?\b(e4b_\w+)\s*\(", text, flags=re.M)))


def _check(status: int, where: str):
    if status != E4B_OK:
        raise E4BError(status, where)


def _ptr(t) -> Optional[int]:
    """Device address of a tensor's first element; for an empty view, the address it would have in its
    storage (torch reports 0 for empty tensors)."""
    if t is None:
        return None
    if t.numel() == 0:
        return t.untyped_storage().data_ptr() + t.storage_offset() * t.element_size() or None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _torch_dtype(name):
    import torch
    return {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32, "u8": torch.uint8}[name]


def _dev(t, dtype: str, min_numel: int, name: str, device=None, optional=None, where=True) -> Optional[int]:
    """Device address of ``t`` after checking that it is a contiguous CUDA tensor of ``dtype``
    holding at least ``min_numel`` elements (on ``device`` when given).  ``None`` passes where the
    header allows NULL: by default where nothing is read or written (``min_numel == 0``)."""
    import torch
    if optional is None:
        optional = min_numel == 0
    if t is None:
        if optional:
            return None
        raise ValueError("%s: a tensor is required" % name)
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s: expected a torch.Tensor, got %s" % (name, type(t).__name__))
    if t.dtype != _torch_dtype(dtype):
        raise TypeError("%s: dtype %s, expected %s" % (name, t.dtype, _torch_dtype(dtype)))
    if not t.is_contiguous():
        raise ValueError("%s: must be contiguous" % name)
    if t.numel() < min_numel:
        raise ValueError("%s: %d elements, the call needs %d" % (name, t.numel(), min_numel))
    if not where:  # the caller checks the devices of all its tensors together (_one_cuda_device)
        return _ptr(t)
    if t.device.type != "cuda":
        raise ValueError("%s: must be a CUDA tensor, got one on %s" % (name, t.device))
    if device is not None and t.device != device:
        raise ValueError("%s: on %s, expected %s" % (name, t.device, device))
    return _ptr(t)


def _numel_of(t, name: str) -> int:
    import torch
    if t is None:
        raise ValueError("%s: a tensor is required" % name)
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s: expected a torch.Tensor, got %s" % (name, type(t).__name__))
    return t.numel()


def _one_cuda_device(**tensors):
    """The one CUDA device that all the given tensors are on (None entries are skipped)."""
    devs = set()
    for name, t in tensors.items():
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError("%s: must be a CUDA tensor, got one on %s" % (name, t.device))
        devs.add(t.device)
    if len(devs) > 1:
        raise ValueError("tensors on several devices: %s" % sorted(str(d) for d in devs))
    return devs.pop() if devs else None


@dataclass(frozen=True)
class Dims:
    E: int
    H: int
    I: int  # noqa: E741
    top_k: int
    r: int
    alpha: float

    def c(self) -> MoeDims:
        return MoeDims(self.E, self.H, self.I, self.top_k, self.r, float(self.alpha), 64, 0)


def e4b_get_sizes(dims: Dims, T: int) -> Sizes:
    out = Sizes()
    d = dims.c()
    _check(lib().e4b_get_sizes(ctypes.byref(d), T, ctypes.byref(out)), "e4b_get_sizes")
    return out


def e4b_nf4_levels():
    buf = (c_f32 * 16)()
    lib().e4b_nf4_levels(buf)
    return [buf[i] for i in range(16)]


def e4b_workspace_init(ws, stream=None):
    p = _dev(ws, "u8", 1, "ws")
    _check(lib().e4b_workspace_init(p, ws.numel(), _stream(stream)), "e4b_workspace_init")


def e4b_check_device_error(ws, stream=None) -> int:
    """Synchronises the stream; returns the status (does not raise)."""
    return lib().e4b_check_device_error(_dev(ws, "u8", 1, "ws"), _stream(stream))


def e4b_nf4_dequant(packed, absmax, out, stream=None):
    """packed NF4 codes [n/2] u8 and absmax [n/64] f32 -> bf16 [n] (n = out.numel())."""
    n = _numel_of(out, "out")
    pp = _dev(packed, "u8", n // 2, "packed", where=False)
    pa = _dev(absmax, "f32", n // 64, "absmax", where=False)
    po = _dev(out, "bf16", 0, "out", optional=False, where=False)
    _one_cuda_device(packed=packed, absmax=absmax, out=out)
    _check(lib().e4b_nf4_dequant(pp, pa, n, po, _stream(stream)), "e4b_nf4_dequant")


def e4b_nf4_quantize(w, packed, absmax, stream=None):
    """bf16 weights (n elements, n % 64 == 0) -> packed NF4 codes [n/2] u8 and absmax [n/64] f32."""
    n = _numel_of(w, "w")
    pp = _dev(packed, "u8", n // 2, "packed", where=False)
    pa = _dev(absmax, "f32", n // 64, "absmax", where=False)
    pw = _dev(w, "bf16", 0, "w", optional=False, where=False)
    _one_cuda_device(w=w, packed=packed, absmax=absmax)
    _check(lib().e4b_nf4_quantize(pw, n, pp, pa, _stream(stream)), "e4b_nf4_quantize")


def e4b_debug_watchdog(ws, timeout_ns: int, stream=None):
    p = _dev(ws, "u8", 1, "ws")
    _check(lib().e4b_debug_watchdog(p, ws.numel(), int(timeout_ns), _stream(stream)), "e4b_debug_watchdog")


def e4b_profiler_enable(on: bool):
    _check(lib().e4b_profiler_enable(1 if on else 0), "e4b_profiler_enable")


def e4b_profiler_read():
    """Per-kernel {name: (launches, total_ms)} recorded since the last read (waits for the events)."""
    cap = 64
    buf = (KernelTime * cap)()
    n = c_i32(0)
    _check(lib().e4b_profiler_read(buf, cap, ctypes.byref(n)), "e4b_profiler_read")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n.value, cap))}


def e4b_launch_count() -> int:
    return int(lib().e4b_launch_count())


class Block:
    """Device buffers of one block problem (``dims``, ``T`` tokens), allocated with torch.

    Holds the routing arrays, the forward activations, the backward
    intermediates, the workspace and the outputs, laid out as ``include/e4b.h``
    requires, and calls the four entry points on them.
    """

    def __init__(self, dims: Dims, T: int, device="cuda"):
        import torch
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.dims, self.T, self.device = dims, T, dev
        sz = e4b_get_sizes(dims, T)
        self.sizes = sz
        E, H, I, k, r = dims.E, dims.H, dims.I, dims.top_k, dims.r
        R = sz.rows_cap
        dev = self.device

        def z(shape, dtype):
            n = 1
            for s in shape:
                n *= s
            return torch.zeros(max(n, 8), dtype=dtype, device=dev)[:n].view(*shape)

        bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
        self.topk_ids, self.topk_w = z((T, k), i32), z((T, k), f32)
        self.counts, self.offsets = z((E,), i32), z((E + 1,), i32)
        self.row_of_slot, self.slot_of_row, self.tiles = z((T * k,), i32), z((R,), i32), z((sz.tiles_cap,), i32)
        self.x_perm, self.p_gu, self.gu = z((R, H), bf), z((R, r), bf), z((R, 2 * I), bf)
        self.act, self.p_d, self.y_perm = z((R, I), bf), z((R, r), bf), z((R, H), bf)
        self.dyw, self.q_d, self.dgu = z((R, H), bf), z((R, r), bf), z((R, 2 * I), bf)
        self.q_gu, self.dx_perm = z((R, r), bf), z((R, H), bf)
        self.y, self.dx = z((T, H), bf), z((T, H), bf)
        # the four LoRA gradients are views of one flat buffer, so that a data-parallel step sums them
        # with one collective and no packing copy (every size is a multiple of 8 elements: r % 8 == 0)
        gshapes = ((E, r, H), (E, 2 * I, r), (E, r, I), (E, H, r))
        gsizes = [a * b * c for a, b, c in gshapes]
        self.lora_grads = z((sum(gsizes),), bf)
        views, o = [], 0
        for shp, n in zip(gshapes, gsizes):
            views.append(self.lora_grads[o:o + n].view(*shp))
            o += n
        self.dA_gu, self.dB_gu, self.dA_d, self.dB_d = views
        self.ws = z((int(sz.workspace_bytes),), torch.uint8)
        e4b_workspace_init(self.ws)
        self._dims_c = dims.c()
        self._routing = Routing(*(_ptr(t) for t in (self.topk_ids, self.topk_w, self.counts, self.offsets,
                                                      self.row_of_slot, self.slot_of_row, self.tiles)))
        self._fwd = FwdBuffers(*(_ptr(t) for t in (self.x_perm, self.p_gu, self.gu, self.act, self.p_d,
                                                    self.y_perm)))
        self._fwd_nogu = FwdBuffers(self.x_perm.data_ptr(), self.p_gu.data_ptr(), None, self.act.data_ptr(),
                                    self.p_d.data_ptr(), self.y_perm.data_ptr())
        self._bwd = BwdBuffers(*(t.data_ptr() for t in (self.dyw, self.q_d, self.dgu, self.q_gu, self.dx_perm)))

    # -- argument checks (see the module docstring) ----------------------------
    def _rows(self, t, dtype, cols, name, required=True):
        """A [T, cols] token tensor of this problem (at least T * cols elements)."""
        return _dev(t, dtype, self.T * cols, name, self.device, optional=not required or self.T == 0)

    def _base(self, base: Nf4Experts):
        """The NF4 base struct; when made by :func:`nf4_experts`, its sizes and device are checked
        against this problem."""
        d = self.dims
        need = {"gate_up_nf4": d.E * 2 * d.I * d.H // 2, "gate_up_absmax": d.E * 2 * d.I * d.H // 64,
                "down_nf4": d.E * d.H * d.I // 2, "down_absmax": d.E * d.H * d.I // 64}
        _check_struct(base, need, self.device, "base")
        return ctypes.byref(base)

    def _lora(self, lora: Lora):
        d = self.dims
        need = {"A_gu": d.E * d.r * d.H, "B_gu": d.E * 2 * d.I * d.r, "A_d": d.E * d.r * d.I,
                "B_d": d.E * d.H * d.r}
        _check_struct(lora, need, self.device, "lora")
        return ctypes.byref(lora)

    # -- the four hot-path calls -------------------------------------------------
    def e4b_route_permute(self, logits, x, gather=True, stream=None):
        """Routing tables; with ``gather`` also ``x_perm`` (else the forward gathers, given ``x``)."""
        pl = self._rows(logits, "f32", self.dims.E, "logits")
        px = self._rows(x, "bf16", self.dims.H, "x", required=gather)
        _check(lib().e4b_route_permute(ctypes.byref(self._dims_c), self.T, pl, px,
                                       ctypes.byref(self._routing), _ptr(self.x_perm) if gather else None,
                                       _ptr(self.ws), self.ws.numel(), _stream(stream)), "e4b_route_permute")

    def e4b_route_permute_noalloc(self, logits, x, gather=True, stream=None):
        """As ``e4b_route_permute``, with the library's fixed scratch instead of ``ws`` (capturable in
        a global-mode CUDA graph once a first call on the device has been made)."""
        pl = self._rows(logits, "f32", self.dims.E, "logits")
        px = self._rows(x, "bf16", self.dims.H, "x", required=gather)
        _check(lib().e4b_route_permute_noalloc(ctypes.byref(self._dims_c), self.T, pl, px,
                                               ctypes.byref(self._routing), _ptr(self.x_perm) if gather else None,
                                               _stream(stream)), "e4b_route_permute_noalloc")

    def e4b_grouped_nf4_lora_fwd(self, base: Nf4Experts, lora: Lora, x=None, stream=None):
        """Forward; with ``x`` the call also writes ``x_perm`` (fused with the first projection)."""
        px = self._rows(x, "bf16", self.dims.H, "x", required=False)
        _check(lib().e4b_grouped_nf4_lora_fwd(ctypes.byref(self._dims_c), self.T, ctypes.byref(self._routing),
                                              self._base(base), self._lora(lora), px,
                                              ctypes.byref(self._fwd), _ptr(self.y), _ptr(self.ws),
                                              self.ws.numel(), _stream(stream)), "e4b_grouped_nf4_lora_fwd")

    def e4b_grouped_nf4_lora_dgrad(self, base: Nf4Experts, lora: Lora, dY, stream=None):
        pdy = self._rows(dY, "bf16", self.dims.H, "dY")
        _check(lib().e4b_grouped_nf4_lora_dgrad(ctypes.byref(self._dims_c), self.T, ctypes.byref(self._routing),
                                                self._base(base), self._lora(lora), ctypes.byref(self._fwd),
                                                pdy, ctypes.byref(self._bwd), _ptr(self.dx), _ptr(self.ws),
                                                self.ws.numel(), _stream(stream)), "e4b_grouped_nf4_lora_dgrad")

    def e4b_lora_wgrad(self, stream=None):
        _check(lib().e4b_lora_wgrad(ctypes.byref(self._dims_c), self.T, ctypes.byref(self._routing),
                                    ctypes.byref(self._fwd), ctypes.byref(self._bwd), _ptr(self.dA_gu),
                                    _ptr(self.dB_gu), _ptr(self.dA_d), _ptr(self.dB_d), _ptr(self.ws),
                                    self.ws.numel(), _stream(stream)), "e4b_lora_wgrad")

    def e4b_moe_serve_fwd(self, logits, x, base: Nf4Experts, lora: Lora, keep_gu=None, stream=None):
        """Routing + forward for inference into ``self.y``.  ``keep_gu=False`` passes no gu buffer,
        which the call allows for decode-sized batches only (at most 16 * E routed slots; larger ones
        run the training forward, which writes gu); ``None`` keeps gu exactly when it is required."""
        if keep_gu is None:
            keep_gu = self.T * self.dims.top_k > 16 * self.dims.E
        fwd = self._fwd if keep_gu else self._fwd_nogu
        pl = self._rows(logits, "f32", self.dims.E, "logits")
        px = self._rows(x, "bf16", self.dims.H, "x")
        _check(lib().e4b_moe_serve_fwd(ctypes.byref(self._dims_c), self.T, pl, px,
                                       ctypes.byref(self._routing), self._base(base), self._lora(lora),
                                       ctypes.byref(fwd), _ptr(self.y), _ptr(self.ws), self.ws.numel(),
                                       _stream(stream)), "e4b_moe_serve_fwd")

    def e4b_router_backward(self, dY, d_logits, dw=None, stream=None):
        pdy = self._rows(dY, "bf16", self.dims.H, "dY")
        pdl = self._rows(d_logits, "f32", self.dims.E, "d_logits")
        pdw = self._rows(dw, "f32", self.dims.top_k, "dw", required=False)
        _check(lib().e4b_router_backward(ctypes.byref(self._dims_c), self.T, ctypes.byref(self._routing),
                                         _ptr(self.y_perm), pdy, pdl, pdw, _stream(stream)),
               "e4b_router_backward")

    def check_device_error(self, stream=None) -> int:
        return e4b_check_device_error(self.ws, stream)


def _make_struct(cls, tensors, dtypes):
    """A pointer struct over contiguous CUDA tensors on one device.  The struct keeps the tensors
    alive (it holds their raw addresses) and records their sizes for the calls' checks."""
    names = [f[0] for f in cls._fields_]
    st = cls(*(_dev(t, dt, 1, n, where=False) for t, dt, n in zip(tensors, dtypes, names)))
    dev = _one_cuda_device(**dict(zip(names, tensors)))
    st._keep, st._device = tuple(tensors), dev
    st._numel = {n: t.numel() for n, t in zip(names, tensors)}
    return st


def _check_struct(st, need, device, what):
    """Sizes and device of a struct made by :func:`nf4_experts` / :func:`lora_factors` against a
    problem (a struct built field by field carries no sizes and is passed as is)."""
    numel = getattr(st, "_numel", None)
    if numel is None:
        return
    if st._device != device:
        raise ValueError("%s: tensors on %s, the problem is on %s" % (what, st._device, device))
    for name, n in need.items():
        if numel[name] < n:
            raise ValueError("%s.%s: %d elements, the dims need %d" % (what, name, numel[name], n))


def nf4_experts(gate_up_nf4, gate_up_absmax, down_nf4, down_absmax) -> Nf4Experts:
    """The frozen NF4 base: codes u8 [E,2I,H/2] and [E,H,I/2], block absmax f32 [E,2I,H/64] and
    [E,H,I/64]."""
    return _make_struct(Nf4Experts, (gate_up_nf4, gate_up_absmax, down_nf4, down_absmax), ("u8", "f32", "u8", "f32"))


def lora_factors(A_gu, B_gu, A_d, B_d) -> Lora:
    """The per-expert LoRA factors, bf16 [E,r,H], [E,2I,r], [E,r,I], [E,H,r]."""
    return _make_struct(Lora, (A_gu, B_gu, A_d, B_d), ("bf16",) * 4)

"""Python binding of libafd_ffn.so, the FFN-service MoE layer of Attention-FFN Disaggregation
on one B200.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.  The
functions below carry the C names of include/afd_ffn.h and return its status codes; the
``AfdFfn`` class wraps a handle, keeps the borrowed weight tensors alive, and raises
``AfdError`` on a non-zero status.  torch is used only for device memory and streams.

Importing fails (ImportError) when the library has not been built:
``python ffn_side_expert_b200/build.py``.  There is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libafd_ffn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "afd_ffn.h")

AFD_OK = 0
AFD_ERR_INVALID_ARG = -1
AFD_ERR_UNSUPPORTED = -2
AFD_ERR_T_TOO_LARGE = -3
AFD_ERR_CUDA = -4
AFD_ERR_DEVICE_FLAG = -5
AFD_ERR_DEVICE_TIMEOUT = -6
AFD_ERR_NO_DEVICE = -7
AFD_ERR_TIMEOUT = -8
AFD_ERR_STOPPED = -9
AFD_MAILBOX_PINNED = 1
AFD_DT_BF16 = 0
AFD_DT_FP8_E4M3 = 1
AFD_FFN_NUM_STAGES = 9
STAGE_NAMES = ("router_logits", "router_topk", "dispatch_order", "gather_rows", "gemm_schedule",
               "gemm_gate_up", "quantize_act", "gemm_down", "combine")


class afd_ffn_cfg(ctypes.Structure):
    _fields_ = [("T_max", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("weight_dtype", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("has_router_bias", ctypes.c_int32)]


class afd_ffn_weights(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w13", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("w13_scale", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p)]


class afd_ffn_service_stats(ctypes.Structure):
    _fields_ = [("served", ctypes.c_int64), ("status", ctypes.c_int32), ("device_status", ctypes.c_int32),
                ("last_cuda_error", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_L = ctypes.c_int64
_SIGNATURES = {
    "afd_ffn_create": (ctypes.c_int, [ctypes.POINTER(afd_ffn_cfg), ctypes.POINTER(afd_ffn_weights),
                                      ctypes.POINTER(ctypes.c_void_p)]),
    "afd_ffn_create_ex": (ctypes.c_int, [ctypes.POINTER(afd_ffn_cfg), ctypes.POINTER(afd_ffn_weights),
                                         ctypes.c_uint32, ctypes.POINTER(ctypes.c_void_p)]),
    "afd_ffn_destroy": (None, [_P]),
    "afd_ffn_route": (ctypes.c_int, [_P, _P, _I, _P, _P, _P]),
    "afd_ffn_permute": (ctypes.c_int, [_P, _P, _P, _I, _P, _P, _P, _P, _P]),
    "afd_ffn_expert_gemm": (ctypes.c_int, [_P, _P, _I, _P, _P, _P]),
    "afd_ffn_combine": (ctypes.c_int, [_P, _P, _P, _I, _P, _P]),
    "afd_ffn_forward": (ctypes.c_int, [_P, _P, _I, _P, _P]),
    "afd_ffn_forward_host": (ctypes.c_int, [_P, _P, _I, _P, _P]),
    "afd_ffn_forward_host_batches": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_void_p),
                                                    ctypes.POINTER(ctypes.c_void_p), _I, _I, _P]),
    "afd_ffn_set_stage_events": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_void_p), _I]),
    "afd_ffn_get_error": (ctypes.c_int, [_P]),
    "afd_ffn_last_cuda_error": (ctypes.c_int, [_P]),
    "afd_ffn_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "afd_ffn_route_static": (ctypes.c_int, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "afd_ffn_dispatch_rows": (ctypes.c_int, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "afd_ffn_expert_rows": (ctypes.c_int, [_P, _P, _P, _I, _P, _P]),
    "afd_ffn_copy_row_blocks": (ctypes.c_int, [_P, _P, _P, _I, _I, _P]),
    "afd_ffn_combine_rows": (ctypes.c_int, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "afd_ffn_dispatch_rows_fp8": (ctypes.c_int, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "afd_ffn_expert_rows_fp8": (ctypes.c_int, [_P, _P, _P, _P, _I, _P, _P]),
    "afd_ffn_combine_rows_bf16": (ctypes.c_int, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "afd_ffn_rows_error": (ctypes.c_int, []),
    "afd_ffn_get_info": (ctypes.c_int, [_P, ctypes.POINTER(afd_ffn_cfg), ctypes.POINTER(ctypes.c_int32)]),
    "afd_ffn_check_bounded_wait": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int64)]),
    "afd_ffn_mailbox_create": (ctypes.c_int, [_I, _I, _I, _I, ctypes.POINTER(ctypes.c_void_p)]),
    "afd_ffn_mailbox_destroy": (None, [_P]),
    "afd_ffn_mailbox_input": (_P, [_P, _I]),
    "afd_ffn_mailbox_output": (_P, [_P, _I]),
    "afd_ffn_mailbox_post": (ctypes.c_int, [_P, _I, _I]),
    "afd_ffn_mailbox_wait": (ctypes.c_int, [_P, _I, _L]),
    "afd_ffn_mailbox_take": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), _L]),
    "afd_ffn_mailbox_complete": (ctypes.c_int, [_P, _I, _I]),
    "afd_ffn_mailbox_times": (ctypes.c_int, [_P, _I, ctypes.POINTER(ctypes.c_int64)]),
    "afd_ffn_service_start": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(ctypes.c_void_p)]),
    "afd_ffn_service_stop": (ctypes.c_int, [_P, ctypes.POINTER(afd_ffn_service_stats)]),
    "afd_ffn_service_slot_timeline": (ctypes.c_int, [_P, _I, ctypes.POINTER(ctypes.c_float)]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python ffn_side_expert_b200/build.py` "
                          "(the layer has no CPU or library fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def declared_functions(header: str = HEADER_PATH) -> list:
    """Names of the entry points declared in include/afd_ffn.h."""
    with open(header) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(afd_ffn_\w+)\s*\(", text)))


class AfdError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {afd_ffn_strerror(status)} ({status})")


# ------------------------------------------------------------------ marshalling helpers
def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ------------------------------------------------------------------ C entry points
def afd_ffn_strerror(status: int) -> str:
    return _lib.afd_ffn_strerror(status).decode()


def afd_ffn_create(cfg: afd_ffn_cfg, weights: afd_ffn_weights):
    """Returns (status, handle or None)."""
    h = ctypes.c_void_p()
    st = _lib.afd_ffn_create(ctypes.byref(cfg) if cfg is not None else None,
                             ctypes.byref(weights) if weights is not None else None, ctypes.byref(h))
    return st, (h.value if st == AFD_OK else None)


AFD_CREATE_NO_W2_COPY = 1


def afd_ffn_create_ex(cfg: afd_ffn_cfg, weights: afd_ffn_weights, flags: int):
    """Returns (status, handle or None)."""
    h = ctypes.c_void_p()
    st = _lib.afd_ffn_create_ex(ctypes.byref(cfg) if cfg is not None else None,
                                ctypes.byref(weights) if weights is not None else None, flags, ctypes.byref(h))
    return st, (h.value if st == AFD_OK else None)


def afd_ffn_destroy(h) -> None:
    _lib.afd_ffn_destroy(h)


def afd_ffn_route(h, hidden, T, topk_idx, topk_w, stream=None) -> int:
    return _lib.afd_ffn_route(h, _ptr(hidden), T, _ptr(topk_idx), _ptr(topk_w), _stream(stream))


def afd_ffn_permute(h, hidden, topk_idx, T, counts, offsets, pos, src, stream=None) -> int:
    return _lib.afd_ffn_permute(h, _ptr(hidden), _ptr(topk_idx), T, _ptr(counts), _ptr(offsets), _ptr(pos),
                                _ptr(src), _stream(stream))


def afd_ffn_expert_gemm(h, offsets, T, Y=None, Ys=None, stream=None) -> int:
    return _lib.afd_ffn_expert_gemm(h, _ptr(offsets), T, _ptr(Y), _ptr(Ys), _stream(stream))


def afd_ffn_combine(h, topk_w, pos, T, out, stream=None) -> int:
    return _lib.afd_ffn_combine(h, _ptr(topk_w), _ptr(pos), T, _ptr(out), _stream(stream))


def afd_ffn_forward(h, hidden, T, out, stream=None) -> int:
    return _lib.afd_ffn_forward(h, _ptr(hidden), T, _ptr(out), _stream(stream))


def afd_ffn_forward_host(h, hidden_host, T, out_host, stream=None) -> int:
    return _lib.afd_ffn_forward_host(h, _ptr(hidden_host), T, _ptr(out_host), _stream(stream))


def afd_ffn_forward_host_batches(h, hidden_host_list, out_host_list, T, stream=None) -> int:
    """hidden_host_list / out_host_list: sequences of pinned host tensors [T, H] bf16."""
    n = len(hidden_host_list)
    ins = (ctypes.c_void_p * max(n, 1))(*[_ptr(x) for x in hidden_host_list])
    outs = (ctypes.c_void_p * max(n, 1))(*[_ptr(x) for x in out_host_list])
    return _lib.afd_ffn_forward_host_batches(h, ins, outs, n, T, _stream(stream))


def afd_ffn_set_stage_events(h, events) -> int:
    """events: sequence of torch.cuda.Event or None entries (AFD_FFN_NUM_STAGES + 1 of them; a
    None entry skips that stage boundary), or None to turn stage events off.

    torch creates an event's CUDA handle at its first record; events not yet created are
    recorded once on the current stream here so that the library receives real handles.
    """
    if not events:
        return _lib.afd_ffn_set_stage_events(h, None, 0)
    for e in events:
        if e is not None and not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event if e is not None else None for e in events])
    return _lib.afd_ffn_set_stage_events(h, arr, len(events))


def afd_ffn_get_error(h) -> int:
    return _lib.afd_ffn_get_error(h)


def afd_ffn_last_cuda_error(h) -> int:
    return _lib.afd_ffn_last_cuda_error(h)


def afd_ffn_route_static(hidden, router_w, router_bias, T, H, E, k, topk_idx, topk_w, stream=None) -> int:
    """Router without a handle or any allocation (scratch in a static device array); see the
    declaration in include/afd_ffn.h for the size limit and the first-call set-up."""
    return _lib.afd_ffn_route_static(_ptr(hidden), _ptr(router_w), _ptr(router_bias), T, H, E, k,
                                     _ptr(topk_idx), _ptr(topk_w), _stream(stream))


AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS = 1 << 20


# expert-parallel building blocks (declarations in include/afd_ffn.h)
def afd_ffn_dispatch_rows(hidden, topk_idx, T, k, E, H, counts, offsets, pos, src, rows, scratch,
                          stream=None) -> int:
    return _lib.afd_ffn_dispatch_rows(_ptr(hidden), _ptr(topk_idx), T, k, E, H, _ptr(counts), _ptr(offsets),
                                      _ptr(pos), _ptr(src), _ptr(rows), _ptr(scratch), _stream(stream))


def afd_ffn_expert_rows(h, rows, counts, n_rows, Y, stream=None) -> int:
    return _lib.afd_ffn_expert_rows(h, _ptr(rows), _ptr(counts), n_rows, _ptr(Y), _stream(stream))


def afd_ffn_copy_row_blocks(src, dst, blocks, n_blocks, row_bytes, stream=None) -> int:
    return _lib.afd_ffn_copy_row_blocks(_ptr(src), _ptr(dst), _ptr(blocks), n_blocks, row_bytes, _stream(stream))


def afd_ffn_dispatch_rows_fp8(hidden, topk_idx, T, k, E, H, with_shared, counts, offsets, pos, src, rows,
                              row_scale, scratch, stream=None) -> int:
    return _lib.afd_ffn_dispatch_rows_fp8(_ptr(hidden), _ptr(topk_idx), T, k, E, H, with_shared, _ptr(counts),
                                          _ptr(offsets), _ptr(pos), _ptr(src), _ptr(rows), _ptr(row_scale),
                                          _ptr(scratch), _stream(stream))


def afd_ffn_expert_rows_fp8(h, rows, row_scale, counts, n_rows, Y, stream=None) -> int:
    return _lib.afd_ffn_expert_rows_fp8(h, _ptr(rows), _ptr(row_scale), _ptr(counts), n_rows, _ptr(Y),
                                        _stream(stream))


def afd_ffn_combine_rows_bf16(Y, Ys, topk_w, pos, T, k, H, out, stream=None) -> int:
    return _lib.afd_ffn_combine_rows_bf16(_ptr(Y), _ptr(Ys), _ptr(topk_w), _ptr(pos), T, k, H, _ptr(out),
                                          _stream(stream))


def afd_ffn_combine_rows(Y, Ys, topk_w, pos, T, k, H, out, stream=None) -> int:
    return _lib.afd_ffn_combine_rows(_ptr(Y), _ptr(Ys), _ptr(topk_w), _ptr(pos), T, k, H, _ptr(out),
                                     _stream(stream))


def afd_ffn_rows_error() -> int:
    return _lib.afd_ffn_rows_error()


def afd_ffn_check_bounded_wait():
    """Returns (status, SM cycles the wait took); AFD_ERR_DEVICE_TIMEOUT is the expected status."""
    cycles = ctypes.c_int64(0)
    st = _lib.afd_ffn_check_bounded_wait(ctypes.byref(cycles))
    return st, cycles.value


def afd_ffn_get_info(h):
    """Returns (status, afd_ffn_cfg, device)."""
    cfg, dev = afd_ffn_cfg(), ctypes.c_int32(-1)
    st = _lib.afd_ffn_get_info(h, ctypes.byref(cfg), ctypes.byref(dev))
    return st, cfg, dev.value


# FFN service: mailbox and serving loop (declarations in include/afd_ffn.h)
def afd_ffn_mailbox_create(n_slots, T_max, H, flags=0):
    """Returns (status, mailbox or None)."""
    mb = ctypes.c_void_p()
    st = _lib.afd_ffn_mailbox_create(n_slots, T_max, H, flags, ctypes.byref(mb))
    return st, (mb.value if st == AFD_OK else None)


def afd_ffn_mailbox_destroy(mb) -> None:
    _lib.afd_ffn_mailbox_destroy(mb)


def afd_ffn_mailbox_input(mb, slot):
    return _lib.afd_ffn_mailbox_input(mb, slot)


def afd_ffn_mailbox_output(mb, slot):
    return _lib.afd_ffn_mailbox_output(mb, slot)


def afd_ffn_mailbox_post(mb, slot, T) -> int:
    return _lib.afd_ffn_mailbox_post(mb, slot, T)


def afd_ffn_mailbox_wait(mb, slot, timeout_us) -> int:
    return _lib.afd_ffn_mailbox_wait(mb, slot, timeout_us)


def afd_ffn_mailbox_take(mb, timeout_us):
    """Returns (status, slot, T)."""
    slot, T = ctypes.c_int32(-1), ctypes.c_int32(-1)
    st = _lib.afd_ffn_mailbox_take(mb, ctypes.byref(slot), ctypes.byref(T), timeout_us)
    return st, slot.value, T.value


def afd_ffn_mailbox_complete(mb, slot, status) -> int:
    return _lib.afd_ffn_mailbox_complete(mb, slot, status)


def afd_ffn_mailbox_times(mb, slot):
    """Returns (status, (post_ns, take_ns, done_ns))."""
    t = (ctypes.c_int64 * 3)()
    st = _lib.afd_ffn_mailbox_times(mb, slot, t)
    return st, tuple(t)


def afd_ffn_service_start(h, mb, stream=None):
    """Returns (status, service or None)."""
    svc = ctypes.c_void_p()
    st = _lib.afd_ffn_service_start(h, mb, _stream(stream), ctypes.byref(svc))
    return st, (svc.value if st == AFD_OK else None)


def afd_ffn_service_slot_timeline(svc, slot):
    """Returns (status, (origin->H2D start, H2D end, layer start, layer end, D2H end)) in ms,
    the last four from the H2D start."""
    ms = (ctypes.c_float * 5)()
    st = _lib.afd_ffn_service_slot_timeline(svc, slot, ms)
    return st, tuple(ms)


def afd_ffn_service_stop(svc):
    """Returns (status, afd_ffn_service_stats)."""
    stats = afd_ffn_service_stats()
    st = _lib.afd_ffn_service_stop(svc, ctypes.byref(stats))
    return st, stats


# ------------------------------------------------------------------ convenience wrapper
class AfdFfn:
    """A handle on the current CUDA device.

    weights: dict with device tensors router_w [E,H] fp32, optional router_bias [E] fp32,
    w13 [E+S,2I,H] and w2 [E+S,H,I] (bf16 or float8_e4m3fn), and for e4m3 w13_scale [E+S,2I],
    w2_scale [E+S,H] fp32.  The tensors are referenced for the handle's lifetime.
    """

    def __init__(self, *, T_max, H, E, k, I, n_shared, fp8, weights, flags=0):
        dt = AFD_DT_FP8_E4M3 if fp8 else AFD_DT_BF16
        self.cfg = afd_ffn_cfg(T_max, H, E, k, I, n_shared, dt, dt,
                               1 if weights.get("router_bias") is not None else 0)
        self._keep = dict(weights)
        w = afd_ffn_weights(_ptr(weights["router_w"]), _ptr(weights.get("router_bias")),
                            _ptr(weights["w13"]), _ptr(weights["w2"]),
                            _ptr(weights.get("w13_scale")), _ptr(weights.get("w2_scale")))
        st, self.h = afd_ffn_create_ex(self.cfg, w, flags)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_create_ex")
        self._events = None

    def close(self):
        if getattr(self, "h", None):
            if getattr(self, "_served_by", 0):
                raise RuntimeError("an FfnService is still running on this layer: stop it first")
            afd_ffn_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st, what):
        if st != AFD_OK:
            raise AfdError(st, what)

    def route(self, hidden, T, topk_idx, topk_w, stream=None):
        self._check(afd_ffn_route(self.h, hidden, T, topk_idx, topk_w, stream), "afd_ffn_route")

    def permute(self, hidden, topk_idx, T, counts, offsets, pos, src, stream=None):
        self._check(afd_ffn_permute(self.h, hidden, topk_idx, T, counts, offsets, pos, src, stream),
                    "afd_ffn_permute")

    def expert_gemm(self, offsets, T, Y=None, Ys=None, stream=None):
        self._check(afd_ffn_expert_gemm(self.h, offsets, T, Y, Ys, stream), "afd_ffn_expert_gemm")

    def combine(self, topk_w, pos, T, out, stream=None):
        self._check(afd_ffn_combine(self.h, topk_w, pos, T, out, stream), "afd_ffn_combine")

    def forward(self, hidden, out, T=None, stream=None):
        T = hidden.shape[0] if T is None else T
        self._check(afd_ffn_forward(self.h, hidden, T, out, stream), "afd_ffn_forward")

    def forward_host(self, hidden_host, out_host, T=None, stream=None):
        T = hidden_host.shape[0] if T is None else T
        self._check(afd_ffn_forward_host(self.h, hidden_host, T, out_host, stream), "afd_ffn_forward_host")

    def forward_host_batches(self, hidden_host_list, out_host_list, T=None, stream=None):
        T = hidden_host_list[0].shape[0] if T is None else T
        self._check(afd_ffn_forward_host_batches(self.h, hidden_host_list, out_host_list, T, stream),
                    "afd_ffn_forward_host_batches")

    def set_stage_events(self, events):
        self._events = events          # keep the events alive while the library records them
        self._check(afd_ffn_set_stage_events(self.h, events), "afd_ffn_set_stage_events")

    def get_error(self) -> int:
        return afd_ffn_get_error(self.h)


__all__ = [n for n in list(globals()) if n.startswith(("afd_ffn", "AFD_", "Afd"))] + [
    "declared_functions", "LIB_PATH", "STAGE_NAMES"]

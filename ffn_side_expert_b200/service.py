"""The FFN-service loop of an A/F split on one host: a mailbox of host buffers between the
attention side and the FFN side, and a native serving thread that runs the layer on each
micro-batch posted to it (vLLM AFD Plugin page, section 系統架構, "2. FFN Service").

Argument marshalling only: the mailbox protocol and the serving loop are C++ in
libafd_ffn.so, the layer is afd_ffn_forward.  Typical use (the attention side posts, the
service computes, the attention side reads the result)::

    mb = Mailbox(n_slots=2, T_max=256, H=7168)
    svc = FfnService(layer, mb)            # starts the serving thread
    mb.write_input(0, hidden)              # attention output of micro-batch 0, [T, H] bf16
    mb.post(0, T)
    mb.wait(0)                             # raises AfdError on failure or timeout
    y = mb.output(0)[:T]
    svc.stop()
"""
from __future__ import annotations

import ctypes

import torch

from . import (AFD_MAILBOX_PINNED, AFD_OK, AfdError, afd_ffn_mailbox_complete, afd_ffn_mailbox_create,
               afd_ffn_mailbox_destroy, afd_ffn_mailbox_input, afd_ffn_mailbox_output, afd_ffn_mailbox_post,
               afd_ffn_mailbox_take, afd_ffn_mailbox_times, afd_ffn_mailbox_wait, afd_ffn_service_slot_timeline,
               afd_ffn_service_start, afd_ffn_service_stop)


def _host_view(ptr: int, rows: int, cols: int) -> torch.Tensor:
    """A bf16 [rows, cols] tensor over host memory the mailbox owns (no copy)."""
    buf = (ctypes.c_uint8 * (rows * cols * 2)).from_address(ptr)
    return torch.frombuffer(buf, dtype=torch.bfloat16).view(rows, cols)


class Mailbox:
    """n_slots slots of input / output buffers [T_max, H] bf16 in host memory (page-locked when
    `pinned`, which needs a CUDA device).  Views from input()/output() are valid until close()."""

    def __init__(self, n_slots: int, T_max: int, H: int, pinned: bool = True):
        st, self.mb = afd_ffn_mailbox_create(n_slots, T_max, H, AFD_MAILBOX_PINNED if pinned else 0)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_mailbox_create")
        self.n_slots, self.T_max, self.H = n_slots, T_max, H
        self._served_by = 0          # running FfnService loops on this mailbox
        self._in = [_host_view(afd_ffn_mailbox_input(self.mb, i), T_max, H) for i in range(n_slots)]
        self._out = [_host_view(afd_ffn_mailbox_output(self.mb, i), T_max, H) for i in range(n_slots)]

    def input(self, slot: int) -> torch.Tensor:
        return self._in[slot]

    def output(self, slot: int) -> torch.Tensor:
        return self._out[slot]

    def write_input(self, slot: int, rows: torch.Tensor) -> None:
        """Copy a contiguous CPU bf16 tensor [T, H] into the slot's input on the calling thread
        (one memmove: no worker threads that would compete with the serving loop for cores)."""
        if not 0 <= slot < self.n_slots:
            raise IndexError(f"slot {slot} outside [0, {self.n_slots})")
        if rows.device.type != "cpu" or rows.dtype != torch.bfloat16 or not rows.is_contiguous():
            raise ValueError("rows must be a contiguous CPU bf16 tensor")
        if rows.dim() != 2 or rows.shape[1] != self.H or rows.shape[0] > self.T_max:
            raise ValueError(f"rows must be [T <= {self.T_max}, {self.H}]")
        ctypes.memmove(afd_ffn_mailbox_input(self.mb, slot), rows.data_ptr(), rows.numel() * 2)

    def post(self, slot: int, T: int) -> None:
        st = afd_ffn_mailbox_post(self.mb, slot, T)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_mailbox_post")

    def wait(self, slot: int, timeout_s: float = 60.0) -> None:
        st = afd_ffn_mailbox_wait(self.mb, slot, int(timeout_s * 1e6))
        if st != AFD_OK:
            raise AfdError(st, f"afd_ffn_mailbox_wait(slot {slot})")

    def take(self, timeout_s: float):
        """Consumer side: (status, slot, T) of the oldest posted slot."""
        return afd_ffn_mailbox_take(self.mb, int(timeout_s * 1e6))

    def complete(self, slot: int, status: int = AFD_OK) -> int:
        return afd_ffn_mailbox_complete(self.mb, slot, status)

    def times_ns(self, slot: int):
        """(post, take, done) CLOCK_MONOTONIC nanoseconds of the slot's latest round."""
        st, t = afd_ffn_mailbox_times(self.mb, slot)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_mailbox_times")
        return t

    def close(self) -> None:
        if getattr(self, "mb", None):
            if self._served_by:
                raise RuntimeError("an FfnService is still running on this mailbox: stop it first")
            self._in, self._out = [], []
            afd_ffn_mailbox_destroy(self.mb)
            self.mb = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class FfnService:
    """The serving loop of `layer` (an AfdFfn) on `mailbox`, started at construction on its own
    native thread.  While it runs, make no other call on the layer."""

    def __init__(self, layer, mailbox: Mailbox, stream=None):
        self.svc = None
        if not getattr(layer, "h", None) or not getattr(mailbox, "mb", None):
            raise ValueError("the layer and the mailbox must be open")
        st, svc = afd_ffn_service_start(layer.h, mailbox.mb, stream)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_service_start")
        self.svc, self.layer, self.mailbox = svc, layer, mailbox
        self.stats = None
        # neither may be closed while the loop runs on them
        mailbox._served_by += 1
        layer._served_by = getattr(layer, "_served_by", 0) + 1

    def timeline(self, slot: int):
        """Device timeline (ms) of the slot's latest micro-batch: service start -> H2D start, then
        from the H2D start the H2D end, layer start, layer end and D2H end.  Call it after the
        slot's wait returned and before it is posted again."""
        st, ms = afd_ffn_service_slot_timeline(self.svc, slot)
        if st != AFD_OK:
            raise AfdError(st, "afd_ffn_service_slot_timeline")
        return ms

    def stop(self):
        """Stop the loop; returns its afd_ffn_service_stats (status, served, device_status)."""
        if self.svc:
            _, self.stats = afd_ffn_service_stop(self.svc)
            self.svc = None
            self.mailbox._served_by -= 1
            self.layer._served_by -= 1
        return self.stats

    def __del__(self):
        try:
            self.stop()
        except Exception:
            pass

"""Failure detection on the device: a bounded wait that can never complete gives up, records the
timeout bit that the host reads as AFD_ERR_DEVICE_TIMEOUT, and leaves the context usable (the
next forward is correct).  The wait is the one every GEMM role uses; nothing faults or traps."""
import time

import pytest
import torch

import ffn_side_expert_b200 as afd
import synth
from layer_support import BF16_TOL, Layer, rel_max_err, to64

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    L = Layer(synth.CONFIGS["tiny"])
    try:
        t0 = time.perf_counter()
        st, cycles = afd.afd_ffn_check_bounded_wait()
        elapsed = time.perf_counter() - t0
        assert st == afd.AFD_ERR_DEVICE_TIMEOUT, afd.afd_ffn_strerror(st)
        assert cycles > 4_000_000_000          # the limit of the GEMM roles' waits
        assert elapsed < 60.0
        out = torch.empty_like(L.h)
        L.mod.forward(L.h, out)
        torch.cuda.synchronize()
        assert L.mod.get_error() == afd.AFD_OK
        assert rel_max_err(to64(out), L.oracle()["out"]) <= BF16_TOL
    finally:
        L.close()

"""The C-ABI library loads, exports every declared entry point, and fails fast on bad
arguments before touching a device (CPU only: no compute call is made here)."""
import ctypes

import pytest

import ffn_side_expert_b200 as afd


def test_every_declared_symbol_is_exported():
    names = afd.declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(afd.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding wraps each one under the same name
    assert all(callable(getattr(afd, n)) for n in names)


def test_strerror_covers_every_status():
    for st in range(0, -8, -1):
        s = afd.afd_ffn_strerror(st)
        assert s and s != "unknown status"
    assert afd.afd_ffn_strerror(12345) == "unknown status"


def _cfg(**kw):
    base = dict(T_max=64, H=256, E=8, k=2, I=512, n_shared=0, weight_dtype=afd.AFD_DT_BF16,
                act_dtype=afd.AFD_DT_BF16, has_router_bias=0)
    base.update(kw)
    return afd.afd_ffn_cfg(**base)


_W = afd.afd_ffn_weights(256, None, 512, 768, None, None)   # fake aligned addresses, never used


@pytest.mark.parametrize("kw,status", [
    (dict(T_max=0), afd.AFD_ERR_INVALID_ARG),
    (dict(k=0), afd.AFD_ERR_INVALID_ARG),
    (dict(k=9), afd.AFD_ERR_INVALID_ARG),            # k > E
    (dict(n_shared=2), afd.AFD_ERR_INVALID_ARG),
    (dict(weight_dtype=7, act_dtype=7), afd.AFD_ERR_INVALID_ARG),
    (dict(act_dtype=afd.AFD_DT_FP8_E4M3), afd.AFD_ERR_UNSUPPORTED),
    (dict(E=300, k=2), afd.AFD_ERR_UNSUPPORTED),
    (dict(E=64, k=33), afd.AFD_ERR_UNSUPPORTED),
    (dict(H=384), afd.AFD_ERR_UNSUPPORTED),           # H must be a multiple of 256
    (dict(I=200), afd.AFD_ERR_UNSUPPORTED),           # I must be a multiple of 128
])
def test_create_rejects_bad_config_on_host(kw, status):
    st, h = afd.afd_ffn_create(_cfg(**kw), _W)
    assert st == status and h is None


def test_create_rejects_bad_weights_on_host():
    st, _ = afd.afd_ffn_create(_cfg(), afd.afd_ffn_weights(None, None, 512, 768, None, None))
    assert st == afd.AFD_ERR_INVALID_ARG
    st, _ = afd.afd_ffn_create(_cfg(), afd.afd_ffn_weights(257, None, 512, 768, None, None))
    assert st == afd.AFD_ERR_INVALID_ARG                      # misaligned router pointer
    st, _ = afd.afd_ffn_create(_cfg(has_router_bias=1), _W)
    assert st == afd.AFD_ERR_INVALID_ARG                      # bias promised, not given
    fp8 = _cfg(weight_dtype=afd.AFD_DT_FP8_E4M3, act_dtype=afd.AFD_DT_FP8_E4M3)
    st, _ = afd.afd_ffn_create(fp8, _W)
    assert st == afd.AFD_ERR_INVALID_ARG                      # e4m3 without scales
    st, _ = afd.afd_ffn_create(None, _W)
    assert st == afd.AFD_ERR_INVALID_ARG


def test_null_handle_calls_fail_fast():
    assert afd.afd_ffn_forward(None, 0, 4, 0, 0) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_get_error(None) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_set_stage_events(None, None) == afd.AFD_ERR_INVALID_ARG
    afd.afd_ffn_destroy(None)

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
    for st in range(0, -10, -1):
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
    st, _ = afd.afd_ffn_create_ex(_cfg(), _W, 2)            # unknown option bit, refused on the host
    assert st == afd.AFD_ERR_INVALID_ARG
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


def test_expert_parallel_calls_fail_fast_on_bad_arguments():
    # host-side checks only: none of these reaches the device
    A = 4096  # a 16-byte aligned stand-in address
    assert afd.afd_ffn_dispatch_rows(A, A, 4, 0, 8, 256, A, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG   # k = 0
    assert afd.afd_ffn_dispatch_rows(A, A, 4, 9, 8, 256, A, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG   # k > E
    assert afd.afd_ffn_dispatch_rows(A, A, 4, 2, 8, 12, A, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG    # H % 8
    assert afd.afd_ffn_dispatch_rows(A, A, 4, 2, 8, 256, A, A, A, A, A + 2, A) == afd.AFD_ERR_INVALID_ARG  # rows
    assert afd.afd_ffn_dispatch_rows(A, A, 4, 2, 8, 256, None, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_expert_rows(None, A, A, 4, A) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_copy_row_blocks(A, A, A, 1, 6) == afd.AFD_ERR_INVALID_ARG                        # 6-byte rows
    assert afd.afd_ffn_copy_row_blocks(A + 2, A, A, 1, 4) == afd.AFD_ERR_INVALID_ARG                    # 4-byte rows
    assert afd.afd_ffn_copy_row_blocks(A + 4, A, A, 1, 32) == afd.AFD_ERR_INVALID_ARG                   # 16-byte moves
    assert afd.afd_ffn_copy_row_blocks(A, A, A, -1, 16) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_copy_row_blocks(A, A, A, 0, 16) == afd.AFD_OK                                    # nothing to do
    assert afd.afd_ffn_combine_rows(A, None, A, A, 4, 33, 256, A) == afd.AFD_ERR_INVALID_ARG            # k > 32
    assert afd.afd_ffn_combine_rows(A, None, A, A, 4, 2, 6, A) == afd.AFD_ERR_INVALID_ARG               # H % 4
    assert afd.afd_ffn_combine_rows(A, A + 4, A, A, 4, 2, 256, A) == afd.AFD_ERR_INVALID_ARG            # Ys align
    assert afd.afd_ffn_combine_rows(A, None, A, A, 0, 2, 256, A) == afd.AFD_OK                          # T = 0
    # the W8A8 exchange
    fp8d = afd.afd_ffn_dispatch_rows_fp8
    assert fp8d(A, A, 4, 2, 8, 264, 1, A, A, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG       # H % 16
    assert fp8d(A, A, 4, 2, 8, 256, 2, A, A, A, A, A, A, A) == afd.AFD_ERR_INVALID_ARG       # with_shared
    assert fp8d(A, A, 4, 2, 8, 256, 1, A, A, A, A, A, None, A) == afd.AFD_ERR_INVALID_ARG    # no scales
    assert fp8d(A, A, 4, 2, 8, 256, 1, A, A, A, A, A + 8, A, A) == afd.AFD_ERR_INVALID_ARG   # rows align
    assert afd.afd_ffn_expert_rows_fp8(None, A, A, A, 4, A) == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_combine_rows_bf16(A, None, A, A, 4, 0, 256, A) == afd.AFD_ERR_INVALID_ARG      # k = 0
    assert afd.afd_ffn_combine_rows_bf16(A, A + 2, A, A, 4, 2, 256, A) == afd.AFD_ERR_INVALID_ARG     # Ys align
    assert afd.afd_ffn_combine_rows_bf16(A, None, A, A, 0, 2, 256, A) == afd.AFD_OK                   # T = 0


def test_service_calls_fail_fast_without_a_handle():
    assert afd.afd_ffn_service_start(None, None)[0] == afd.AFD_ERR_INVALID_ARG
    st, mb = afd.afd_ffn_mailbox_create(1, 4, 64, 0)
    assert st == afd.AFD_OK
    try:
        assert afd.afd_ffn_service_start(None, mb)[0] == afd.AFD_ERR_INVALID_ARG
    finally:
        afd.afd_ffn_mailbox_destroy(mb)
    assert afd.afd_ffn_service_stop(None)[0] == afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_get_info(None)[0] == afd.AFD_ERR_INVALID_ARG


def test_bounded_wait_check_needs_a_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present: the GPU test covers the call")
    assert afd.afd_ffn_check_bounded_wait()[0] == afd.AFD_ERR_NO_DEVICE


def _declared_params(header=afd.HEADER_PATH):
    """name -> list of parameter kinds ('ptr', 'i32', 'u32', 'i64', 'f32') from include/afd_ffn.h."""
    import re
    with open(header) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(afd_ffn_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = " ".join(m.group(2).split())
        kinds = []
        for p in ([] if params in ("", "void") else params.split(",")):
            if "*" in p:
                kinds.append("ptr")
            elif "int64_t" in p:
                kinds.append("i64")
            elif "float" in p:
                kinds.append("f32")
            elif "uint32_t" in p:
                kinds.append("u32")
            else:
                assert re.search(r"\b(int32_t|int)\b", p), p
                kinds.append("i32")
        out[m.group(1)] = kinds
    return out


def _kind(ct):
    if ct in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(ct, type(ctypes.POINTER(ctypes.c_int))):
        return "ptr"
    return {ctypes.c_int32: "i32", ctypes.c_int: "i32", ctypes.c_uint32: "u32", ctypes.c_int64: "i64",
            ctypes.c_float: "f32"}[ct]


def _declared_arities(header=afd.HEADER_PATH):
    return {k: len(v) for k, v in _declared_params(header).items()}


def test_binding_signatures_match_the_header():
    """Every declared entry point is bound with as many ctypes arguments as the header gives
    it, and with a result type (None only for the void ones)."""
    arity = _declared_arities()
    assert set(arity) == set(afd.declared_functions())
    for name, n in arity.items():
        res, args = afd._SIGNATURES[name]
        assert len(args) == n, (name, len(args), n)
    for name in ("afd_ffn_destroy", "afd_ffn_mailbox_destroy"):
        assert afd._SIGNATURES[name][0] is None


def test_binding_argument_kinds_match_the_header():
    for name, kinds in _declared_params().items():
        _, args = afd._SIGNATURES[name]
        assert [_kind(a) for a in args] == kinds, name

"""The C-ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

import weight_only_int4_fp32_b200 as lm

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(HERE), "include", "ling_moe.h")


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ling_moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_list():
    assert declared_symbols() == sorted(lm.EXPORTED)


def test_every_declared_symbol_is_exported():
    L = ctypes.CDLL(lm.library_path())
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_binding_structs_match_header_layout():
    assert ctypes.sizeof(lm.ling_moe_config_t) == 6 * 4
    assert ctypes.sizeof(lm.ling_moe_weights_t) == 11 * ctypes.sizeof(ctypes.c_void_p)
    assert [f for f, _ in lm.ling_moe_weights_t._fields_] == [
        "router_w", "router_bias", "gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s",
        "sh_gate", "sh_up", "sh_down"]


def _cfg(**kw):
    d = dict(hidden=2560, inter=768, num_experts=512, top_k=8, group_size=32, max_tokens=4)
    d.update(kw)
    return lm.ling_moe_config_t(**d)


def _weights(ptr=0x100000):
    return lm.ling_moe_weights_t(*([ptr] * 11))


def _create_rc(cfg, w):
    h = ctypes.c_void_p()
    rc = lm.lib.ling_moe_create(ctypes.byref(cfg) if cfg is not None else None,
                                ctypes.byref(w) if w is not None else None, ctypes.byref(h))
    return rc, h.value


def test_create_rejects_null_arguments():
    rc, h = _create_rc(None, _weights())
    assert rc == lm.LING_MOE_ERR_INVALID_ARG and h is None
    rc, h = _create_rc(_cfg(), None)
    assert rc == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_create(ctypes.byref(_cfg()), ctypes.byref(_weights()), None) == \
        lm.LING_MOE_ERR_INVALID_ARG
    w = _weights()
    w.gate_q = None
    rc, _ = _create_rc(_cfg(), w)
    assert rc == lm.LING_MOE_ERR_INVALID_ARG
    assert "NULL" in lm.ling_moe_last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(top_k=9, num_experts=16), lm.LING_MOE_ERR_UNSUPPORTED),
    (dict(top_k=9, num_experts=8), lm.LING_MOE_ERR_INVALID_ARG),
    (dict(num_experts=513), lm.LING_MOE_ERR_UNSUPPORTED),
    (dict(hidden=2048), lm.LING_MOE_ERR_UNSUPPORTED),
    (dict(inter=1024), lm.LING_MOE_ERR_UNSUPPORTED),
    (dict(group_size=64), lm.LING_MOE_ERR_UNSUPPORTED),
    (dict(hidden=2561), lm.LING_MOE_ERR_INVALID_ARG),
    (dict(max_tokens=0), lm.LING_MOE_ERR_INVALID_ARG),
    (dict(top_k=0), lm.LING_MOE_ERR_INVALID_ARG),
    (dict(num_experts=-1), lm.LING_MOE_ERR_INVALID_ARG),
])
def test_create_rejects_unsupported_shapes(kw, code):
    rc, h = _create_rc(_cfg(**kw), _weights())
    assert rc == code, lm.ling_moe_last_error()
    assert h is None


def test_create_rejects_misaligned_weights():
    w = _weights()
    w.down_s = 0x100008
    rc, _ = _create_rc(_cfg(), w)
    assert rc == lm.LING_MOE_ERR_INVALID_ARG
    assert "aligned" in lm.ling_moe_last_error()


def test_null_handle_is_rejected_everywhere():
    assert lm.lib.ling_moe_forward(None, 16, 1, 32, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_forward_ex(None, 16, 1, 32, None, None, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_forward_host(None, 16, 1, 32, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_status(None, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_test_set_wait(None, 0, 0) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_set_kernel_timing(None, 1) == lm.LING_MOE_ERR_INVALID_ARG
    n = ctypes.c_int(-7)
    assert lm.lib.ling_moe_kernel_times(None, None, 0, ctypes.byref(n)) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_kernel_name(None, 0) == b""
    assert lm.ling_moe_describe(None) == ""
    assert lm.ling_moe_launch_count(None) == 0
    lm.ling_moe_destroy(None)  # no-op


def test_python_errors_carry_the_code():
    with pytest.raises(lm.LingMoEError) as ei:
        lm.ling_moe_create(_cfg(top_k=9, num_experts=16), _weights())
    assert ei.value.code == lm.LING_MOE_ERR_UNSUPPORTED


def _lmh_create_rc(w, vocab, hidden):
    h = ctypes.c_void_p()
    rc = lm.lib.ling_moe_lmhead_create(w, vocab, hidden, ctypes.byref(h))
    return rc, h.value


@pytest.mark.parametrize("w,vocab,hidden,code", [
    (None, 1000, 2560, lm.LING_MOE_ERR_INVALID_ARG),
    (0x100008, 1000, 2560, lm.LING_MOE_ERR_INVALID_ARG),      # misaligned
    (0x100000, 0, 2560, lm.LING_MOE_ERR_INVALID_ARG),
    (0x100000, 1000, -512, lm.LING_MOE_ERR_INVALID_ARG),
    (0x100000, 1000, 2304, lm.LING_MOE_ERR_UNSUPPORTED),      # not a multiple of 512
    (0x100000, 1000, 4608, lm.LING_MOE_ERR_UNSUPPORTED),      # above 4096
])
def test_lmhead_create_rejects_bad_arguments(w, vocab, hidden, code):
    rc, h = _lmh_create_rc(w, vocab, hidden)
    assert rc == code, lm.ling_moe_last_error()
    assert h is None
    assert lm.lib.ling_moe_lmhead_create(0x100000, 1000, 2560, None) == lm.LING_MOE_ERR_INVALID_ARG


def test_lmhead_null_handle_is_rejected_everywhere():
    assert lm.lib.ling_moe_lmhead_forward(None, 16, 1, 32, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_forward_ex(None, 16, 1, 32, None, None, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_forward_host(None, 16, 1, 32, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_weights(None, 16, 32, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_status(None, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_test_set_wait(None, 0, 0) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_lmhead_launch_count(None) == 0
    lm.lib.ling_moe_lmhead_destroy(None)  # no-op


def test_create_mxfp4_checks_arguments():
    h = ctypes.c_void_p()
    assert lm.lib.ling_moe_create_mxfp4(None, ctypes.byref(_weights()), ctypes.byref(h)) == \
        lm.LING_MOE_ERR_INVALID_ARG
    rc = lm.lib.ling_moe_create_mxfp4(ctypes.byref(_cfg(group_size=64)), ctypes.byref(_weights()), ctypes.byref(h))
    assert rc == lm.LING_MOE_ERR_UNSUPPORTED and h.value is None
    rc = lm.lib.ling_moe_create_mxfp4(ctypes.byref(_cfg(top_k=9, num_experts=16)), ctypes.byref(_weights()),
                                      ctypes.byref(h))
    assert rc == lm.LING_MOE_ERR_UNSUPPORTED and h.value is None


def test_binding_rejects_wrong_tensors_before_any_call():
    import torch
    layer = object.__new__(lm.MoELayer)   # no handle: the checks run before the library is called
    layer.H, layer.k, layer._torch, layer.handle = 2560, 8, torch, None
    with pytest.raises(ValueError):
        layer.forward(torch.zeros((1, 2560), dtype=torch.bfloat16))          # not on the GPU
    with pytest.raises(ValueError):
        layer.forward_host(torch.zeros((2, 2048), dtype=torch.bfloat16))     # wrong hidden
    with pytest.raises(ValueError):
        layer.forward_host(torch.zeros((2, 2560), dtype=torch.bfloat16), torch.zeros((2, 2560)))  # fp32 out
    head = object.__new__(lm.LMHeadFP8)
    head.vocab, head.hidden, head._torch, head.handle = 1000, 2560, torch, None
    with pytest.raises(ValueError):
        head.forward_host(torch.zeros((1, 2560), dtype=torch.bfloat16), torch.zeros((1, 999)))
    with pytest.raises(ValueError):
        head.forward(torch.zeros((1, 2560), dtype=torch.bfloat16))


def _ep_rc(cfg, w, ep):
    h = ctypes.c_void_p()
    rc = lm.lib.ling_moe_create_ep(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(ep) if ep is not None else None,
                                   ctypes.byref(h))
    return rc, h.value


@pytest.mark.parametrize("begin,count,shared,fmt", [
    (-1, 4, 1, 0),      # range starts before 0
    (0, 0, 1, 0),       # no expert
    (510, 4, 1, 0),     # past the router's experts
    (0, 4, 2, 0),       # with_shared not 0/1
    (0, 4, 1, 7),       # unknown format
])
def test_create_ep_rejects_bad_ranges_before_the_gpu(begin, count, shared, fmt):
    rc, h = _ep_rc(_cfg(), _weights(), lm.ling_moe_ep_t(begin, count, shared, fmt))
    assert rc == lm.LING_MOE_ERR_INVALID_ARG and h is None
    rc, h = _ep_rc(_cfg(), _weights(), None)
    assert rc == lm.LING_MOE_ERR_INVALID_ARG and h is None


def test_create_ep_needs_shared_weights_only_where_it_computes_them():
    w = _weights()
    w.sh_gate = w.sh_up = w.sh_down = None
    rc, _ = _ep_rc(_cfg(), w, lm.ling_moe_ep_t(0, 4, 1, 0))
    assert rc == lm.LING_MOE_ERR_INVALID_ARG  # the shared expert is computed here: its weights are required
    assert "NULL" in lm.ling_moe_last_error()
    import torch
    if not torch.cuda.is_available():  # with a GPU the fake pointers would reach the copies
        rc, _ = _ep_rc(_cfg(), w, lm.ling_moe_ep_t(0, 4, 0, 0))
        assert rc == lm.LING_MOE_ERR_CUDA  # accepted on the host, then no device to copy to


def test_partial_and_round_reject_bad_arguments():
    assert lm.lib.ling_moe_forward_partial(None, None, 1, None, None, None, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_round_bf16(None, None, 8, None) == lm.LING_MOE_ERR_INVALID_ARG
    assert lm.lib.ling_moe_round_bf16(0x100000, 0x200000, 7, None) == lm.LING_MOE_ERR_INVALID_ARG  # n % 8
    assert lm.lib.ling_moe_round_bf16(0x100004, 0x200000, 8, None) == lm.LING_MOE_ERR_INVALID_ARG  # alignment
    assert lm.lib.ling_moe_round_bf16(0x100000, 0x100010, 64, None) == lm.LING_MOE_ERR_INVALID_ARG  # overlap
    assert lm.lib.ling_moe_round_bf16(0x100000, 0x200000, 0, None) == lm.LING_MOE_OK  # nothing to do

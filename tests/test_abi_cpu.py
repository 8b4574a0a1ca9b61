"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad configurations on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

import compressed_decode_attention_fdms_b200 as fd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fdms.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fdms_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from compressed_decode_attention_fdms_b200 import build
    build.build()
    return fd.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "fdms_decode_attn" in names and "fdms_append_evict" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(fd.EXPORTED)


def test_status_strings(lib):
    for s in range(6):
        assert fd.status_string(s)
    assert fd.status_string(99) == "unknown status"


def _create(cfg):
    h = ctypes.c_void_p()
    return fd.load_library().fdms_cache_create(ctypes.byref(cfg), 0, None, ctypes.byref(h))


def test_invalid_configs_are_rejected_before_any_device_call(lib):
    good = dict(num_layers=1, max_batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64, window=16)
    bad = [dict(num_layers=0), dict(num_q_heads=5), dict(window=-1), dict(compact_period=0),
           dict(max_seq_len=0), dict(num_blocks=-1), dict(kv_dtype=7), dict(softmax_scale=-1.0)]
    for b in bad:
        kw = {**good, **b}
        assert _create(fd.make_config(**kw)) == fd.FDMS_ERR_INVALID_ARG, b
    for u in [dict(head_dim=96), dict(num_q_heads=6, num_kv_heads=2),
              dict(max_batch=4096, num_kv_heads=2)]:
        assert _create(fd.make_config(**{**good, **u})) == fd.FDMS_ERR_UNSUPPORTED, u


def test_null_arguments(lib):
    P = ctypes.c_void_p
    assert lib.fdms_cache_create(None, 0, None, ctypes.byref(P())) == fd.FDMS_ERR_INVALID_ARG
    assert lib.fdms_cache_destroy(None) == fd.FDMS_OK
    assert lib.fdms_append_evict(None, 0, 1, None, 1, None, None, None, None, None) == \
        fd.FDMS_ERR_INVALID_ARG
    assert lib.fdms_decode_attn(None, 0, 1, None, None, None) == fd.FDMS_ERR_INVALID_ARG
    assert lib.fdms_cache_stats(None, None, None) == fd.FDMS_ERR_INVALID_ARG


def test_binding_rejects_what_the_c_abi_cannot_take():
    """The binding's tensor check: a non-tensor, a host tensor (before any
    device call), and, through the same check, dtype / shape / layout."""
    import torch
    t = torch.zeros((2, 3), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        fd._dev_tensor([0.0] * 6, torch.bfloat16, (2, 3), "x", 0)
    with pytest.raises(ValueError, match="cuda:0"):
        fd._dev_tensor(t, torch.bfloat16, (2, 3), "x", 0)
    with pytest.raises(ValueError):
        fd._dev_tensor(t.t(), torch.bfloat16, (3, 2), "x", 0)
    with pytest.raises((TypeError, ValueError)):
        fd._dev_tensor(t.float(), torch.bfloat16, (2, 3), "x", 0)

"""The decode entry point that allocates nothing, against the regular one.

fdms_decode_attn_noalloc is for callers that cannot call cudaMalloc on their
decode path (their device memory is handed out by another owner, or they must
not allocate once running). It keeps the split partials in a fixed array
compiled into the library instead of the cache's workspace. This checks,
through the C ABI, that two calls in a row give what fdms_decode_attn gives,
and that a call needing more scratch than the array holds is refused.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wk

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import compressed_decode_attention_fdms_b200 as fd  # noqa: E402

TOL = 3e-3   # the BF16 bound of the parity tests (plus half a bf16 ulp of the value)


def _close(a, b):
    a = a.float().cpu().numpy()
    b = b.float().cpu().numpy()
    half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    return float(np.max(np.abs(a - b) - half_ulp)) <= TOL


@pytest.mark.parametrize("name", ["tiny", "llama_shape"])
def test_noalloc_matches_regular_decode_two_calls(name):
    wl = wk.get("tiny") if name == "tiny" else \
        wk.scaled(wk.get("llama1b_c8"), layers=2, batch=3, ctx=900, steps=2)
    dev = "cuda:0"
    cfg = fd.make_config(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                         wl.period, wl.max_seq_len, 0, wl.kv_dtype)
    cache = fd.fdms_cache_create(cfg, 0)
    lib = fd.load_library()
    try:
        for layer in range(wl.layers):
            inp = wk.prefill_inputs(wl, layer)
            fd.fdms_append_evict(cache, layer, wl.batch, inp["n_new"].to(dev), inp["max_new"],
                                 inp["k"].to(dev), inp["v"].to(dev), inp["keep"].to(dev))
        for step in range(2):
            for layer in range(wl.layers):
                inp = wk.decode_inputs(wl, layer, step)
                fd.fdms_append_evict(cache, layer, wl.batch, inp["n_new"].to(dev), 1,
                                     inp["k"].to(dev), inp["v"].to(dev), inp["keep"].to(dev))
                q = wk.decode_query(wl, layer, step).to(dev)
                ref = torch.empty_like(q)
                fd.fdms_decode_attn(cache, layer, wl.batch, q, ref)
                outs = []
                for _ in range(2):          # two calls in a row on the shared array
                    out = torch.full_like(q, float("nan"))
                    st = lib.fdms_decode_attn_noalloc(
                        ctypes.c_void_p(cache.handle), layer, wl.batch,
                        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
                    assert st == fd.FDMS_OK, fd.status_string(st)
                    outs.append(out)
                torch.cuda.synchronize()
                for out in outs:
                    assert _close(out, ref), (name, step, layer)
        assert fd.fdms_cache_stats(cache)["error"] == 0
    finally:
        fd.fdms_cache_destroy(cache)


def test_noalloc_refuses_more_scratch_than_the_array():
    # 1024 (seq, kv head) pairs with G = 8, D = 128 need about 7 MB of partials
    cfg = fd.make_config(1, 128, 64, 8, 128, 16, 1, 64, 0, "bf16")
    cache = fd.fdms_cache_create(cfg, 0)
    try:
        q = torch.zeros((128, 64, 128), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(q)
        st = fd.load_library().fdms_decode_attn_noalloc(
            ctypes.c_void_p(cache.handle), 0, 128, ctypes.c_void_p(q.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), None)
        assert st == fd.FDMS_ERR_INVALID_ARG
    finally:
        fd.fdms_cache_destroy(cache)

"""The decode entry point that allocates nothing, against the regular one.

fdms_decode_attn_noalloc is for callers that cannot call cudaMalloc on their
decode path (their device memory is handed out by another owner, or they must
not allocate once running). It keeps the split partials in a fixed array
compiled into the library instead of the cache's workspace. Through the C ABI,
two calls in a row must give exactly what fdms_decode_attn gives (same kernels,
same inputs; only the scratch address differs) and stay within the BF16 bar of
the fp64 oracle, in both decode modes: per-head clusters (partials in shared
memory) and the global plan, whose split and combine kernels write and read
the partials in the static array. A call needing more scratch than the array
holds is refused.
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
from _pair import Pair  # noqa: E402

TOL = 3e-3   # the BF16 bar of the parity tests, beyond half a bf16 ulp of the value


def _oracle_err(out, ref: dict):
    g = out.float().cpu().numpy()
    worst = 0.0
    for b, r in ref.items():
        half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -126))) - 7)
        worst = max(worst, float(np.max(np.abs(g[b] - r) - half_ulp)))
    return worst


def _noalloc(cache, layer, batch, q, out):
    return fd.load_library().fdms_decode_attn_noalloc(
        ctypes.c_void_p(cache.handle), layer, batch, ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# "auto": few heads, one cluster of CTAs per head (no scratch); "plan": an
# explicit split grid, the global tile plan whose partials live in the array.
MODES = {"auto": 0, "plan": 148}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("name", ["tiny", "llama_shape"])
def test_noalloc_matches_regular_decode_two_calls(name, mode):
    wl = wk.get("tiny") if name == "tiny" else \
        wk.scaled(wk.get("llama1b_c8"), layers=2, batch=3, ctx=900, steps=2)
    dev = "cuda:0"
    p = Pair(wl, decode_ctas=MODES[mode])
    try:
        for layer in range(wl.layers):
            p.append(layer, wk.prefill_inputs(wl, layer))
        for step in range(2):
            for layer in range(wl.layers):
                p.append(layer, wk.decode_inputs(wl, layer, step))
                q = wk.decode_query(wl, layer, step)
                qd = q.to(dev)
                ref = torch.empty_like(qd)
                for _ in range(2):   # the second regular call is the reference
                    fd.fdms_decode_attn(p.cache, layer, wl.batch, qd, ref)
                outs = []
                for _ in range(2):          # two calls in a row on the shared array
                    out = torch.full_like(qd, float("nan"))
                    st = _noalloc(p.cache, layer, wl.batch, qd, out)
                    assert st == fd.FDMS_OK, fd.status_string(st)
                    outs.append(out)
                torch.cuda.synchronize()
                exact = p.oracle_out(layer, q)
                for out in outs:
                    assert torch.equal(out, ref), (name, mode, step, layer)
                    assert _oracle_err(out, exact) <= TOL, (name, mode, step, layer)
        assert fd.fdms_cache_stats(p.cache)["error"] == 0
    finally:
        p.close()


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

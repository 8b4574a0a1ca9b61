"""Parity at the benchmark workloads' full sizes, in the launch configuration
bench.py times (needs a B200).

The GPU cache holds every sequence of the workload at full context length and
runs the default decode launch (llama1b_c8 and qwen8b_c8_fp8: one cluster of
CTAs per (seq, kv head); qwen8b_long_fp8, 256 heads: the global tile plan with
its combine kernel); the fp64 oracle follows a
few sampled sequences one by one (a one-sequence oracle each, fed that
sequence's inputs, which do not depend on the other sequences). One layer: the
kernels' launch configuration and per-call sizes do not depend on the number
of layers. Checked after the prefill and after each decode step: the sampled
sequences' heads (store and ring) bit-exact, and their decode outputs within
the bars of test_gpu_parity; FP8 outputs also within the stated 3e-2 of the
oracle fed the unquantised bf16 values (the method's own E4M3 error, which
averages out over the thousands of tokens these heads see).
"""
import numpy as np
import pytest
import torch

import compressed_decode_attention_fdms_b200 as fd
import workloads as wk
from oracle.cache import OracleCache

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from _pair import bits  # noqa: E402

TOL_BF16 = 3e-3
TOL_FP8_MIRROR = 3e-3
TOL_FP8_TRUE = 3e-2   # the stated FP8 bar, against the unquantised bf16 inputs
STEPS = 3


def _half_ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-300)))
    return np.where(x == 0, 0.0, 2.0 ** (e - 8))


def _check_head(cache, oc, b, h, layer_gpu, seq_gpu, kv_dtype):
    got = fd.fdms_cache_read_head(cache, layer_gpu, seq_gpu, h)
    pos, kp, vp = oc.store(0, 0, h)
    rpos, rk, rv, rkeep = oc.ring(0, 0, h)
    ctx = f"seq {seq_gpu} head {h}"
    assert got["num_tokens"] == int(oc.n[0, 0]), ctx
    assert got["resolved"] == int(oc.r[0, 0]), ctx
    assert got["store_len"] == len(pos), ctx
    n_s = len(pos)
    assert np.array_equal(got["pos"][:n_s], pos), ctx
    assert np.array_equal(got["pos"][n_s:], rpos), ctx
    assert np.array_equal(got["keep"][n_s:], rkeep), ctx
    exp_k = np.concatenate([kp, rk]) if len(rk) else kp
    exp_v = np.concatenate([vp, rv]) if len(rv) else vp
    if kv_dtype == "bf16":
        gk, gv = got["k"].view(np.uint16), got["v"].view(np.uint16)
    else:
        gk, gv = got["k"], got["v"]
    assert np.array_equal(gk, exp_k.reshape(gk.shape)), ctx + " K payload"
    assert np.array_equal(gv, exp_v.reshape(gv.shape)), ctx + " V payload"


@pytest.mark.parametrize("name", ["llama1b_c8", "qwen8b_c8_fp8", "qwen8b_long_fp8"])
def test_full_size_sampled_sequences(name):
    wl = wk.scaled(wk.get(name), layers=1, steps=STEPS)
    ctx = wk.context_lengths(wl)
    sample = sorted({0, int(np.argmax(ctx))})          # the first and the longest
    dev = torch.device("cuda", 0)
    cfg = fd.make_config(1, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                         wl.period, wl.max_seq_len, 0, wl.kv_dtype)
    cache = fd.fdms_cache_create(cfg, 0)
    ocs = {b: OracleCache(1, 1, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window, wl.period,
                          wl.kv_dtype, capacity=wl.max_seq_len) for b in sample}
    tol = TOL_BF16 if wl.kv_dtype == "bf16" else TOL_FP8_MIRROR
    try:
        # prefill: every sequence on the GPU, the sampled ones in their oracles
        inp = wk.prefill_inputs(wl, 0, device=dev)
        fd.fdms_append_evict(cache, 0, wl.batch, inp["n_new"], inp["max_new"], inp["k"],
                             inp["v"], inp["keep"])
        for b in sample:
            n = int(ctx[b])
            ocs[b].append(0, np.array([n]), bits(inp["k"][b:b + 1, :n]),
                          bits(inp["v"][b:b + 1, :n]), inp["keep"][b:b + 1, :n].cpu().numpy())
        del inp
        torch.cuda.synchronize()
        for b in sample:
            for h in range(wl.kv_heads):
                _check_head(cache, ocs[b], b, h, 0, b, wl.kv_dtype)
        out = torch.empty((wl.batch, wl.q_heads, wl.head_dim), dtype=torch.bfloat16,
                          device=dev)
        for step in range(STEPS):
            st = wk.decode_inputs(wl, 0, step, device=dev)
            fd.fdms_append_evict(cache, 0, wl.batch, st["n_new"], 1, st["k"], st["v"],
                                 st["keep"])
            q = wk.decode_query(wl, 0, step, device=dev)
            fd.fdms_decode_attn(cache, 0, wl.batch, q, out)
            torch.cuda.synchronize()
            g = out.float().cpu().numpy().astype(np.float64)
            for b in sample:
                ocs[b].append(0, st["n_new"][b:b + 1].cpu().numpy(), bits(st["k"][b:b + 1]),
                              bits(st["v"][b:b + 1]), st["keep"][b:b + 1].cpu().numpy())
                ref = ocs[b].attention(0, 0, bits(q[b]))
                err = float(np.max(np.abs(g[b] - ref) - _half_ulp_bf16(ref)))
                assert err <= tol, (name, step, b, err)
                if wl.kv_dtype == "fp8_e4m3":
                    ref_t = ocs[b].attention(0, 0, bits(q[b]), mode="true")
                    err_t = float(np.max(np.abs(g[b] - ref_t) - _half_ulp_bf16(ref_t)))
                    assert err_t <= TOL_FP8_TRUE, (name, step, b, err_t)
                for h in range(wl.kv_heads):
                    _check_head(cache, ocs[b], b, h, 0, b, wl.kv_dtype)
        assert fd.fdms_cache_stats(cache)["error"] == 0
    finally:
        fd.fdms_cache_destroy(cache)

"""Failure detection of the decode kernels' bounded waits (needs a B200).

Every wait of a decode kernel on its tile copies gives up after 2 s, latches
FDMS_ERR_DEVICE and lets the kernel finish (its copies landed, every barrier of
the CTA and the cluster is still reached), so that the host reads an error and
the context stays usable. FDMS_TEST_STALL_COPIES, set when a cache is created,
makes every tile stage of that cache expect 16 bytes more than its copies bring:
the copies land, no stage completes, and every wait runs out. No fault, trap or
endless wait is involved.
"""
import os
import time

import numpy as np
import pytest
import torch

import compressed_decode_attention_fdms_b200 as fd
import workloads as wk
from _pair import Pair

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _half_ulp_bf16(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - 7)


def _stalled_pair(wl, decode_ctas):
    os.environ["FDMS_TEST_STALL_COPIES"] = "1"
    try:
        return Pair(wl, decode_ctas=decode_ctas, max_seq_len=wl.ctx + 16)
    finally:
        del os.environ["FDMS_TEST_STALL_COPIES"]


# (kv dtype, head dim, decode_ctas): per-head clusters, the global plan, and
# the per-block FP8 variant of the cluster kernel
@pytest.mark.parametrize("kv_dtype,head_dim,decode_ctas",
                         [("bf16", 64, 0), ("bf16", 64, 148), ("fp8_e4m3_block", 128, 0)])
def test_stage_waits_run_out_latch_and_leave_the_context_usable(kv_dtype, head_dim, decode_ctas):
    wl = wk.scaled(wk.get("llama1b_c8"), layers=1, batch=2, ctx=200, steps=0, kv_dtype=kv_dtype,
                   head_dim=head_dim)
    q = wk.decode_query(wl, 0, 0)
    p = _stalled_pair(wl, decode_ctas)
    try:
        lay = fd.fdms_decode_layout(p.cache, wl.batch)
        assert (lay["cluster_ctas"] == 0) == (decode_ctas > 0)
        p.append(0, wk.prefill_inputs(wl, 0))
        assert fd.fdms_cache_stats(p.cache)["error"] == 0   # appends do not stall
        t0 = time.monotonic()
        p.decode(0, q)
        torch.cuda.synchronize()
        took = time.monotonic() - t0
        st = fd.fdms_cache_stats(p.cache)
        assert st["error"] == fd.FDMS_ERR_DEVICE
        assert 2.0 <= took < 30.0, took   # each wait gave up after its limit
    finally:
        p.close()
    # the same context decodes correctly afterwards
    p2 = Pair(wl, decode_ctas=decode_ctas, max_seq_len=wl.ctx + 16)
    try:
        p2.append(0, wk.prefill_inputs(wl, 0))
        out = p2.decode(0, q)
        torch.cuda.synchronize()
        assert fd.fdms_cache_stats(p2.cache)["error"] == 0
        ref = p2.oracle_out(0, q)
        g = out.float().cpu().numpy()
        for b in ref:
            err = float(np.max(np.abs(g[b] - ref[b]) - _half_ulp_bf16(ref[b])))
            assert err <= 3e-3, (b, err)
    finally:
        p2.close()

"""Decode layout and the decode counters (needs a B200).

fdms_decode_layout reports the mode a call runs (per-head clusters or the
global plan); every decode call adds the slots and the K/V bytes it scans to
fdms_stats, which must equal the oracle's store + ring sizes of the call's heads
(per-block FP8: sealed slots in E4M3, staged and ring slots in bf16).
"""
import numpy as np
import pytest
import torch

import compressed_decode_attention_fdms_b200 as fd
import workloads as wk
from _pair import Pair

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _expected(oc, layer, batch, wl):
    """(slots, bytes) a decode of `batch` sequences of `layer` scans."""
    elt = 1 if wl.kv_dtype.startswith("fp8") else 2
    row = 2 * wl.head_dim * elt
    slots = nbytes = 0
    for b in range(batch):
        r, n = int(oc.r[layer, b]), int(oc.n[layer, b])
        for h in range(wl.kv_heads):
            ln = int(np.count_nonzero(oc.keep[layer, b, :r, h]))
            slots += ln + (n - r)
            if wl.kv_dtype == "fp8_e4m3_block":
                sealed = ln // 64 * 64
                nbytes += sealed * row + (ln - sealed + n - r) * 2 * row
            else:
                nbytes += (ln + n - r) * row
    return slots, nbytes


@pytest.mark.parametrize("kv_dtype,decode_ctas", [("bf16", 0), ("bf16", 148), ("fp8_e4m3", 0),
                                                   ("fp8_e4m3_block", 0), ("fp8_e4m3_block", 148)])
def test_layout_and_decode_counters(kv_dtype, decode_ctas):
    wl = wk.scaled(wk.get("llama1b_c8"), layers=2, ctx=300, steps=0, kv_dtype=kv_dtype,
                   head_dim=128 if kv_dtype.startswith("fp8") else 64)
    p = Pair(wl, decode_ctas=decode_ctas, max_seq_len=400)
    try:
        lay = fd.fdms_decode_layout(p.cache, wl.batch)
        cs, split = lay["cluster_ctas"], lay["split_ctas"]
        nh = wl.batch * wl.kv_heads
        if decode_ctas > 0:
            assert cs == 0                       # the global plan
        else:
            assert cs in (2, 4, 8) and nh * cs <= torch.cuda.get_device_properties(0).multi_processor_count
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        if decode_ctas > 0:
            assert split == decode_ctas
        else:   # every resident slot of the device: a whole number of CTAs per SM
            assert split >= sms and split % sms == 0
        with pytest.raises(fd.FdmsError):
            fd.fdms_decode_layout(p.cache, wl.batch + 1)
        for layer in range(wl.layers):
            p.append(layer, wk.prefill_inputs(wl, layer))
        g = torch.Generator().manual_seed(5)
        for step in range(3):
            for layer in range(wl.layers):
                p.append(layer, wk.decode_inputs(wl, layer, step))
                q = torch.randn((wl.batch, wl.q_heads, wl.head_dim), generator=g).to(torch.bfloat16)
                st0 = fd.fdms_cache_stats(p.cache)
                p.decode(layer, q)
                st1 = fd.fdms_cache_stats(p.cache)
                slots, nbytes = _expected(p.oc, layer, wl.batch, wl)
                assert st1["decode_calls"] - st0["decode_calls"] == 1
                assert st1["slots_decoded"] - st0["slots_decoded"] == slots, (layer, step)
                assert st1["bytes_decoded"] - st0["bytes_decoded"] == nbytes, (layer, step)
                assert st1["error"] == 0
    finally:
        p.close()

"""Test helper: drive the CUDA cache and the fp64 oracle with the same inputs.

Inputs come from ``workloads`` (seeded); the oracle sees the exact bf16 bits the
GPU sees. Nothing here computes the method: comparisons only.
"""
from __future__ import annotations

import numpy as np
import torch

import compressed_decode_attention_fdms_b200 as fd
import workloads as wk
from oracle.cache import OracleCache


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class Pair:
    def __init__(self, wl: wk.Workload, device=0, num_blocks=0, decode_ctas=0, max_seq_len=None,
                 oracle_capacity=None):
        self.wl = wl
        self.device = device
        msl = max_seq_len or wl.max_seq_len
        self.cfg = fd.make_config(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim,
                                  wl.window, wl.period, msl, num_blocks, wl.kv_dtype,
                                  0.0, decode_ctas)
        self.cache = fd.fdms_cache_create(self.cfg, device)
        self.oc = OracleCache(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim,
                              wl.window, wl.period, wl.kv_dtype,
                              capacity=oracle_capacity or msl)

    def close(self):
        fd.fdms_cache_destroy(self.cache)

    # ------------------------------------------------------------- steps
    def append(self, layer, inp, kv_scale=None):
        dev = f"cuda:{self.device}"
        B = inp["k"].shape[0]
        n_new = inp["n_new"].to(torch.int32)
        fd.fdms_append_evict(self.cache, layer, B, n_new.to(dev), inp["max_new"],
                             inp["k"].to(dev).contiguous(), inp["v"].to(dev).contiguous(),
                             inp["keep"].to(dev).contiguous(),
                             None if kv_scale is None else kv_scale.to(dev))
        self.oc.append(layer, n_new.cpu().numpy(), bits(inp["k"]), bits(inp["v"]),
                       inp["keep"].cpu().numpy(),
                       None if kv_scale is None else kv_scale.cpu().numpy())

    def decode(self, layer, q, f32=False):
        dev = f"cuda:{self.device}"
        B = q.shape[0]
        qd = q.to(dev).contiguous()
        if f32:
            out = torch.empty(q.shape, dtype=torch.float32, device=dev)
            lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
            fd.fdms_decode_attn_f32(self.cache, layer, B, qd, out, lse)
            return out, lse
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        fd.fdms_decode_attn(self.cache, layer, B, qd, out)
        return out

    def oracle_out(self, layer, q, mode="stored", seqs=None):
        qb = bits(q)
        seqs = range(q.shape[0]) if seqs is None else seqs
        return {b: self.oc.attention(layer, b, qb[b], mode=mode) for b in seqs}

    # ----------------------------------------------------------- checks
    def check_heads(self, layer, seqs=None, heads=None):
        """Store and ring of every (seq, head): bit-exact against the oracle."""
        wl = self.wl
        elt = 1 if wl.kv_dtype == "fp8_e4m3" else 2
        for b in (range(wl.batch) if seqs is None else seqs):
            for h in (range(wl.kv_heads) if heads is None else heads):
                got = fd.fdms_cache_read_head(self.cache, layer, b, h)
                pos, kp, vp = self.oc.store(layer, b, h)
                rpos, rk, rv, rkeep = self.oc.ring(layer, b, h)
                ctx = f"layer {layer} seq {b} head {h}"
                assert got["num_tokens"] == int(self.oc.n[layer, b]), ctx
                assert got["resolved"] == int(self.oc.r[layer, b]), ctx
                assert got["store_len"] == len(pos), ctx
                assert got["ring_len"] == len(rpos), ctx
                n_s = len(pos)
                assert np.array_equal(got["pos"][:n_s], pos), ctx
                assert np.array_equal(got["pos"][n_s:], rpos), ctx
                assert np.array_equal(got["keep"][n_s:], rkeep), ctx
                exp_k = np.concatenate([kp, rk]) if len(rk) else kp
                exp_v = np.concatenate([vp, rv]) if len(rv) else vp
                if elt == 2:
                    gk = got["k"].view(np.uint16)
                    gv = got["v"].view(np.uint16)
                else:
                    gk, gv = got["k"], got["v"]
                assert np.array_equal(gk, exp_k.reshape(gk.shape)), ctx + " K payload"
                assert np.array_equal(gv, exp_v.reshape(gv.shape)), ctx + " V payload"
                if wl.kv_dtype == "fp8_e4m3" and len(got["scale"]):
                    sc = self.oc.kv_scale[layer, b, h]
                    assert np.all(got["scale"] == sc[None, :]), ctx + " scales"

    def check_stats(self):
        got = fd.fdms_cache_stats(self.cache)
        exp = self.oc.stats()
        for k, v in exp.items():
            assert got[k] == v, (k, got[k], v)
        assert got["error"] == 0
        return got

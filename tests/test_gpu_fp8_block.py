"""Per-block FP8 cache (FDMS_KV_FP8_E4M3_BLOCK) against the oracle's second FP8
reading (needs a B200).

Appends go through the block-mode kernels (a warp per head for a few tokens, a
CTA per head for 64 or more); after each call every head is read back and
compared bit-exactly: positions, lengths, keep bits, the
codes and (K, V) scales of every sealed block, the bf16 rows of the staging
block and of the ring, and the byte and saturation counters. Decode (sealed
blocks in E4M3 with their own scales, the staged block and the ring in bf16)
is compared with the oracle's attention over the same stored values (3e-3,
bf16 and fp32 outputs) and over the unquantised inputs (3e-2).
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

B64 = OracleCache.BLOCK
TOL_MIRROR = 3e-3   # against the oracle's own quantisation of the sealed blocks
TOL_TRUE = 3e-2     # the stated FP8 bar, against the unquantised bf16 inputs


def _half_ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-300)))
    return np.where(x == 0, 0.0, 2.0 ** (e - 8))


def _check_decode(cache, oc, layer, batch, q_heads, head_dim, seed):
    """Decode of every sequence of `layer` (bf16 and fp32 outputs) against the
    oracle over the stored values and over the true inputs."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((batch, q_heads, head_dim), generator=g).to(torch.bfloat16)
    qd = q.to("cuda")
    out = torch.empty_like(qd)
    out32 = torch.empty((batch, q_heads, head_dim), dtype=torch.float32, device="cuda")
    fd.fdms_decode_attn(cache, layer, batch, qd, out)
    fd.fdms_decode_attn_f32(cache, layer, batch, qd, out32)
    torch.cuda.synchronize()
    o16 = out.float().cpu().numpy().astype(np.float64)
    o32 = out32.cpu().numpy().astype(np.float64)
    for b in range(batch):
        ref = oc.attention(layer, b, bits(q[b]))
        err = float(np.max(np.abs(o16[b] - ref) - _half_ulp_bf16(ref)))
        assert err <= TOL_MIRROR, (layer, b, err)
        assert float(np.max(np.abs(o32[b] - ref))) <= TOL_MIRROR, (layer, b)
        ref_t = oc.attention(layer, b, bits(q[b]), mode="true")
        assert float(np.max(np.abs(o16[b] - ref_t) - _half_ulp_bf16(ref_t))) <= TOL_TRUE, (layer, b)


def _bf16_rows(raw):
    """[n][2 D] host bytes of bf16 rows -> uint16 [n][D]."""
    return np.ascontiguousarray(raw).view(np.uint16)


def _check_head(cache, oc, layer, b, h):
    got = fd.fdms_cache_read_head(cache, layer, b, h)
    ctx = (layer, b, h)
    assert got["num_tokens"] == int(oc.n[layer, b]), ctx
    assert got["resolved"] == int(oc.r[layer, b]), ctx
    pos, kp, vp = oc.store(layer, b, h)                  # bf16 bits of the survivors
    rpos, rk, rv, rkeep = oc.ring(layer, b, h)
    n_s = len(pos)
    assert got["store_len"] == n_s, ctx
    assert np.array_equal(got["pos"][:n_s], pos), ctx
    assert np.array_equal(got["pos"][n_s:], rpos), ctx
    assert np.array_equal(got["keep"][n_s:], rkeep), ctx
    spos, kq, vq, scales, _ = oc.sealed_blocks(layer, b, h)
    ns = len(spos)
    D = oc.D
    if ns:
        assert np.array_equal(got["k"][:ns, :D], kq), ctx + ("sealed K",)
        assert np.array_equal(got["v"][:ns, :D], vq), ctx + ("sealed V",)
        assert not got["k"][:ns, D:].any() and not got["v"][:ns, D:].any(), ctx
        exp_sc = np.repeat(scales, B64, axis=0)
        assert np.array_equal(got["scale"][:ns], exp_sc), ctx + ("scales",)
    # staged rows (the store's open block) and the ring: bf16, scale 0
    assert np.array_equal(_bf16_rows(got["k"][ns:n_s]), kp[ns:].reshape(-1, D)), ctx
    assert np.array_equal(_bf16_rows(got["v"][ns:n_s]), vp[ns:].reshape(-1, D)), ctx
    assert np.array_equal(_bf16_rows(got["k"][n_s:]), rk.reshape(-1, D)), ctx
    assert np.array_equal(_bf16_rows(got["v"][n_s:]), rv.reshape(-1, D)), ctx
    assert not got["scale"][ns:].any(), ctx


def _append(cache, oc, layer, inp):
    dev = "cuda:0"
    B = inp["k"].shape[0]
    n_new = inp["n_new"].to(torch.int32)
    fd.fdms_append_evict(cache, layer, B, n_new.to(dev), inp["max_new"],
                         inp["k"].to(dev).contiguous(), inp["v"].to(dev).contiguous(),
                         inp["keep"].to(dev).contiguous())
    oc.append(layer, n_new.cpu().numpy(), bits(inp["k"]), bits(inp["v"]),
              inp["keep"].cpu().numpy())


# decode_ctas 0: per-head clusters; 148: the global plan
@pytest.mark.parametrize("head_dim,window,period,decode_ctas",
                         [(128, 16, 1, 0), (128, 16, 1, 148), (64, 5, 7, 0), (64, 5, 7, 148),
                          (128, 0, 64, 0)])
def test_block_fp8_appends_match_the_oracle(head_dim, window, period, decode_ctas):
    wl = wk.scaled(wk.get("qwen8b_c8_fp8"), layers=2, batch=2, ctx=700, steps=0,
                   head_dim=head_dim, window=window, period=period, rate=0.4)
    cap = wl.ctx + 500
    cfg = fd.make_config(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                         wl.period, cap, 0, "fp8_e4m3_block", decode_ctas=decode_ctas)
    cache = fd.fdms_cache_create(cfg, 0)
    oc = OracleCache(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                     wl.period, "fp8_e4m3_block", capacity=cap)
    rng = np.random.default_rng(head_dim + window + period)
    if decode_ctas == 0:   # per-head clusters at this batch
        assert fd.fdms_decode_layout(cache, wl.batch)["cluster_ctas"] in (2, 4, 8)
    try:
        for layer in range(wl.layers):
            _append(cache, oc, layer, wk.prefill_inputs(wl, layer))
            for b in range(wl.batch):
                for h in range(wl.kv_heads):
                    _check_head(cache, oc, layer, b, h)
        for step in range(40):
            layer = step % wl.layers
            if step % 7 == 3:   # a few tokens at once, none for one sequence
                inp = wk.prefill_inputs(wk.scaled(wl, ctx=5), layer)
                inp = {**inp, "n_new": torch.tensor([5, 0], dtype=torch.int32)}
            elif step in (21, 30):   # a large call (a CTA per head) over staged and ring rows
                inp = wk.prefill_inputs(wk.scaled(wl, ctx=150), layer)
                inp = {**inp, "n_new": torch.tensor([150, 97], dtype=torch.int32)}
            else:
                inp = wk.decode_inputs(wl, layer, step)
            _append(cache, oc, layer, inp)
            if step % 5 == 0 or step == 39:
                b, h = int(rng.integers(wl.batch)), int(rng.integers(wl.kv_heads))
                _check_head(cache, oc, layer, b, h)
            if step % 4 == 0:
                _check_decode(cache, oc, layer, wl.batch, wl.q_heads, wl.head_dim, 100 + step)
        for layer in range(wl.layers):
            for b in range(wl.batch):
                for h in range(wl.kv_heads):
                    _check_head(cache, oc, layer, b, h)
        st = fd.fdms_cache_stats(cache)
        ost = oc.stats()
        assert st["error"] == 0
        assert st["bytes_compact"] == ost["bytes_compact"]
        assert st["slots_store"] == ost["slots_store"]
        assert st["fp8_saturations"] == ost["fp8_saturations"]
        for layer in range(wl.layers):
            _check_decode(cache, oc, layer, wl.batch, wl.q_heads, wl.head_dim, 7 + layer)
    finally:
        fd.fdms_cache_destroy(cache)


def test_block_fp8_large_append_out_of_blocks_leaves_head_unchanged():
    """The CTA-per-head append reserves a head's seals before any write: with
    room for one head's seven sealed blocks of two, exactly one head appends
    (which one depends on the order the CTAs reach the pool), the other is left
    unchanged, OUT_OF_BLOCKS is latched and the pool count stays exact."""
    wl = wk.scaled(wk.get("tiny"), ctx=500, steps=0, window=0, rate=1.0, head_dim=64)
    cfg = fd.make_config(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                         wl.period, 640, 8, "fp8_e4m3_block")   # a pool of 8 blocks
    cache = fd.fdms_cache_create(cfg, 0)
    oc = OracleCache(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                     wl.period, "fp8_e4m3_block", capacity=640)
    dev = "cuda:0"
    try:
        inp = wk.prefill_inputs(wl, 0)
        fd.fdms_append_evict(cache, 0, 1, inp["n_new"].to(dev), inp["max_new"],
                             inp["k"].to(dev), inp["v"].to(dev), inp["keep"].to(dev))
        oc.append(0, inp["n_new"].numpy(), bits(inp["k"]), bits(inp["v"]), inp["keep"].numpy())
        st = fd.fdms_cache_stats(cache)
        assert st["error"] == fd.FDMS_ERR_OUT_OF_BLOCKS
        assert st["blocks_used"] == 7 and st["blocks_free"] == 1
        infos = [fd.fdms_cache_read_head(cache, 0, 0, h) for h in range(wl.kv_heads)]
        done = [h for h in range(wl.kv_heads) if infos[h]["num_tokens"] == 500]
        left = [h for h in range(wl.kv_heads) if infos[h]["num_tokens"] == 0]
        assert len(done) == 1 and len(left) == 1, [i["num_tokens"] for i in infos]
        assert infos[left[0]]["store_len"] == 0
        _check_head(cache, oc, 0, 0, done[0])   # the head that fits: bit-exact
    finally:
        fd.fdms_cache_destroy(cache)

"""GPU path against the fp64 oracle, through the C ABI (needs a B200).

Bars (max-abs on the decode output; a bf16 output may in addition be off by
half a bf16 ulp of the exact value, its own final rounding):
  * BF16 cache: 3e-3 against the oracle (the stated tolerance).
  * FP8 cache: the oracle models the FP8 cache (its own E4M3 encoding times
    the scale). The stated tolerance is 3e-2; the check uses 3e-3, since the
    GPU and the oracle then differ only by fp32 vs fp64 arithmetic. Against the
    unquantised bf16 inputs the gap is the E4M3 quantisation error of the
    method itself (up to 1/16 relative per element), which averages below 3e-2
    only when many tokens are visible; that check runs on the 8K-context shapes
    (``true_tol``), not on short sequences.
  * fp32 output: 2e-5 + 2e-5 * |o| against the mirror oracle. Derivation: scores
    and sums are fp32 (unit roundoff 6e-8) over at most a few thousand terms,
    and 2^x uses the hardware approximation (relative error below 2^-21), so
    the relative error of o stays below ~1e-5.
  * Compaction (positions, keep bits, lengths, payload bytes, scales) and the
    integer counters: bit-exact.
"""
import numpy as np
import pytest
import torch

import workloads as wk

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from _pair import Pair, bits  # noqa: E402

TOL_BF16 = 3e-3
TOL_FP8_TRUE = 3e-2
TOL_FP8_MIRROR = 3e-3


def _half_ulp_bf16(x):
    """Half a unit in the last place of bf16 (8 significant bits) at |x|."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - 7)


def _max_err(gpu_out, ref: dict):
    """Largest error of a bf16 output beyond its own final rounding.

    The output is stored as bf16, so even the exact result rounded to bf16 is
    off by up to half an ulp (3.9e-3 for |o| in [1, 2)). The tolerances bound
    the computation; the final rounding is allowed on top of them.
    """
    g = gpu_out.float().cpu().numpy()
    return max(float(np.max(np.abs(g[b] - ref[b]) - _half_ulp_bf16(ref[b]))) for b in ref)


def _f32_ok(gpu_f32, ref: dict):
    g = gpu_f32.cpu().numpy().astype(np.float64)
    for b in ref:
        err = np.abs(g[b] - ref[b])
        assert np.all(err <= 2e-5 + 2e-5 * np.abs(ref[b])), float(err.max())


def run_workload(wl, steps=None, check_every=1, num_blocks=0, decode_ctas=0, prefill_seqs=None,
                 true_tol=None):
    p = Pair(wl, num_blocks=num_blocks, decode_ctas=decode_ctas)
    try:
        for layer in range(wl.layers):
            p.append(layer, wk.prefill_inputs(wl, layer, seqs=prefill_seqs))
            p.check_heads(layer)
        for step in range(wl.steps if steps is None else steps):
            for layer in range(wl.layers):
                p.append(layer, wk.decode_inputs(wl, layer, step))
                q = wk.decode_query(wl, layer, step)
                out = p.decode(layer, q)
                ref = p.oracle_out(layer, q)
                tol = TOL_BF16 if wl.kv_dtype == "bf16" else TOL_FP8_MIRROR
                assert _max_err(out, ref) <= tol, (layer, step)
                if wl.kv_dtype == "fp8_e4m3" and true_tol is not None:
                    ref_t = p.oracle_out(layer, q, mode="true")
                    assert _max_err(out, ref_t) <= true_tol
                if step % check_every == 0:
                    of, lse = p.decode(layer, q, f32=True)
                    _f32_ok(of, ref)
                    p.check_heads(layer)
        p.check_stats()
    finally:
        p.close()


def test_tiny_workload_all_steps():
    run_workload(wk.get("tiny"))


# Scaled-down shapes of the larger workloads: several 64-slot pages, ragged tails,
# all group sizes and head dims the configs use.
SMALL = {
    "llama_shape_c1": wk.scaled(wk.get("llama1b_c1"), layers=2, ctx=1000, steps=5),
    "llama_shape_c3_ragged": wk.scaled(wk.get("llama1b_c8"), layers=2, batch=3, ctx=777, steps=4),
    "qwen_shape_fp8": wk.scaled(wk.get("qwen8b_c8_fp8"), layers=2, batch=2, ctx=901, steps=4),
    "long_fp8_p64": wk.scaled(wk.get("qwen8b_long_fp8"), layers=1, batch=4,
                              ctx_range=(60, 1500), steps=70),
}


# Decode modes: "auto" (decode_ctas = 0) runs these few-head calls as one
# cluster of CTAs per head; "plan" (an explicit grid) forces the global tile
# plan, which calls with many heads use.
MODES = {"auto": 0, "plan": 148}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("name", list(SMALL))
def test_scaled_workloads(name, mode):
    wl = SMALL[name]
    true_tol = TOL_FP8_TRUE if name == "qwen_shape_fp8" else None
    run_workload(wl, check_every=max(1, wl.steps // 3), true_tol=true_tol,
                 decode_ctas=MODES[mode])


# Edge cases: window / period / group / head dim / dtype sweeps on tiny shapes.
EDGE = [
    dict(window=0, period=1), dict(window=1, period=1), dict(window=16, period=64),
    dict(window=0, period=64), dict(window=256, period=1, ctx=100),
    dict(q_heads=2, kv_heads=2), dict(q_heads=8, kv_heads=1), dict(q_heads=16, kv_heads=2),
    dict(head_dim=128), dict(kv_dtype="fp8_e4m3"), dict(kv_dtype="fp8_e4m3", head_dim=64),
    dict(kv_dtype="fp8_e4m3", q_heads=2, kv_heads=1, head_dim=128, period=5, window=3),
]


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("i", range(len(EDGE)))
def test_edge_shapes(i, mode):
    base = wk.scaled(wk.get("tiny"), ctx=200, steps=6, batch=2, rate=0.3)
    run_workload(wk.scaled(base, **EDGE[i]), decode_ctas=MODES[mode])


@pytest.mark.parametrize("ctx", [0, 1, 63, 64, 65, 127, 128, 129])
def test_store_lengths_around_page_boundaries(ctx):
    # W = 0, keep-all: the store length is exactly ctx + steps
    wl = wk.scaled(wk.get("tiny"), ctx=max(ctx, 1), steps=3, window=0, rate=1.0)
    p = Pair(wl)
    try:
        if ctx > 0:
            p.append(0, wk.prefill_inputs(wl, 0))
            p.check_heads(0)
        for step in range(3):
            p.append(0, wk.decode_inputs(wl, 0, step))
            q = wk.decode_query(wl, 0, step)
            assert _max_err(p.decode(0, q), p.oracle_out(0, q)) <= TOL_BF16
            p.check_heads(0)
    finally:
        p.close()


def test_all_evicted_outside_window_and_keep_all():
    for rate in (0.0, 1.0):
        run_workload(wk.scaled(wk.get("tiny"), ctx=300, steps=4, rate=rate))


def test_empty_sequences_in_a_ragged_batch():
    wl = wk.scaled(wk.get("llama1b_c8"), layers=1, batch=4, ctx=300, steps=3)
    run_workload(wl, prefill_seqs=[0, 2])


def test_single_visible_token_is_returned_exactly():
    # W = 1, nothing kept: after each decode step only the newest token is visible
    wl = wk.scaled(wk.get("tiny"), ctx=50, steps=3, window=1, rate=0.0)
    p = Pair(wl)
    try:
        p.append(0, wk.prefill_inputs(wl, 0))
        for step in range(3):
            inp = wk.decode_inputs(wl, 0, step)
            p.append(0, inp)
            q = wk.decode_query(wl, 0, step)
            out = p.decode(0, q)
            G = wl.group
            for qh in range(wl.q_heads):
                assert torch.equal(out[0, qh].cpu(), inp["v"][0, 0, qh // G])
    finally:
        p.close()


def test_decode_is_deterministic_and_split_invariant():
    wl = wk.scaled(wk.get("llama1b_c8"), layers=1, batch=3, ctx=2000, steps=1)
    outs = []
    for ctas in (0, 7, 300):
        p = Pair(wl, decode_ctas=ctas)
        try:
            p.append(0, wk.prefill_inputs(wl, 0))
            p.append(0, wk.decode_inputs(wl, 0, 0))
            q = wk.decode_query(wl, 0, 0)
            a, _ = p.decode(0, q, f32=True)
            b, _ = p.decode(0, q, f32=True)
            assert torch.equal(a, b)
            outs.append(a.cpu())
        finally:
            p.close()
    for o in outs[1:]:
        assert torch.allclose(o, outs[0], atol=1e-5, rtol=1e-5)


def test_lse_matches_oracle():
    wl = wk.scaled(wk.get("tiny"), ctx=300, steps=1)
    p = Pair(wl)
    try:
        p.append(0, wk.prefill_inputs(wl, 0))
        p.append(0, wk.decode_inputs(wl, 0, 0))
        q = wk.decode_query(wl, 0, 0)
        _, lse = p.decode(0, q, f32=True)
        from oracle.numerics import bf16_to_f64
        qf = bf16_to_f64(bits(q))[0]
        G = wl.group
        for qh in range(wl.q_heads):
            h = qh // G
            S = np.flatnonzero(p.oc.visible(0, 0, h))
            k, _ = p.oc.values(0, 0, h, S)
            s = (k @ qf[qh]) / np.sqrt(wl.head_dim)
            ref = np.log(np.sum(np.exp(s - s.max()))) + s.max()
            assert abs(float(lse[0, qh]) - ref) <= 1e-4 * max(1.0, abs(ref))
    finally:
        p.close()


def test_caller_fp8_scales():
    wl = wk.scaled(wk.get("tiny"), ctx=120, steps=2, kv_dtype="fp8_e4m3")
    p = Pair(wl)
    try:
        sc = torch.tensor([[[0.01, 0.02], [0.005, 0.04]]], dtype=torch.float32)
        p.append(0, wk.prefill_inputs(wl, 0), kv_scale=sc)
        for step in range(2):
            p.append(0, wk.decode_inputs(wl, 0, step))
            q = wk.decode_query(wl, 0, step)
            assert _max_err(p.decode(0, q), p.oracle_out(0, q)) <= TOL_FP8_MIRROR
        p.check_heads(0)
        st = p.check_stats()
        assert st["fp8_saturations"] > 0     # 0.005 * 448 = 2.24 < max |N(0,1)|
    finally:
        p.close()


def test_pool_exhaustion_latches_error_and_leaves_head_unchanged():
    """A head whose survivors do not fit is left unchanged, the pool counter
    does not move past the blocks handed out, and a later, smaller request
    still gets the blocks that are left."""
    import compressed_decode_attention_fdms_b200 as fd
    wl = wk.scaled(wk.get("tiny"), ctx=500, steps=0, window=0, rate=1.0)
    p = Pair(wl, num_blocks=9, max_seq_len=640, oracle_capacity=640)   # 2 heads x 8 blocks
    dev = "cuda:0"
    try:
        p.append(0, wk.prefill_inputs(wl, 0))
        st = fd.fdms_cache_stats(p.cache)
        assert st["error"] == fd.FDMS_ERR_OUT_OF_BLOCKS
        infos = [fd.fdms_cache_read_head(p.cache, 0, 0, h) for h in range(2)]
        assert infos[0]["num_tokens"] == 500 and infos[0]["store_len"] == 500
        assert infos[1]["num_tokens"] == 0 and infos[1]["store_len"] == 0   # first fit, head order
        assert st["blocks_used"] == 8 and st["blocks_free"] == 1
        # 30 more tokens: head 0 keeps none (no block needed), head 1 keeps all
        # (one block): the block left over goes to head 1
        more = wk.prefill_inputs(wk.scaled(wl, ctx=30), 0)
        keep = more["keep"].clone()
        keep[:, :, 0] = 0
        keep[:, :, 1] = 1
        fd.fdms_append_evict(p.cache, 0, 1, more["n_new"].to(dev), more["max_new"],
                             more["k"].to(dev), more["v"].to(dev), keep.to(dev))
        st = fd.fdms_cache_stats(p.cache)
        assert st["blocks_used"] == 9 and st["blocks_free"] == 0
        h1 = fd.fdms_cache_read_head(p.cache, 0, 0, 1)
        assert h1["num_tokens"] == 30 and h1["store_len"] == 30
        assert np.array_equal(h1["pos"][:30], np.arange(30))
        assert np.array_equal(h1["k"].view(np.uint16).reshape(30, -1),
                              bits(more["k"][0, :30, 1]).reshape(30, -1))
        h0 = fd.fdms_cache_read_head(p.cache, 0, 0, 0)
        assert h0["num_tokens"] == 530 and h0["store_len"] == 500
        # the pool is now full: a step that needs a block fails and changes nothing
        step = wk.decode_inputs(wl, 0, 0)
        skeep = step["keep"].clone()
        skeep[:] = 1
        for _ in range(40):     # head 1 fills its block (64 slots) and needs another
            fd.fdms_append_evict(p.cache, 0, 1, step["n_new"].to(dev), 1, step["k"].to(dev),
                                 step["v"].to(dev), skeep.to(dev))
        st = fd.fdms_cache_stats(p.cache)
        assert st["blocks_used"] == 9 and st["blocks_free"] == 0
        h1 = fd.fdms_cache_read_head(p.cache, 0, 0, 1)
        assert h1["store_len"] == 64 and h1["num_tokens"] == 64
    finally:
        p.close()


def test_sequence_longer_than_max_latches_device_error():
    import compressed_decode_attention_fdms_b200 as fd
    wl = wk.scaled(wk.get("tiny"), ctx=100, steps=0)
    p = Pair(wl, max_seq_len=128, oracle_capacity=256)
    try:
        dev = "cuda:0"
        p.append(0, wk.prefill_inputs(wl, 0))
        more = wk.prefill_inputs(wk.scaled(wl, ctx=40), 0)     # 100 + 40 > 128
        fd.fdms_append_evict(p.cache, 0, 1, more["n_new"].to(dev), more["max_new"],
                             more["k"].to(dev), more["v"].to(dev), more["keep"].to(dev))
        st = fd.fdms_cache_stats(p.cache)
        assert st["error"] == fd.FDMS_ERR_DEVICE
        assert fd.fdms_cache_read_head(p.cache, 0, 0, 0)["num_tokens"] == 100
    finally:
        p.close()


def test_host_side_argument_errors():
    import compressed_decode_attention_fdms_b200 as fd
    wl = wk.get("tiny")
    p = Pair(wl)
    try:
        lib = fd.load_library()
        import ctypes
        h = ctypes.c_void_p(p.cache.handle)
        assert lib.fdms_append_evict(h, 5, 1, None, 1, None, None, None, None, None) == \
            fd.FDMS_ERR_INVALID_ARG
        assert lib.fdms_decode_attn(h, 0, 2, None, None, None) == fd.FDMS_ERR_INVALID_ARG
        x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
        # bf16 cache must not receive FP8 scales
        assert lib.fdms_append_evict(h, 0, 1, ctypes.c_void_p(x.data_ptr()), 1,
                                     ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                     ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                     None) == fd.FDMS_ERR_INVALID_ARG
        assert fd.fdms_cache_stats(p.cache)["error"] == 0
    finally:
        p.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("window,period", [(16, 1), (0, 1), (5, 7), (16, 64)])
def test_mixed_append_sizes(kv_dtype, window, period):
    """Appends of 1..16 tokens (warp path) mixed with larger ones (CTA path)."""
    rng = np.random.default_rng(window * 100 + period)
    wl = wk.scaled(wk.get("tiny"), batch=3, ctx=40, steps=0, window=window, period=period,
                   kv_dtype=kv_dtype, rate=0.4)
    p = Pair(wl, max_seq_len=1200, oracle_capacity=1200)
    try:
        step = 0
        for it in range(24):
            m = int(rng.choice([1, 1, 2, 5, 16, 17, 40, 0]))
            big = wk.scaled(wl, ctx=max(m, 1))
            inp = wk.prefill_inputs(big, 0)
            inp = {**inp, "n_new": torch.tensor([m, max(m - 1, 0), m // 2], dtype=torch.int32)}
            p.append(0, inp)
            q = wk.decode_query(wl, 0, step)
            step += 1
            out = p.decode(0, q)
            assert _max_err(out, p.oracle_out(0, q)) <= (TOL_BF16 if kv_dtype == "bf16" else
                                                          TOL_FP8_MIRROR)
            p.check_heads(0)
        p.check_stats()
    finally:
        p.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("window,period", [(16, 1), (300, 64)])
def test_large_appends_span_chunks(kv_dtype, window, period):
    """Bulk appends of thousands of tokens onto sequences that already hold
    tokens: the positions resolved at once come from the ring and from the
    call's input and span several 1024-position chunks, whose boundaries fall
    anywhere in the store's pages; single-token steps in between."""
    rng = np.random.default_rng(window + period)
    wl = wk.scaled(wk.get("tiny"), batch=3, ctx=40, steps=0, window=window, period=period,
                   kv_dtype=kv_dtype, rate=0.35)
    p = Pair(wl, max_seq_len=9000, oracle_capacity=9000)
    try:
        step = 0
        for m in [700, 1, 2500, 1, 1, 3100, 1]:
            big = wk.scaled(wl, ctx=m)
            inp = wk.prefill_inputs(big, 0)
            n = [m, max(m - int(rng.integers(1, 300)), 0) if m > 1 else 1, m // 3]
            inp = {**inp, "n_new": torch.tensor(n, dtype=torch.int32)}
            p.append(0, inp)
            p.check_heads(0)
            q = wk.decode_query(wl, 0, step)
            step += 1
            out = p.decode(0, q)
            assert _max_err(out, p.oracle_out(0, q)) <= (TOL_BF16 if kv_dtype == "bf16" else
                                                          TOL_FP8_MIRROR)
        p.check_stats()
    finally:
        p.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("window,period", [(4, 1), (0, 1), (3, 5), (2, 40)])
def test_step_appends_back_to_back(kv_dtype, window, period):
    """Step-sized appends (one or two tokens) queued with no other work between
    them: several in a row to one layer, each of which must see the state the
    one before it left, and alternating between two layers with no decode
    between them; one decode per layer at the end. Inputs are staged on the
    device first, so the append kernels follow each other directly on the
    stream."""
    import compressed_decode_attention_fdms_b200 as fd
    dev = torch.device("cuda", 0)
    wl = wk.scaled(wk.get("tiny"), layers=2, batch=3, ctx=30, steps=0, window=window,
                   period=period, kv_dtype=kv_dtype, rate=0.4)
    p = Pair(wl, max_seq_len=96, oracle_capacity=96)
    tol = TOL_BF16 if kv_dtype == "bf16" else TOL_FP8_MIRROR
    try:
        for layer in range(2):
            p.append(layer, wk.prefill_inputs(wl, layer))
        order = [0, 0, 0, 1, 0, 1, 1, 0, 1, 1, 1, 0, 0, 1, 0, 0]
        staged = []
        for i, layer in enumerate(order):
            if i % 3 == 2:   # two tokens for some sequences, none for one
                inp = wk.prefill_inputs(wk.scaled(wl, ctx=2), layer)
                n = [2, 1, 0]
                inp = {**inp, "n_new": torch.tensor(n[i % 3:] + n[:i % 3], dtype=torch.int32)}
            else:
                inp = wk.decode_inputs(wl, layer, i)
            d = {k: (t.to(dev).contiguous() if torch.is_tensor(t) else t) for k, t in inp.items()}
            staged.append((layer, inp, d))
        torch.cuda.synchronize()
        for layer, _, d in staged:
            fd.fdms_append_evict(p.cache, layer, wl.batch, d["n_new"].to(torch.int32),
                                 d["max_new"], d["k"], d["v"], d["keep"])
        torch.cuda.synchronize()
        for layer, inp, _ in staged:
            p.oc.append(layer, inp["n_new"].to(torch.int32).numpy(), bits(inp["k"]),
                        bits(inp["v"]), inp["keep"].numpy())
        for layer in range(2):
            p.check_heads(layer)
            q = wk.decode_query(wl, layer, 99)
            assert _max_err(p.decode(layer, q), p.oracle_out(layer, q)) <= tol
        p.check_stats()
    finally:
        p.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("mode", list(MODES))
def test_snapshot_rules(mode, kv_dtype):
    """Decode plans from the lengths the previous decode of the layer saw (a
    snapshot) and adds what was appended since. Cases that bend the rules: a
    smaller then a larger batch than the previous decode, many tokens appended
    in between (beyond the global plan's spare tiles), two decodes with no
    append in between, a decode after appends to other layers only, and
    sequences growing unevenly; every output against the oracle."""
    wl = wk.scaled(wk.get("llama1b_c8"), layers=2, batch=6, ctx=350, steps=0, kv_dtype=kv_dtype,
                   head_dim=128 if kv_dtype == "fp8_e4m3" else 64)
    p = Pair(wl, decode_ctas=MODES[mode], max_seq_len=800)
    tol = TOL_BF16 if kv_dtype == "bf16" else TOL_FP8_MIRROR
    g = torch.Generator().manual_seed(11)
    step = [0]

    def q_of(batch):
        return torch.randn((batch, wl.q_heads, wl.head_dim), generator=g).to(torch.bfloat16)

    def decode(layer, batch):
        q = q_of(batch)
        out = p.decode(layer, q)
        ref = p.oracle_out(layer, q)
        assert _max_err(out, ref) <= tol, (layer, batch)

    def append(layer, n_per_seq):
        base = wk.scaled(wl, ctx=max(n_per_seq), steps=0)
        inp = wk.prefill_inputs(base, layer)
        inp = {**inp, "n_new": torch.tensor(n_per_seq, dtype=torch.int32),
               "max_new": max(n_per_seq)}
        # fresh values per call: shift the generator's stream by the step
        step[0] += 1
        k = inp["k"].float().roll(step[0], dims=1).to(torch.bfloat16)
        v = inp["v"].float().roll(-step[0], dims=1).to(torch.bfloat16)
        p.append(layer, {**inp, "k": k, "v": v})

    try:
        for layer in range(wl.layers):
            p.append(layer, wk.prefill_inputs(wl, layer))
        B = wl.batch
        for layer in range(wl.layers):
            decode(layer, B)                      # first decode: no snapshot yet
        for layer in range(wl.layers):
            append(layer, [1] * B)
            decode(layer, B // 2)                 # fewer sequences than the snapshot's call
        for layer in range(wl.layers):
            append(layer, [1] * B)
            decode(layer, B)                      # more sequences than the last decode's
        for layer in range(wl.layers):
            append(layer, [100] * B)              # beyond the spare tiles
            decode(layer, B)
        decode(0, B)                              # nothing appended since
        decode(0, B)
        append(1, [3] * B)                        # another layer only
        decode(0, B)
        for layer in range(wl.layers):
            append(layer, [1, 2, 0, 5, 1, 64][:B])   # uneven growth, one sequence idle
            decode(layer, B)
            append(layer, [40, 1, 1, 0, 2, 1][:B])
            decode(layer, B)
        for layer in range(wl.layers):
            p.check_heads(layer)
        p.check_stats()
    finally:
        p.close()

"""Pins of the oracle's compact-store model (CPU only).

The set definition in oracle/cache.py is checked against an event-driven
simulation of the mechanism (tokens age out of a window of W, wait in staging,
and are kept or dropped in passes once P are waiting), against popcount and
order invariants, and against dense attention with -inf masking. The memory
formula is checked against the KV-memory table printed by the FastDMS
announcement (tests/golden/kv_memory_table.txt).
"""
import os
from collections import deque

import numpy as np
import pytest

from oracle import numerics as nm
from oracle.attention import attend_dense_masked, attend_gather
from oracle.cache import OracleCache
from oracle.memory import dense_kv_bytes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def simulate(calls, keep, W, P):
    """Queue simulation: returns (store positions, staging positions) after the calls."""
    window, waiting, store, pos = deque(), [], [], 0
    for m in calls:
        for _ in range(m):
            window.append(pos)
            pos += 1
            if len(window) > W:
                waiting.append(window.popleft())
        if len(waiting) >= P:
            store.extend(p for p in waiting if keep[p])
            waiting = []
    return store, waiting + list(window)


def _rand_bits(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)   # bf16 by truncation (any bits do)


@pytest.mark.parametrize("W", [0, 1, 3, 16])
@pytest.mark.parametrize("P", [1, 2, 5, 64])
def test_store_and_ring_match_queue_simulation(W, P):
    rng = np.random.default_rng(100 * W + P)
    for trial in range(4):
        calls = [int(rng.integers(0, 90))] + [1] * int(rng.integers(0, 80))
        calls += [int(x) for x in rng.integers(0, 7, size=5)]
        total = sum(calls)
        keep = (rng.random((total, 2)) < rng.uniform(0.0, 1.0)).astype(np.uint8)
        # compare after every call
        done = 0
        oc = OracleCache(1, 1, 2, 2, 4, W, P, capacity=max(total, 1))
        for i, m in enumerate(calls):
            kb = np.zeros((1, max(m, 1), 2, 4), np.uint16)
            pad = np.zeros((1, max(m, 1), 2), np.uint8)
            pad[0, :m] = keep[done:done + m]
            oc.append(0, [m], kb, kb, pad)
            done += m
            for h in range(2):
                st, rg = simulate(calls[:i + 1], keep[:, h], W, P)
                pos, _, _ = oc.store(0, 0, h)
                rpos, _, _, rkeep = oc.ring(0, 0, h)
                assert list(pos) == st
                assert list(rpos) == rg
                assert np.array_equal(rkeep, keep[rg, h])


def test_store_len_is_popcount_and_positions_increase():
    rng = np.random.default_rng(1)
    keep = (rng.random((300, 3)) < 0.3).astype(np.uint8)
    oc = OracleCache(1, 1, 3, 3, 4, 16, 1, capacity=300)
    kb = np.zeros((1, 300, 3, 4), np.uint16)
    oc.append(0, [300], kb, kb, keep[None])
    r = int(oc.r[0, 0])
    assert r == 300 - 16
    for h in range(3):
        pos, _, _ = oc.store(0, 0, h)
        assert len(pos) == int(keep[:r, h].sum())
        assert np.all(np.diff(pos) > 0)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("W,P", [(8, 1), (8, 4), (0, 1), (0, 3)])
def test_decode_over_store_and_ring_equals_masked_dense_attention(kv_dtype, W, P):
    rng = np.random.default_rng(11 + W + P)
    L, B, Hq, Hkv, D = 1, 2, 4, 2, 8
    n_pre, steps = 40, 9
    cap = n_pre + steps
    oc = OracleCache(L, B, Hq, Hkv, D, W, P, kv_dtype=kv_dtype, capacity=cap)
    k = _rand_bits(rng, (B, cap, Hkv, D))
    v = _rand_bits(rng, (B, cap, Hkv, D))
    keep = (rng.random((B, cap, Hkv)) < 0.3).astype(np.uint8)
    oc.append(0, [n_pre, n_pre - 7], k[:, :n_pre], v[:, :n_pre], keep[:, :n_pre])
    for s in range(steps):
        n0 = oc.n[0].copy()
        kk = np.stack([k[b, n0[b]:n0[b] + 1] for b in range(B)])
        vv = np.stack([v[b, n0[b]:n0[b] + 1] for b in range(B)])
        kp = np.stack([keep[b, n0[b]:n0[b] + 1] for b in range(B)])
        oc.append(0, [1, 1], kk, vv, kp)
        q = _rand_bits(rng, (B, Hq, D))
        for b in range(B):
            o_gather = oc.attention(0, b, q[b])
            o_dense = oc.attention(0, b, q[b], routine="dense")
            assert np.allclose(o_gather, o_dense, atol=1e-12, rtol=0)
            # rebuild the visible set from the store and ring views alone
            n = int(oc.n[0, b])
            qf = nm.bf16_to_f64(q[b])
            for h in range(Hkv):
                pos, _, _ = oc.store(0, b, h)
                rpos, _, _, rkeep = oc.ring(0, b, h)
                ring_vis = rpos[(rpos >= n - W) | (rkeep == 1)]
                S = np.concatenate([pos, ring_vis])
                assert np.array_equal(np.sort(S), np.flatnonzero(oc.visible(0, b, h)))
                kf, vf = oc.values(0, b, h, S)
                o = attend_gather(qf[2 * h:2 * h + 2], kf, vf, 1 / np.sqrt(D))
                assert np.allclose(o, o_gather[2 * h:2 * h + 2], atol=1e-12, rtol=0)


def test_fp8_payload_is_the_quantised_input_with_first_call_scale():
    rng = np.random.default_rng(3)
    B, Hkv, D = 1, 2, 8
    oc = OracleCache(1, B, 2, Hkv, D, 4, 1, kv_dtype="fp8_e4m3", capacity=40)
    k = _rand_bits(rng, (B, 40, Hkv, D))
    v = _rand_bits(rng, (B, 40, Hkv, D))
    keep = np.ones((B, 40, Hkv), np.uint8)
    oc.append(0, [30], k[:, :30], v[:, :30], keep[:, :30])
    # a decode token 10x larger than anything seen saturates
    big = (nm.bf16_to_f32(k[:, 30:31]) * 10).astype(np.float32)
    kb = (big.view(np.uint32) >> 16).astype(np.uint16)
    oc.append(0, [1], kb, v[:, 30:31], keep[:, 30:31])
    for h in range(Hkv):
        amax_k = np.max(np.abs(nm.bf16_to_f32(k[0, :30, h])))
        sk = np.float32(amax_k / np.float32(448))
        assert oc.kv_scale[0, 0, h, 0] == sk
        pos, kp, _ = oc.store(0, 0, h)
        assert np.array_equal(pos, np.arange(27))
        q = (nm.bf16_to_f32(k[0, :27, h]) / sk).astype(np.float32)
        assert np.array_equal(kp, nm.e4m3_from_f32(q))
        assert np.max(np.abs(nm.e4m3_to_f64(kp))) == 448.0   # amax maps to the top code
    assert oc.saturations > 0
    st = oc.stats()
    assert st["fp8_saturations"] == oc.saturations


def _table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "kv_memory_table.txt"))
            if l.strip() and not l.startswith("#")]
    return [(r[0], int(r[1]), *map(float, r[2:])) for r in rows]


SHAPES = {"llama-3.2-1b": (16, 8, 64), "qwen3-8b": (36, 8, 128)}
TOKENS = {1: 10240, 8: 67584}      # token pools implied by the table's dense columns


def test_dense_bytes_reproduce_the_pages_kv_memory_table():
    for model, c, bf16_gib, fp8_gib, fastdms_gib, bf16_saved, fp8_saved in _table():
        L, H, D = SHAPES[model]
        b16 = dense_kv_bytes(TOKENS[c], L, H, D, 2) / 2 ** 30
        b8 = dense_kv_bytes(TOKENS[c], L, H, D, 1) / 2 ** 30
        assert f"{b16:.3f}" == f"{bf16_gib:.3f}", (model, c, b16)
        assert f"{b8:.3f}" == f"{fp8_gib:.3f}", (model, c, b8)
        # the printed ratios are the printed GiB divided (transcription check)
        assert f"{bf16_gib / fastdms_gib:.1f}" == f"{bf16_saved:.1f}"
        assert f"{fp8_gib / fastdms_gib:.1f}" == f"{fp8_saved:.1f}"


def test_per_token_dense_sizes():
    assert dense_kv_bytes(1, 16, 8, 64, 2) == 32 * 1024
    assert dense_kv_bytes(1, 36, 8, 128, 2) == 144 * 1024


def test_stats_counts():
    rng = np.random.default_rng(9)
    oc = OracleCache(2, 3, 4, 2, 8, 5, 1, capacity=64)
    k = _rand_bits(rng, (3, 50, 2, 8))
    keep = (rng.random((3, 50, 2)) < 0.5).astype(np.uint8)
    for layer in range(2):
        oc.append(layer, [50, 20, 0], k, k, keep)
    st = oc.stats()
    assert st["tokens_appended"] == 2 * 70
    exp_store = 2 * (int(keep[0, :45].sum()) + int(keep[1, :15].sum()))
    assert st["slots_store"] == exp_store
    assert st["slots_ring"] == 2 * (5 + 5) * 2
    assert st["bytes_dense_equiv"] == 140 * 2 * 2 * 8 * 2
    assert st["bytes_compact"] == (exp_store + 40) * 2 * 8 * 2

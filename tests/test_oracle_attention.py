"""Pins of the oracle's decode attention (CPU only).

Checked against: torch's scaled_dot_product_attention in fp64 (a library
routine; a boolean mask plays the part of eviction), a hand-worked two-token
example, and closed-form special cases of softmax attention.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle.attention import attend_dense_masked, attend_gather, gqa_kv_head


def _sdpa(q, k, v, visible, scale):
    qt = torch.from_numpy(q)[None, :, None, :]                 # [1][G][1][D]
    kt = torch.from_numpy(k)[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(v)[None, None].expand(1, q.shape[0], -1, -1)
    mask = torch.from_numpy(visible)[None, None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0, :, 0, :].numpy()


def test_two_token_worked_example():
    # D = 2, scale = 1/sqrt(2). q = (sqrt2, 0); k1 = (0, 0) -> s1 = 0;
    # k2 = (ln 3, 0) -> s2 = ln 3. Weights e^0 : e^ln3 = 1 : 3 -> (1/4, 3/4).
    # v1 = (4, 0), v2 = (0, 8) -> o = (1, 6).
    q = np.array([[np.sqrt(2.0), 0.0]])
    k = np.array([[0.0, 0.0], [np.log(3.0), 0.0]])
    v = np.array([[4.0, 0.0], [0.0, 8.0]])
    o, w = attend_dense_masked(q, k, v, np.array([True, True]), 1 / np.sqrt(2))
    assert np.allclose(w, [[0.25, 0.75]], atol=1e-15)
    assert np.allclose(o, [[1.0, 6.0]], atol=1e-14)
    # evicting token 2 leaves o = v1
    o, _ = attend_dense_masked(q, k, v, np.array([True, False]), 1 / np.sqrt(2))
    assert np.array_equal(o, [[4.0, 0.0]])


@pytest.mark.parametrize("n", [1, 2, 5, 9])
def test_keep_all_equals_library_sdpa(n):
    rng = np.random.default_rng(n)
    G, D = 3, 8
    q, k, v = rng.standard_normal((G, D)), rng.standard_normal((n, D)), rng.standard_normal((n, D))
    vis = np.ones(n, bool)
    ref = _sdpa(q, k, v, vis, 1 / np.sqrt(D))
    assert np.allclose(attend_dense_masked(q, k, v, vis, 1 / np.sqrt(D))[0], ref, atol=1e-13)
    assert np.allclose(attend_gather(q, k, v, 1 / np.sqrt(D)), ref, atol=1e-13)


def test_every_eviction_mask_equals_masked_sdpa_and_gather():
    # all 2^10 masks over 10 tokens (the all-evicted mask gives 0)
    rng = np.random.default_rng(7)
    G, D, n = 2, 4, 10
    q = rng.standard_normal((G, D)) * 2
    k, v = rng.standard_normal((n, D)) * 2, rng.standard_normal((n, D))
    scale = 1 / np.sqrt(D)
    for bits in itertools.product([False, True], repeat=n):
        vis = np.array(bits)
        o_dense, w = attend_dense_masked(q, k, v, vis, scale)
        o_gather = attend_gather(q, k[vis], v[vis], scale)
        if not vis.any():
            assert np.array_equal(o_dense, np.zeros((G, D)))
            assert np.array_equal(o_gather, np.zeros((G, D)))
            continue
        assert np.allclose(o_dense, o_gather, atol=1e-12, rtol=0)
        assert np.allclose(o_dense, _sdpa(q, k, v, vis, scale), atol=1e-12, rtol=0)
        assert np.all(np.abs(w.sum(axis=1) - 1) < 1e-12)
        assert np.all(w[:, ~vis] == 0)


def test_single_visible_token_returns_its_value_exactly():
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((4, 16)), rng.standard_normal((6, 16)), rng.standard_normal((6, 16))
    vis = np.zeros(6, bool)
    vis[4] = True
    o, _ = attend_dense_masked(q, k, v, vis, 0.25)
    assert np.array_equal(o, np.broadcast_to(v[4], (4, 16)))


def test_zero_query_gives_mean_of_visible_values():
    rng = np.random.default_rng(4)
    k, v = rng.standard_normal((12, 8)), rng.standard_normal((12, 8))
    vis = rng.random(12) < 0.5
    vis[0] = True
    o = attend_gather(np.zeros((2, 8)), k[vis], v[vis], 0.3)
    assert np.allclose(o, v[vis].mean(axis=0), atol=1e-14)


def test_equal_values_and_duplicate_keys():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((2, 8)), rng.standard_normal((7, 8))
    row = rng.standard_normal(8)
    o = attend_gather(q, k, np.tile(row, (7, 1)), 0.35)
    assert np.allclose(o, np.tile(row, (2, 1)), atol=1e-14)
    k[3] = k[1]
    _, w = attend_dense_masked(q, k, rng.standard_normal((7, 8)), np.ones(7, bool), 0.35)
    assert np.allclose(w[:, 3], w[:, 1], atol=1e-16)


def test_common_key_shift_leaves_output_unchanged():
    # adding c to every key adds scale*q.c to every score of a head: softmax is shift invariant
    rng = np.random.default_rng(6)
    q, k, v = rng.standard_normal((3, 8)), rng.standard_normal((9, 8)), rng.standard_normal((9, 8))
    c = rng.standard_normal(8) * 3
    a = attend_gather(q, k, v, 0.4)
    b = attend_gather(q, k + c, v, 0.4)
    assert np.allclose(a, b, atol=1e-12)


def test_identical_queries_in_a_group_give_identical_outputs():
    rng = np.random.default_rng(8)
    q = np.tile(rng.standard_normal(8), (4, 1))
    k, v = rng.standard_normal((5, 8)), rng.standard_normal((5, 8))
    o = attend_gather(q, k, v, 0.3)
    assert np.all(o == o[0])


def test_gqa_mapping_is_contiguous_groups():
    assert [gqa_kv_head(i, 32, 8) for i in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [gqa_kv_head(i, 4, 2) for i in range(4)] == [0, 0, 1, 1]

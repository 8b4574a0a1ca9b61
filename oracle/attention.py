"""Single-token decode attention over the tokens that survive eviction.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

Definition (FastDMS announcement, aiwitness.kr/community/1t3vlrx: DMS drops
KV slots per head, FastDMS decodes over the compact store of survivors). For one
query head g with query q_g, the kv head it shares with its GQA group, and the
set S of visible token positions of that kv head:

    s_j = scale * sum_c q_g[c] * k_j[c]            for j in S
    w_j = exp(s_j - max_S s) / sum_{i in S} exp(s_i - max_S s)
    o_g = sum_{j in S} w_j * v_j

``scale`` is 1/sqrt(D) unless the caller gives another. Evicting token j is the
same as setting s_j = -inf in dense attention over all tokens; routine
``attend_dense_masked`` computes it that way, ``attend_gather`` gathers S first.
An empty S gives o = 0 (reachable only with a zero window).

Readings: query head i uses kv head floor(i / G), G = Hq / Hkv (contiguous GQA
groups; the pages are silent).
"""
from __future__ import annotations

import numpy as np


def attend_dense_masked(q, k, v, visible, scale):
    """Routine (i): dense scores over all n tokens, evicted ones at -inf.

    q [G][D], k [n][D], v [n][D] (fp64), visible bool [n].
    Returns (o [G][D], w [G][n]) with w the softmax weights (0 where evicted).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    visible = np.asarray(visible, bool)
    G, D = q.shape
    if not visible.any():
        return np.zeros((G, v.shape[1])), np.zeros((G, k.shape[0]))
    s = scale * (q @ k.T)
    s = np.where(visible[None, :], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    w = e / e.sum(axis=1, keepdims=True)
    return w @ v, w


def attend_gather(q, k_vis, v_vis, scale):
    """Routine (ii): softmax over the gathered survivors only.

    q [G][D], k_vis / v_vis [|S|][D]. Returns o [G][D].
    """
    q = np.asarray(q, np.float64)
    k_vis = np.asarray(k_vis, np.float64)
    v_vis = np.asarray(v_vis, np.float64)
    if k_vis.shape[0] == 0:
        return np.zeros((q.shape[0], v_vis.shape[1] if v_vis.ndim == 2 else q.shape[1]))
    s = scale * (q @ k_vis.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return (e @ v_vis) / e.sum(axis=1, keepdims=True)


def gqa_kv_head(q_head: int, q_heads: int, kv_heads: int) -> int:
    """kv head read by a query head: floor(i / G)."""
    return q_head // (q_heads // kv_heads)

"""fp64 CPU oracle for compact-KV decode attention (DMS / FastDMS style).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import,
call or execute anything here. The CUDA library never does, and this package
never imports the CUDA library: the two share no code. Both take their inputs
from the seeded generators in ``workloads/``.

What the oracle computes, and the passage it follows (the FastDMS announcement,
aiwitness.kr/community/1t3vlrx, "FastDMS: 6.4X KV-cache compression running
faster than vLLM BF16/FP8"):

* DMS learns, per head, which KV slots of which tokens to drop (paragraph on
  DMS: per-head token eviction, up to 8x compression). Here the decision is an
  input: one keep bit per (layer, seq, kv head, token).
* FastDMS physically reclaims the dropped slots in a compact KV store, next to a
  staging area (paragraph introducing FastDMS, and the sentence under the
  KV-memory table: "KV/stage memory is the cache or cache plus staging").
  ``cache.py`` models that store: survivors in order, plus the recent-window
  ring that plays the part of the staging area.
* Decode attention reads only what survives (paragraph on decode speed at 8K).
  ``attention.py`` holds two routines for it: dense softmax with evicted
  scores set to -inf, and gather-then-softmax over the survivors.
* The KV-memory table compares vLLM BF16 and FP8 KV bytes with FastDMS bytes.
  ``memory.py`` holds the dense-equivalent byte count that reproduces the vLLM
  columns.
* BF16 and FP8 KV (table columns "vLLM BF16 KV" and "vLLM FP8 KV").
  ``numerics.py`` decodes bf16 and encodes/decodes FP8 E4M3 from the formats'
  definitions.

Readings where the pages are silent are stated in each module's header.
Everything is fp64 unless a step is fixed to another precision (the fp32
quotient before E4M3 rounding).
"""
from . import numerics, attention, cache, memory  # noqa: F401

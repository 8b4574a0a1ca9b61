"""Dense-equivalent KV bytes: what an uncompressed paged cache holds.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

The KV-memory table of the FastDMS announcement (aiwitness.kr/community/1t3vlrx,
ctx_len 8192, gen_len 128, concurrency 1 and 8) compares "vLLM BF16 KV" and
"vLLM FP8 KV" bytes with FastDMS bytes. The dense side is one K row and one V
row of D elements per token, per layer and per kv head:

    bytes = tokens * layers * 2 * kv_heads * head_dim * element_bytes

element_bytes = 2 for BF16, 1 for FP8. For Llama-3.2-1B (16 layers, 8 kv heads,
D = 64) that is 32 KiB per token in BF16; for Qwen3-8B (36 layers, 8 kv heads,
D = 128) 144 KiB. The token counts behind the table (10240 at c=1, 67584 at c=8)
are not stated on the page; they are the counts these per-token sizes imply.
"""
from __future__ import annotations


def dense_kv_bytes(tokens: int, layers: int, kv_heads: int, head_dim: int, elt: int) -> int:
    return int(tokens) * int(layers) * 2 * int(kv_heads) * int(head_dim) * int(elt)

"""KV-cache size formula.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"1. KV 캐시란" (hjr-study-book Day 3) gives the approximate size of a KV cache
as 2 (K and V) x layers x heads x head_dim x sequence length x bytes per element.
The supersilo.blog vLLM summary ("배칭과 메모리 용량") says one OPT-13B request
with a long sequence can need up to about 1.6 GB.  Per decoded layer the same
formula with layers = 1 and heads = the kv heads gives the bytes the decode
kernel must read per token.
"""


def kv_cache_bytes(num_layers: int, num_heads: int, head_dim: int, seq_len: int,
                   dtype_bytes: int) -> int:
    return 2 * num_layers * num_heads * head_dim * seq_len * dtype_bytes


def kv_bytes_per_token(num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    """One layer's K and V bytes for a single token."""
    return kv_cache_bytes(1, num_kv_heads, head_dim, 1, dtype_bytes)

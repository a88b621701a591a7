"""Host-side schedule choice of paged_kv_cache_475_b200.step (no GPU needed).

The single-pass decode is used when the (sequence, KV head) CTAs fill the GPU
(three per SM) and no context is very long; otherwise the context is split
into 512-token partitions. The bench's configurations land where the
measurements put them: the Llama-shaped batch on the fused single pass, the
100k-token batch on split-KV.
"""
from paged_kv_cache_475_b200.step import choose_partition


def test_bench_configurations():
    assert choose_partition(64, 8, 4096) is None        # Llama-shaped decode: 512 CTAs >= 3 x 148
    assert choose_partition(4, 8, 100_000) == 512        # 100k tokens: 32 CTAs, split
    assert choose_partition(256, 8, 9216) == 512         # chat trace without the cascade: one context past 8192


def test_policy_edges():
    assert choose_partition(56, 8, 8192, num_sms=148) is None  # 448 CTAs >= 444: single pass
    assert choose_partition(55, 8, 8192, num_sms=148) == 512   # 440 < 444: split
    assert choose_partition(56, 8, 8193, num_sms=148) == 512   # a context past 8192: split
    assert choose_partition(1000, 8, 1, num_sms=148) is None

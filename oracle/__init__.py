"""Float64 CPU oracles of the SAGA + Atop-N decode attention step and of the
closed-form GQA-to-SAGA key-head merge (``oracle.key_merge``).

TEST INFRASTRUCTURE: imported only by the tests, the smoke check and the
benchmark's CPU baseline. The product path never touches it.
"""
from .saga_oracle import (NEG_INF, append, decode_chain, decode_step, dense_attend,
                          f32_from_order_key, f32_order_key, key_head,
                          nth_largest, nth_largest_f32, refresh, scores,
                          select, sparse_attend, top_n_exact, topn_step, value_head)

__all__ = ["NEG_INF", "append", "decode_chain", "decode_step", "dense_attend",
           "f32_from_order_key", "f32_order_key", "key_head", "nth_largest",
           "nth_largest_f32", "refresh", "scores", "select", "sparse_attend",
           "top_n_exact", "topn_step", "value_head"]

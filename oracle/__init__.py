"""CPU oracle for exact attention (test infrastructure only).

Plain, slow, fp64 restatements of what the attention forward pass computes, used to check the CUDA
library.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import anything here; the library itself never does, and this package imports nothing from the
library.  The two sides share only the seeded input generator, which holds no attention arithmetic.

Modules:
  attention  -- the materialised definition O = softmax(scale*Q*K^T + mask)*V with LSE, per (b, h);
                dense, packed-varlen, row-sampled and single-query (decode) forms, the latter also
                with grouped KV heads, per-sequence cache lengths, over one key shard of a cache and
                over a paged cache (a page pool addressed through a per-sequence block table).
  online     -- the tiled algorithm in the order the pages give it (Q blocks outside, K/V blocks
                inside, running max m and running sum l), and the pairwise merge of softmax
                statistics of key groups, including the split-KV partial/combine form.
  brute      -- scalar pure-Python (math.fsum) evaluation for tiny inputs.
  backward   -- dQ, dK, dV: the derivative of the forward definition for an upstream gradient dO
                (whole head, dense, packed varlen, and at sampled rows of long heads).
"""
from .attention import (attention_head, attention_dense, attention_varlen, attention_rows,
                        attention_decode, attention_decode_gqa, attention_decode_shard,
                        attention_decode_paged, padded_key_mask_attention)
from .online import (tiled_online_attention, group_stats, merge_groups, softmax_by_groups,
                     split_kv_partials, combine_partials)
from .brute import brute_attention_head
from .backward import (attention_head_backward, attention_dense_backward, attention_varlen_backward,
                       attention_rows_backward)

__all__ = [
    "attention_head", "attention_dense", "attention_varlen", "attention_rows", "attention_decode",
    "attention_decode_gqa", "attention_decode_shard", "attention_decode_paged",
    "padded_key_mask_attention", "tiled_online_attention", "group_stats", "merge_groups",
    "softmax_by_groups", "split_kv_partials", "combine_partials", "brute_attention_head",
    "attention_head_backward", "attention_dense_backward", "attention_varlen_backward",
    "attention_rows_backward",
]

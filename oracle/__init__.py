"""CPU oracle for the paged KV-cache decode path (fp64, NumPy).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference legs may import or run anything in this package.
The product path (the CUDA library and its Python binding) never calls it, and
this package imports nothing from the product package.

Contents, each following the pages it cites:
- block_manager: the block engine's free list, block tables, slot mapping,
  reference counts and copy-on-write ("LLM 推理引擎内部原理" §2.3;
  "vLLM PagedAttention 解析" §3.3, §4.1, §4.2).
- cache_ops: the KV append (scatter of new tokens' K/V into their slots) and the
  block copy used by copy-on-write forks.
- paged_attention: decode attention over the block-table-addressed cache:
  walk the block table to materialise the logical K/V, then plain softmax
  attention in fp64 ("LLM 推理引擎内部原理" §2.4).

Every function is pinned by `-m "not gpu"` tests in tests/test_oracle_*.py
(worked examples from the pages, closed forms, equality with an independent
dense attention routine, permutation invariance, invariants, planted-mistake
checks). No function here is "parity unpinned".
"""

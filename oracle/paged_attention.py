"""Oracle paged decode attention (fp64).

TEST INFRASTRUCTURE (see oracle/__init__.py).

What it computes, as the pages state it:
1. Logical materialisation ("为什么PagedAttention能让大模型推理吞吐量提升数倍",
   section "Block Table：GPU上的页表": a request sees a logically contiguous KV
   cache whose blocks sit anywhere in memory; "LLM 推理引擎内部原理" §2.4: two-level
   addressing, block table -> physical block, then the offset inside the block).
   Token j of sequence s is row (table[s][j // bs], j % bs) of the cache.
2. Decode attention of the one new query per head over those ctx tokens: the
   plain definition out = softmax(scale * q K^T) V, in fp64, no partitioning.

Readings where the pages are silent: grouped-query attention (not on the pages)
maps query head h to KV head h // (Hq / Hkv); the scale is applied to the
logits before the softmax; a sequence of context length 0 gives a zero output.
The pages' kernel sketch indexes the block table with its length inside the
loop; that is read as indexing with the loop's block index.
"""
from __future__ import annotations

import numpy as np


def gather_logical(cache, table_row, ctx: int, block_size: int) -> np.ndarray:
    """The sequence's first ctx tokens as [ctx, Hkv, D] fp64, walking its block table."""
    n_blk = -(-int(ctx) // int(block_size))
    ids = np.asarray(table_row[:n_blk], dtype=np.int64)
    blocks = np.asarray(cache[ids], dtype=np.float64)          # [n_blk, bs, Hkv, D]
    flat = blocks.reshape((n_blk * block_size,) + blocks.shape[2:])
    return flat[:ctx]


def attend(q_s: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One sequence: q_s [Hq, D], K/V [ctx, Hkv, D] -> [Hq, D] fp64."""
    hq = q_s.shape[0]
    hkv = K.shape[1]
    group = hq // hkv
    out = np.zeros((hq, q_s.shape[1]), dtype=np.float64)
    if K.shape[0] == 0:
        return out
    q_s = np.asarray(q_s, dtype=np.float64)
    for h in range(hq):
        g = h // group
        x = scale * (K[:, g, :] @ q_s[h])
        p = np.exp(x - x.max())
        out[h] = (p @ V[:, g, :]) / p.sum()
    return out


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale,
                           block_size: int, seqs=None) -> np.ndarray:
    """out[s, h, :] for every sequence (or the listed `seqs`): [len, Hq, D] fp64."""
    q = np.asarray(q)
    idx = range(q.shape[0]) if seqs is None else [int(s) for s in seqs]
    out = np.zeros((len(idx), q.shape[1], q.shape[2]), dtype=np.float64)
    for i, s in enumerate(idx):
        ctx = int(context_lens[s])
        K = gather_logical(k_cache, block_tables[s], ctx, block_size)
        V = gather_logical(v_cache, block_tables[s], ctx, block_size)
        out[i] = attend(q[s], K, V, float(scale))
    return out


def paged_attention_decode_fp8(q, k_codes, v_codes, block_tables, context_lens, scale, block_size: int,
                               k_scale: float, v_scale: float, seqs=None) -> np.ndarray:
    """Decode attention over an FP8 (e4m3) cache: the logical K/V are the
    dequantised cache values decode(code) * scale (oracle.fp8), then the same
    fp64 attention as paged_attention_decode."""
    from oracle import fp8
    q = np.asarray(q)
    idx = range(q.shape[0]) if seqs is None else [int(s) for s in seqs]
    out = np.zeros((len(idx), q.shape[1], q.shape[2]), dtype=np.float64)
    for i, s in enumerate(idx):
        ctx = int(context_lens[s])
        n_blk = -(-ctx // int(block_size))
        ids = np.asarray(block_tables[s][:n_blk], dtype=np.int64)
        kb = fp8.dequantize(np.asarray(k_codes[ids]), k_scale)
        vb = fp8.dequantize(np.asarray(v_codes[ids]), v_scale)
        K = kb.reshape((n_blk * block_size,) + kb.shape[2:])[:ctx]
        V = vb.reshape((n_blk * block_size,) + vb.shape[2:])[:ctx]
        out[i] = attend(q[s], K, V, float(scale))
    return out


def paged_attention_multi_query(q, k_cache, v_cache, block_tables, context_lens, query_start, scale,
                                block_size: int) -> np.ndarray:
    """Several new query tokens per sequence over the paged cache, with a
    causal mask: chunked prefill ("vLLM PagedAttention 深度解析" §7.2: a long
    prompt is cut into chunks that join the batch; each chunk's K/V go into the
    sequence's blocks and the chunk attends over everything cached so far) and
    speculative verification (§7.5; "LLM 推理引擎内部原理" §5.2: the target model
    checks the draft tokens, whose K/V sit in the same blocks).

    Reading (the pages describe the idea, not the indexing): the chunk's K/V
    are already in the cache, so context_lens[s] counts them; sequence s's
    queries are rows query_start[s] .. query_start[s+1]-1 of q ([T, Hq, D]);
    its i-th query sits at position context_lens[s] - n_s + i and sees the
    cache tokens 0 .. that position (itself included, none after it).
    Returns [T, Hq, D] fp64; rows of no sequence stay zero."""
    q = np.asarray(q)
    out = np.zeros(q.shape, dtype=np.float64)
    qs = [int(x) for x in np.asarray(query_start).tolist()]
    for s in range(len(qs) - 1):
        n = qs[s + 1] - qs[s]
        ctx = int(context_lens[s])
        if n == 0:
            continue
        if n > ctx:
            raise ValueError("a sequence has more queries than cached tokens")
        K = gather_logical(k_cache, block_tables[s], ctx, block_size)
        V = gather_logical(v_cache, block_tables[s], ctx, block_size)
        for i in range(n):
            visible = ctx - n + i + 1
            out[qs[s] + i] = attend(q[qs[s] + i], K[:visible], V[:visible], float(scale))
    return out

"""Seeded synthetic inputs for the paged decode path.

This module only draws random numbers and describes workload shapes. It holds
none of the method's arithmetic: no slot or block-table computation, no
attention, no cache addressing. Both the CUDA path's tests/bench and the CPU
oracle take their inputs from here, and each side then builds its own block
tables and slot mappings with its own block manager.

Workload shapes follow the pages' decode-serving workloads (7B/13B/70B-class
head shapes, block size 16 as the default block size in "为什么PagedAttention能让
大模型推理吞吐量提升数倍", section "Block Table：GPU上的页表", mixed context
lengths as produced by continuous batching, shared prompt prefixes as in
"vLLM PagedAttention 解析" §4.1 parallel sampling).

Random streams are keyed by (seed, stream, index) through numpy's SeedSequence,
so any one sequence's data can be regenerated alone (the oracle's sampled
checks and the CPU baseline use that) and generation can run in threads.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# stream identifiers for SeedSequence keys
_S_LENS, _S_PLACE, _S_Q, _S_PK, _S_PV, _S_NK, _S_NV = range(7)


@dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    kv_dtype: str                 # "f32", "bf16" or "fp8" (e4m3 cache codes; q, k, v in bf16)
    ctx: str                      # "fixed" | "uniform" | "loguniform" | "shared_prefix"
    lo: int = 0
    hi: int = 0
    fixed: tuple = ()
    shared_prefix: int = 0        # tokens of the shared prompt (shared_prefix workloads)
    partition_tokens: int = 0     # split-K partition the workload asks for (0 = library default)
    seed: int = 0
    kv_scale: float = 1.0         # per-tensor K and V scale of an fp8 cache
    description: str = field(default="", compare=False)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elt_bytes(self) -> int:
        """Bytes per cache element."""
        return {"f32": 4, "bf16": 2, "fp8": 1}[self.kv_dtype]

    @property
    def in_bytes(self) -> int:
        """Bytes per element of q and of the new K/V the step appends."""
        return 4 if self.kv_dtype == "f32" else 2

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "tiny_fp32": Workload(
        "tiny_fp32", 4, 8, 8, 64, 16, 64, "f32", "fixed", fixed=(7, 33, 100, 250), seed=1000,
        description="tiny fp32 MHA: 4 seqs, ctx {7,33,100,250}, 8 heads, D=64, bs=16, 64-block pool"),
    "llama2_7b": Workload(
        "llama2_7b", 64, 32, 32, 128, 16, 16384, "bf16", "uniform", lo=512, hi=2048, seed=1001,
        description="Llama-2-7B-shaped decode: B=64, 32/32 heads, D=128, bf16, bs=16, ctx U[512,2048], 16384-block pool"),
    "llama2_13b": Workload(
        "llama2_13b", 64, 40, 40, 128, 16, 16384, "bf16", "uniform", lo=512, hi=2048, seed=1005,
        description="Llama-2-13B-shaped decode: B=64, 40/40 heads, D=128, bf16, bs=16, ctx U[512,2048], "
                    "16384-block pool"),
    "gqa_70b": Workload(
        "gqa_70b", 128, 64, 8, 128, 16, 65536, "bf16", "uniform", lo=1024, hi=4096, seed=1002,
        description="70B-shaped GQA decode: B=128, 64/8 heads, D=128, bf16, bs=16, ctx U[1024,4096], 65536-block pool"),
    "shared_prefix": Workload(
        "shared_prefix", 32, 32, 32, 128, 16, 4096, "bf16", "shared_prefix", lo=64, hi=512,
        shared_prefix=1024, seed=1003,
        description="parallel sampling: 32 seqs share a 1024-token prefix (64 blocks, ref 32) + private tails U[64,512]; "
                    "32/32 heads, D=128, bf16, bs=16"),
    "llama2_7b_fp8": Workload(
        "llama2_7b_fp8", 64, 32, 32, 128, 16, 16384, "fp8", "uniform", lo=512, hi=2048, seed=1001, kv_scale=1 / 64,
        description="Llama-2-7B-shaped decode over an FP8 (e4m3, scale 1/64) cache: B=64, 32/32 heads, D=128, "
                    "bs=16, ctx U[512,2048], 16384-block pool"),
    "gqa_70b_fp8": Workload(
        "gqa_70b_fp8", 128, 64, 8, 128, 16, 65536, "fp8", "uniform", lo=1024, hi=4096, seed=1002, kv_scale=1 / 64,
        description="70B-shaped GQA decode over an FP8 (e4m3, scale 1/64) cache: B=128, 64/8 heads, D=128, bs=16, "
                    "ctx U[1024,4096], 65536-block pool"),
    "long_splitk": Workload(
        "long_splitk", 16, 32, 8, 128, 16, 65536, "bf16", "loguniform", lo=16, hi=32768,
        partition_tokens=512, seed=1004,
        description="long-context split-K: B=16, ctx log-uniform [16,32768], 32/8 heads, D=128, bf16, bs=16, "
                    "512-token partitions, 65536-block pool"),
}


def _rng(seed: int, stream: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream), int(index)]))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even. Inputs are finite."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (b >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(w: Workload, rng: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) samples stored in the workload's dtype; returned as float32 values
    exactly representable in that dtype (bf16-rounded for bf16 workloads)."""
    x = rng.standard_normal(shape, dtype=np.float32)
    if w.kv_dtype in ("bf16", "fp8"):
        x = bf16_bits_to_f32(round_to_bf16(x))
    return x


def context_lens(w: Workload) -> np.ndarray:
    """Context length of every sequence before the decode step (int64 [B]).

    For "shared_prefix" this is the shared prompt plus the private tail."""
    rng = _rng(w.seed, _S_LENS)
    if w.ctx == "fixed":
        return np.asarray(w.fixed, dtype=np.int64)
    if w.ctx == "uniform":
        return rng.integers(w.lo, w.hi + 1, size=w.num_seqs).astype(np.int64)
    if w.ctx == "loguniform":
        u = rng.uniform(math.log(w.lo), math.log(w.hi), size=w.num_seqs)
        return np.clip(np.rint(np.exp(u)), w.lo, w.hi).astype(np.int64)
    if w.ctx == "shared_prefix":
        tails = rng.integers(w.lo, w.hi + 1, size=w.num_seqs).astype(np.int64)
        return w.shared_prefix + tails
    raise ValueError(w.ctx)


def free_order(w: Workload) -> np.ndarray:
    """Initial order of the free-block list: a seeded permutation of the pool,
    so physical placement is random scatter (int32 [num_blocks])."""
    return _rng(w.seed, _S_PLACE).permutation(w.num_blocks).astype(np.int32)


def prompt_kv(w: Workload, s: int, ctx: int):
    """K and V of sequence s's first `ctx` tokens, [ctx, Hkv, D] float32 each.

    For "shared_prefix" the first `shared_prefix` tokens are the same for every
    sequence (index -1 stream) and only the tail is per-sequence."""
    shape_tail = (w.num_kv_heads, w.head_dim)
    if w.ctx == "shared_prefix":
        p = w.shared_prefix
        pk = _normal(w, _rng(w.seed, _S_PK, 1 << 20), (p,) + shape_tail)
        pv = _normal(w, _rng(w.seed, _S_PV, 1 << 20), (p,) + shape_tail)
        tk = _normal(w, _rng(w.seed, _S_PK, s), (ctx - p,) + shape_tail)
        tv = _normal(w, _rng(w.seed, _S_PV, s), (ctx - p,) + shape_tail)
        return np.concatenate([pk, tk]), np.concatenate([pv, tv])
    k = _normal(w, _rng(w.seed, _S_PK, s), (ctx,) + shape_tail)
    v = _normal(w, _rng(w.seed, _S_PV, s), (ctx,) + shape_tail)
    return k, v


def prompt_kv_all(w: Workload, lens: np.ndarray, threads: int = 8):
    """prompt_kv for every sequence, generated in threads (numpy releases the GIL)."""
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda s: prompt_kv(w, s, int(lens[s])), range(len(lens))))


def decode_q(w: Workload, step: int) -> np.ndarray:
    """Queries of decode step `step`: [B, Hq, D] float32."""
    return _normal(w, _rng(w.seed, _S_Q, step), (w.num_seqs, w.num_q_heads, w.head_dim))


def decode_kv(w: Workload, step: int):
    """K and V of the token each sequence appends at decode step `step`: [B, Hkv, D] each."""
    shape = (w.num_seqs, w.num_kv_heads, w.head_dim)
    return (_normal(w, _rng(w.seed, _S_NK, step), shape),
            _normal(w, _rng(w.seed, _S_NV, step), shape))


def sample_seqs(w: Workload, n: int, seed_offset: int = 0) -> np.ndarray:
    """A seeded sample of n sequence indices (for checks at full size)."""
    rng = _rng(w.seed + seed_offset, 99)
    return np.sort(rng.choice(w.num_seqs, size=min(n, w.num_seqs), replace=False))

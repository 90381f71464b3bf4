"""The C-ABI library on the CPU: it loads, exports every declared symbol, its
host block manager matches the oracle's bit for bit, and host-side argument
checks reject bad calls before anything reaches a GPU."""
import ctypes
import os
import random
import re

import numpy as np
import pytest

from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import binding, workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from paged_kv_cache_322_b200 import build
        build.build()
    return binding.library()


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pkv_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 17
    for n in sorted(names):
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert lib.pkv_status_string(code)
    assert lib.pkv_status_string(99) == b"unknown status"


def test_walkthrough_and_cow_match_the_pages(lib, golden_dir):
    import json
    g = json.load(open(os.path.join(golden_dir, "block_table_walkthrough.json")))
    bm = binding.BlockManager(g["num_blocks"], g["block_size"], g["free_order"])
    assert bm.allocate(7, g["prompt_tokens"]).tolist() == g["after_prefill"]["slots"]
    t, n = bm.block_tables([7], 4)
    assert t[0, :2].tolist() == g["after_prefill"]["table"] and n[0] == 7
    for step in g["decode"]:
        slots, src, dst = bm.append_slots([7])
        assert slots.tolist() == [step["slot"]] and src.size == 0
        t, _ = bm.block_tables([7], 4)
        assert t[0, :len(step["table"])].tolist() == step["table"]
        assert bm.num_free() == step["num_free"]
    c = json.load(open(os.path.join(golden_dir, "cow_fork.json")))
    bm = binding.BlockManager(c["num_blocks"], c["block_size"], c["free_order"])
    bm.allocate(1, c["prompt_tokens"])
    bm.fork(1, 2)
    slots, src, dst = bm.append_slots([1, 2])
    assert slots.tolist() == [c["A1_append"]["slot"], c["A2_append"]["slot"]]
    assert list(zip(src.tolist(), dst.tolist())) == [tuple(c["A1_append"]["copy"])]
    for b, r in c["ref_after"].items():
        assert bm.ref_count(int(b)) == r


def _run_both(ops, nb, bs, order):
    """Runs one op list on the oracle and on the library's block manager."""
    o = OracleBM(nb, bs, order)
    p = binding.BlockManager(nb, bs, order)
    for op in ops:
        kind = op[0]
        if kind == "alloc":
            r_o = o.allocate(op[1], op[2])
            try:
                r_p = p.allocate(op[1], op[2]).tolist()
            except binding.PkvError as e:
                assert e.status == 5
                r_p = None
            assert r_o == r_p
        elif kind == "fork":
            o.fork(op[1], op[2])
            p.fork(op[1], op[2])
        elif kind == "append":
            exp_slots, exp_pairs = [], []
            oom = False
            for s in op[1]:
                r = o.append_slot(s)
                if r is None:
                    oom = True
                    break
                exp_slots.append(r[0])
                if r[1] is not None:
                    exp_pairs.append(r[1])
            if oom:
                with pytest.raises(binding.PkvError):
                    p.append_slots(op[1])
                return o, p, False
            slots, src, dst = p.append_slots(op[1])
            assert slots.tolist() == exp_slots
            assert list(zip(src.tolist(), dst.tolist())) == exp_pairs
        elif kind == "cow":
            r_o = o.make_writable(op[1], op[2])
            assert p.make_writable(op[1], op[2]) == r_o
        elif kind == "free":
            o.free_seq(op[1])
            p.free(op[1])
        assert o.num_free() == p.num_free()
    return o, p, True


@pytest.mark.parametrize("seed", range(25))
def test_random_ops_bit_exact_vs_oracle(lib, seed):
    rng = random.Random(seed)
    bs = rng.choice([1, 4, 16])
    nb = 96
    order = rng.sample(range(nb), nb)
    ops, live, nxt = [], [], 0
    for _ in range(150):
        x = rng.random()
        if x < 0.2 or not live:
            ops.append(("alloc", nxt, rng.randint(0, 3 * bs)))
            live.append(nxt)
            nxt += 1
        elif x < 0.3:
            ops.append(("fork", rng.choice(live), nxt))
            live.append(nxt)
            nxt += 1
        elif x < 0.8:
            ops.append(("append", rng.sample(live, rng.randint(1, len(live)))))
        elif x < 0.9:
            ops.append(("free", live.pop(rng.randrange(len(live)))))
        else:
            ops.append(("cow", rng.choice(live), 0))
    # an allocation can fail (then the id does not exist): replay with the oracle first
    o = OracleBM(nb, bs, order)
    valid, alive = [], set()
    for op in ops:
        if op[0] == "alloc":
            if o.allocate(op[1], op[2]) is not None:
                alive.add(op[1])
            valid.append(op)
        elif op[0] == "fork":
            if op[1] in alive:
                o.fork(op[1], op[2])
                alive.add(op[2])
                valid.append(op)
        elif op[0] == "append":
            ids = [s for s in op[1] if s in alive]
            if ids:
                if any(o.append_slot(s) is None for s in ids):
                    valid.append(("append", ids))
                    break
                valid.append(("append", ids))
        elif op[0] == "free":
            if op[1] in alive:
                o.free_seq(op[1])
                alive.discard(op[1])
                valid.append(op)
        else:
            if op[1] in alive and o.tables[op[1]]:
                try:
                    o.make_writable(op[1], 0)
                except Exception:
                    break
                valid.append(op)
    _run_both(valid, nb, bs, order)


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_workload_prefill_and_steps_bit_exact(lib, name):
    w = wl.WORKLOADS[name]
    lens = wl.context_lens(w)
    order = wl.free_order(w)
    o = OracleBM(w.num_blocks, w.block_size, order)
    p = binding.BlockManager(w.num_blocks, w.block_size, order)
    if w.ctx == "shared_prefix":
        assert o.allocate(-1, w.shared_prefix) == p.allocate(-1, w.shared_prefix).tolist()
        for s in range(w.num_seqs):
            o.fork(-1, s)
            p.fork(-1, s)
        o.free_seq(-1)
        p.free(-1)
        for s in range(w.num_seqs):
            exp = [o.append_slot(s)[0] for _ in range(int(lens[s]) - w.shared_prefix)]
            got = []
            for _ in range(int(lens[s]) - w.shared_prefix):
                got.append(int(p.append_slots([s])[0][0]))
            assert exp == got
        last = w.shared_prefix // w.block_size - 1
        pairs_o = [o.make_writable(s, last) for s in range(w.num_seqs)]
        pairs_p = [p.make_writable(s, last) for s in range(w.num_seqs)]
        assert pairs_o == pairs_p and sum(x is not None for x in pairs_p) == w.num_seqs - 1
    else:
        for s in range(w.num_seqs):
            assert o.allocate(s, int(lens[s])) == p.allocate(s, int(lens[s])).tolist()
    ids = list(range(w.num_seqs))
    mb = -(-int(lens.max() + 3) // w.block_size)
    for _ in range(3):
        exp = [o.append_slot(s)[0] for s in ids]
        slots, src, dst = p.append_slots(ids)
        assert slots.tolist() == exp and src.size == 0
        tables, plens = p.block_tables(ids, mb)
        for s in ids:
            t = o.block_table(s)
            assert tables[s, :len(t)].tolist() == t and plens[s] == o.lens[s]


def test_block_manager_errors(lib):
    with pytest.raises(binding.PkvError):
        binding.BlockManager(4, 2, [0, 1, 1, 3])           # not a permutation
    bm = binding.BlockManager(2, 4)
    bm.allocate(0, 8)
    with pytest.raises(binding.PkvError) as e:
        bm.append_slots([0])
    assert e.value.status == 5
    with pytest.raises(binding.PkvError) as e:
        bm.allocate(0, 1)                                   # id exists
    assert e.value.status == 1
    with pytest.raises(binding.PkvError):
        bm.block_tables([0], 1)                             # table longer than the row
    with pytest.raises(binding.PkvError):
        bm.fork(5, 6)


def test_kernel_entry_points_reject_bad_arguments_on_host(lib):
    fake = ctypes.c_void_p(1 << 20)
    # head_dim 96 is not built; group 3 is not built; block size 12 is not built
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 96, 16, 4, 64,
                                          0, 0, None, 0, None) == 2
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 12, 4, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 2
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 128, 12, 4, 64,
                                          0, 0, None, 0, None) == 2
    # the persistent schedule serves 16-token blocks only
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 128, 32, 4, 64,
                                          0, -1, None, 0, None) == 2
    # Hq not a multiple of Hkv, negative sizes, bad dtype, NaN scale, misalignment
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 6, 4, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 1
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, -1, 8, 8, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 1
    assert lib.pkv_paged_attention_decode(fake, 7, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 1
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, float("nan"), 2, 8, 8, 128, 16,
                                          4, 64, 0, 0, None, 0, None) == 1
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.pkv_paged_attention_decode(odd, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 1
    # split-K needs a workspace: none given
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 8, 8, 128, 16, 128, 64,
                                          0, 512, None, 0, None) == 1
    # zero sequences / tokens / pairs: nothing to launch
    assert lib.pkv_paged_attention_decode(None, 0, None, None, None, 1, None, None, 1.0, 0, 8, 8, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 0
    assert lib.pkv_reshape_and_cache(None, None, None, None, 1, None, 0, 8, 128, 16, 64, None) == 0
    assert lib.pkv_copy_blocks(None, None, 1, None, None, 0, 16, 8, 128, 64, None) == 0
    assert lib.pkv_reshape_and_cache(fake, fake, fake, fake, 5, fake, 4, 8, 128, 16, 64, None) == 1
    assert lib.pkv_reshape_and_cache(fake, fake, fake, fake, 1, fake, 4, 1, 4, 16, 64, None) == 2  # 8-byte rows
    assert lib.pkv_copy_blocks(fake, fake, 1, fake, fake, -1, 16, 8, 128, 64, None) == 1


def test_fp8_multi_query_and_noalloc_entry_points_reject_bad_arguments_on_host(lib):
    """Every refusal below happens in host code before any device call, so it
    runs without a GPU: status 1 = invalid argument, 2 = not built."""
    fake = ctypes.c_void_p(1 << 20)
    nan, inf = float("nan"), float("inf")

    def dec8(ks, vs, d=128, part=0):
        return lib.pkv_paged_attention_decode_fp8(fake, 0, fake, fake, fake, ks, vs, fake, fake, 1.0, 2, 8, 8, d, 16,
                                                  4, 64, 0, part, None, 0, None)
    assert dec8(0.0, 1.0) == 1 and dec8(1.0, -1.0) == 1 and dec8(nan, 1.0) == 1 and dec8(1.0, inf) == 1
    assert dec8(1.0, 1.0, d=64) == 2                 # e4m3 attention is built for head_dim 128
    assert dec8(1.0, 1.0, part=-1) == 2              # no persistent schedule over e4m3 caches
    # the plain decode call takes fp32 / bf16 caches only; e4m3 goes through the fp8 entry point
    assert lib.pkv_paged_attention_decode(fake, 0, fake, fake, fake, 2, fake, fake, 1.0, 2, 8, 8, 128, 16, 4, 64,
                                          0, 0, None, 0, None) == 1

    def app8(in_dtype=1, ks=1.0, hkv=8, d=128, t=4):
        return lib.pkv_reshape_and_cache_fp8(fake, fake, in_dtype, fake, fake, ks, 1.0, fake, t, hkv, d, 16, 64, None)
    assert app8(in_dtype=2) == 1 and app8(ks=0.0) == 1 and app8(ks=nan) == 1
    assert app8(hkv=1, d=8) == 2                     # 8-element rows: not a whole 16-byte vector of codes
    assert lib.pkv_reshape_and_cache_fp8(None, None, 1, None, None, 1.0, 1.0, None, 0, 8, 128, 16, 64, None) == 0

    def mq(kv=1, hq=8, hkv=8, d=128, bs=16, mb=4, nq=4, ctx=64, part=0, seqs=2, tokens=8, ws=None, ws_n=0):
        return lib.pkv_paged_attention_multi_query(fake, 0, fake, fake, fake, kv, fake, fake, fake, 1.0, seqs, tokens,
                                                   hq, hkv, d, bs, mb, 64, nq, ctx, part, ws, ws_n, None)
    assert mq(kv=0) == 2 and mq(kv=2) == 2          # bf16 caches only
    assert mq(kv=7) == 1
    assert mq(d=96) == 2 and mq(bs=12) == 2 and mq(hq=12, hkv=4) == 2      # head_dim, block size, group 3
    assert mq(hq=6, hkv=4) == 1 and mq(part=-1) == 1
    assert mq(nq=100) == 1                           # more query tokens than the table holds
    assert mq(part=16) == 1                          # four partitions need a workspace; none given
    assert mq(seqs=0) == 0 and mq(nq=0) == 0 and mq(tokens=0) == 0
    assert lib.pkv_paged_attention_multi_query_workspace_bytes(2, 8, 8, 8, 128, 16, 4, 4, 64, 16) > 0
    assert lib.pkv_paged_attention_multi_query_workspace_bytes(2, 8, 8, 8, 128, 16, 4, 4, 64, 64) == 0
    assert lib.pkv_paged_attention_multi_query_workspace_bytes(2, 8, 8, 8, 128, 16, 4, 100, 64, 0) == \
        ctypes.c_size_t(-1).value

    # allocation-free decode: sizes whose split-K scratch exceeds the fixed array, and invalid sizes
    assert lib.pkv_paged_attention_decode_noalloc(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 1024, 64, 8, 128,
                                                  16, 2048, 65536, 32768, 512, None) == 2
    assert lib.pkv_paged_attention_decode_noalloc(fake, 0, fake, fake, fake, 1, fake, fake, 1.0, 2, 6, 4, 128,
                                                  16, 4, 64, 0, 0, None) == 1


def test_native_step_refuses_bad_arguments_on_host(lib):
    """pkv_step_ctx_create and pkv_decode_step refuse invalid sizes, dtypes and
    scales before touching the device; destroying a null context is a no-op."""
    h = ctypes.c_void_p()

    def create(seqs=4, hq=8, hkv=8, d=128, mb=4, bs=16, kv=1, out=0, ks=1.0, vs=1.0):
        return lib.pkv_step_ctx_create(seqs, hq, hkv, d, mb, bs, kv, out, 0, ks, vs, ctypes.byref(h))
    assert create(seqs=0) == 1 and create(hq=6, hkv=4) == 1 and create(d=0) == 1 and create(mb=0) == 1
    assert create(bs=0) == 1 and create(kv=5) == 1 and create(out=2) == 1      # e4m3 is not an output type
    assert create(kv=2, ks=0.0) == 1 and create(kv=2, vs=-1.0) == 1         # e4m3 caches need positive scales
    assert lib.pkv_step_ctx_create(4, 8, 8, 128, 4, 16, 1, 0, 0, 1.0, 1.0, None) == 1
    lib.pkv_step_ctx_destroy(None)
    bm = binding.BlockManager(8, 16)
    ids = np.zeros(1, np.int64)
    fake = ctypes.c_void_p(1 << 20)
    assert lib.pkv_decode_step(None, bm._h, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 1, fake, fake, fake,
                               fake, fake, 8, 1.0, 0, fake, None) == 1


def test_workspace_and_partition_rule(lib):
    # 512-token partitions over a 32768-token cap: 64 partitions of (D + 2) floats per row
    n = binding.workspace_bytes(16, 32, 8, 128, 16, 2048, 32768, 512)
    rows = 16 * 32 * 64
    assert n >= rows * 128 * 4 + rows * 2 * 4
    # one partition: only the longest-first unit list (B units of 8 bytes + a count, 256-byte rounded)
    assert binding.workspace_bytes(4, 8, 8, 64, 16, 16, 256, 512) == 256
    assert binding.workspace_bytes(1, 8, 8, 64, 16, 16, 256, 512) == 0      # one sequence: nothing to order
    assert binding.partition_tokens(16, 32, 8, 128, 16, 2048, 32768, 500) == 512
    # -1 = the persistent, evenly split schedule: per-CTA pieces + one counter per (sequence, KV head)
    assert binding.partition_tokens(64, 32, 32, 128, 16, 128, 2048, -1) == 0
    n = binding.workspace_bytes(64, 32, 32, 128, 16, 128, 2048, -1)
    assert n >= 64 * 32 * 8 and n < 32 * 2 ** 20
    with pytest.raises(binding.PkvError):
        binding.workspace_bytes(4096, 32, 8, 128, 16, 64, 1024, -1)   # more than 2048 sequences
    # 0 = library-chosen partitions: the fewest that fill about one wave (3 CTAs x 148 SMs = 444
    # units), a sequence's partitions estimated at 16 lengths spread over [cap / 2, cap]
    p7 = binding.partition_tokens(64, 32, 32, 128, 16, 256, 2158, 0)                # 7B-shaped batch
    assert p7 >= 2158 and p7 % 16 == 0                                                # one partition, no merge
    assert binding.workspace_bytes(64, 32, 32, 128, 16, 256, 2158, 0) == 768    # the unit list only
    p70 = binding.partition_tokens(128, 64, 8, 128, 16, 512, 4100, 0)               # 70B-shaped batch: 1024 units
    assert p70 >= 4100
    assert binding.workspace_bytes(128, 64, 8, 128, 16, 512, 4100, 0) == 1280   # 128 units + count
    p32 = binding.partition_tokens(32, 64, 8, 128, 16, 512, 4100, 0)                # 256 units per partition
    assert -(-4100 // p32) == 2 and p32 == 2064                                       # two: 512 units
    # one sequence at its full length: 8 heads x 56 partitions = 448 units >= 444 (55 give 440)
    assert binding.partition_tokens(1, 32, 8, 128, 16, 2048, 32768, 0) == 592
    assert binding.partition_tokens(1, 32, 8, 128, 16, 2048, 300, 0) == 304        # short: one partition
    assert binding.partition_tokens(1, 32, 8, 128, 16, 2048, 600, 0) == 304        # two even ones, not 256+256+88
    assert binding.partition_tokens(1, 32, 8, 128, 16, 2048, 100, 0) == 256        # below the floor: one


@pytest.mark.parametrize("seed", range(12))
def test_swap_ops_bit_exact_vs_oracle(lib, seed):
    """Random allocate / append / fork / free / swap-out / swap-in through the
    C++ block manager and the oracle: the same block pairs, tables, counts and
    free lists on both pools, and the same all-or-nothing refusals."""
    rng = random.Random(100 + seed)
    bs = rng.choice([1, 4, 16])
    nb, nh = 48, 40
    order = rng.sample(range(nb), nb)
    horder = rng.sample(range(nh), nh)
    o = OracleBM(nb, bs, order, num_cpu_blocks=nh, cpu_free_order=horder)
    p = binding.BlockManager(nb, bs, order)
    p.set_host_pool(nh, horder)
    alive, nxt = [], 0
    for _ in range(200):
        x = rng.random()
        resident = [s for s in alive if s not in o.swapped]
        out = [s for s in alive if s in o.swapped]
        if x < 0.2 or not alive:
            n = rng.randint(0, 3 * bs)
            r = o.allocate(nxt, n)
            if r is None:
                with pytest.raises(binding.PkvError):
                    p.allocate(nxt, n)
            else:
                assert p.allocate(nxt, n).tolist() == r
                alive.append(nxt)
            nxt += 1
        elif x < 0.3 and resident:
            s = rng.choice(resident)
            o.fork(s, nxt)
            p.fork(s, nxt)
            alive.append(nxt)
            nxt += 1
        elif x < 0.5 and resident:
            s = rng.choice(resident)
            r = o.append_slot(s)
            if r is None:
                with pytest.raises(binding.PkvError):
                    p.append_slots([s])
                break
            slots, src, dst = p.append_slots([s])
            assert slots.tolist() == [r[0]]
            assert list(zip(src.tolist(), dst.tolist())) == ([r[1]] if r[1] else [])
        elif x < 0.6 and alive:
            s = alive.pop(rng.randrange(len(alive)))
            o.free_seq(s)
            p.free(s)
        elif x < 0.8 and resident:
            group = rng.sample(resident, rng.randint(1, min(3, len(resident))))
            r = o.swap_out(group)
            if r is None:
                with pytest.raises(binding.PkvError) as e:
                    p.swap_out(group)
                assert e.value.status == 5
            else:
                a, b = p.swap_out(group)
                assert list(zip(a.tolist(), b.tolist())) == r
        elif out:
            group = rng.sample(out, rng.randint(1, min(3, len(out))))
            r = o.swap_in(group)
            if r is None:
                with pytest.raises(binding.PkvError) as e:
                    p.swap_in(group)
                assert e.value.status == 5
            else:
                a, b = p.swap_in(group)
                assert list(zip(a.tolist(), b.tolist())) == r
        assert o.num_free() == p.num_free() and len(o.cpu_free) == p.num_free_host()
        for s in alive:
            assert p.is_swapped(s) == (s in o.swapped)
            if s not in o.swapped:
                t = o.block_table(s)
                tables, lens = p.block_tables([s], max(len(t), 1))
                assert tables[0, :len(t)].tolist() == t and lens[0] == o.lens[s]
        assert [p.ref_count(b) for b in range(nb)] == o.ref
        assert [p.host_ref_count(b) for b in range(nh)] == o.cpu_ref


def test_swap_errors(lib):
    bm = binding.BlockManager(8, 4)
    bm.allocate(0, 5)
    with pytest.raises(binding.PkvError):
        bm.swap_out([0])                                    # no host pool: 0 free host blocks
    bm.set_host_pool(4)
    with pytest.raises(binding.PkvError):
        bm.set_host_pool(4)                                 # set once
    a, b = bm.swap_out([0])
    assert a.size == 2 and bm.is_swapped(0) and bm.num_free() == 8 and bm.num_free_host() == 2
    for call in (lambda: bm.append_slots([0]), lambda: bm.fork(0, 1), lambda: bm.make_writable(0, 0),
                 lambda: bm.block_tables([0], 4), lambda: bm.swap_out([0])):
        with pytest.raises(binding.PkvError) as e:
            call()
        assert e.value.status == 1
    with pytest.raises(binding.PkvError):
        bm.swap_in([0, 0])                                  # repeated id
    bm.free(0)
    assert bm.num_free_host() == 4
    with pytest.raises(KeyError):
        bm.is_swapped(0)
    # host-side checks of the copy entry point
    fake = ctypes.c_void_p(1 << 20)
    assert lib.pkv_swap_blocks(None, None, 1, None, None, 1, 1, None, None, 0, 16, 8, 128, None) == 0
    assert lib.pkv_swap_blocks(fake, fake, 4, fake, fake, 4, 9, fake, fake, 1, 16, 8, 128, None) == 1
    assert lib.pkv_swap_blocks(fake, fake, 0, fake, fake, 4, 1, fake, fake, 1, 16, 8, 128, None) == 1
    assert lib.pkv_swap_blocks(fake, fake, 4, fake, fake, 4, 1, fake, fake, -1, 16, 8, 128, None) == 1
    assert lib.pkv_swap_blocks(fake, fake, 4, fake, fake, 4, 2, fake, fake, 1, 1, 1, 8, None) == 2  # 8-byte block


def test_binding_requires_one_current_device(monkeypatch):
    """The binding refuses tensors that are not CUDA, not contiguous, on two
    devices, or on a device other than the current one (the library launches on
    the current device). Stand-in tensor objects: no GPU needed."""
    import torch

    class T:
        def __init__(self, idx, cuda=True, contig=True):
            self.device, self.is_cuda, self._contig = torch.device("cuda", idx), cuda, contig

        def is_contiguous(self):
            return self._contig

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    binding._cuda_contig(T(1), T(1), T(1))
    with pytest.raises(ValueError, match="one device"):
        binding._cuda_contig(T(1), T(0))
    with pytest.raises(ValueError, match="current device"):
        binding._cuda_contig(T(0), T(0))
    with pytest.raises(ValueError, match="CUDA tensors"):
        binding._cuda_contig(T(1), T(1, cuda=False))
    with pytest.raises(ValueError, match="contiguous"):
        binding._cuda_contig(T(1, contig=False))


def test_wait_hook_checks_its_arguments_on_host(lib):
    """pkv_test_withhold_copy (test hook for the bounded waits): known kernel ids
    only, a limit in [100 us, 2 s] when arming, -1 disarms without a limit."""
    f = lib.pkv_test_withhold_copy
    assert f(2, 0, 5_000_000) == 1
    assert f(-1, 0, 5_000_000) == 1
    assert f(0, 3, 10) == 1                      # limit too short
    assert f(1, 3, 3_000_000_000) == 1           # longer than the default limit
    assert f(0, -2, 5_000_000) == 1
    assert f(0, 3, 5_000_000) == 0               # armed ...
    assert f(0, -1, 0) == 0                      # ... and disarmed
    assert f(1, -1, 0) == 0


def test_step_timing_checks_its_arguments_on_host(lib):
    buf = (ctypes.c_float * 4)()
    assert lib.pkv_step_ctx_set_timing(None, 1) == 1
    assert lib.pkv_step_ctx_last_timing(None, buf) == 1


def test_shared_prefix_host_refusals(lib):
    """The shared-prefix decode refuses, before any launch: shapes it does not
    build (head_dim 64; fewer than 32 query rows per KV head for its tcgen05 prefix
    call), a prefix that is not whole blocks or reaches the longest context, and
    a workspace below its size."""
    fake = ctypes.c_void_p(1 << 20)
    ws_need = lib.pkv_paged_attention_shared_prefix_workspace_bytes(32, 32, 32, 128, 1008)
    rows = 32 * 32                                 # (sequence, query head) rows: one prefix partial at least
    assert ws_need >= rows * (128 * 4 + 2 * 4) + 32 * 8 + 4 + 3 * 4
    # at most one prefix partial per 128-token tile: 1008 tokens -> 8 tiles; four 256-byte aligned regions
    assert ws_need <= 8 * rows * (128 * 4 + 2 * 4) + 32 * 8 + 4 + 3 * 4 + 4 * 256
    bad = ctypes.c_size_t(-1).value
    assert lib.pkv_paged_attention_shared_prefix_workspace_bytes(0, 32, 32, 128, 1008) == bad
    assert lib.pkv_paged_attention_shared_prefix_workspace_bytes(32, 32, 5, 128, 1008) == bad
    assert lib.pkv_paged_attention_shared_prefix_workspace_bytes(32, 32, 32, 128, 0) == bad

    def call(B=32, hq=32, hkv=32, d=128, bs=16, prefix=1008, maxlen=1500, ws_n=None):
        return lib.pkv_paged_attention_decode_shared_prefix(
            fake, 1, fake, fake, fake, fake, fake, prefix, 0.088, B, hq, hkv, d, bs, 128, 4096, maxlen, fake,
            ws_need if ws_n is None else ws_n, None)

    assert call(d=64) == 2                         # PKV_ERR_UNSUPPORTED
    assert call(B=16) == 2                         # 16 rows per KV head
    assert call(B=8, hq=64, hkv=8, ws_n=0) == 1    # 64 rows per KV head: past the shape checks
    assert call(prefix=1000) == 1                  # PKV_ERR_INVALID_ARG: not whole blocks
    assert call(prefix=1504, maxlen=1500) == 1     # the prefix reaches the longest context
    assert call(ws_n=ws_need - 1) == 1             # workspace too small


def test_shared_prefix_workspace_follows_the_prefix_partition_rule(lib):
    """The shared-prefix workspace holds one normalised partial per (sequence,
    query head, prefix partition) plus the tails' unit list and the prefix
    call's descriptors, each region 256-byte aligned. Prefix partitions: at most
    one wave of the prefix call's CTAs (KV heads x 128-row tiles x partitions,
    one CTA per SM; without a GPU the library assumes 148 SMs), at most one per
    128-token tile of the prefix, at least one."""
    def r256(x):
        return (x + 255) // 256 * 256

    for B, hq, hkv, prefix in [(32, 32, 32, 1008), (8, 64, 8, 4000), (200, 8, 8, 64), (4, 128, 8, 16),
                               (64, 32, 4, 8192), (33, 33, 1, 128)]:
        group = hq // hkv
        row_tiles = -(-B * group // 128)
        parts = max(1, min(max(1, 148 // (hkv * row_tiles)), -(-prefix // 128)))
        rows = B * hq * parts
        want = r256(rows * 128 * 4) + r256(rows * 2 * 4) + r256(B * 8 + 4) + r256(12)
        assert lib.pkv_paged_attention_shared_prefix_workspace_bytes(B, hq, hkv, 128, prefix) == want, (B, hq, hkv)

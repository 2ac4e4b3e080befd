"""The C++ block allocator (through the C ABI) against the pages' demo run and
against the oracle allocator on random operation sequences (bit-exact)."""
import ctypes
import random

import numpy as np

import pytest

import paged_kv_cache_453_b200 as P
import workloads as W
from oracle.allocator import BlockAllocator as OracleAlloc, AllocError
from test_oracle_allocator import run_demo


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_453_b200.build import build
    build()


def test_demo_run_matches_pages():
    run_demo(lambda n, B: P.BlockAllocator(n, B), lambda a, s: a.table(s), lambda a: a.num_free(),
             lambda a, s, n: a.allocate(s, n), lambda a, s, d: a.fork(s, d),
             lambda a, s: a.append_slot(s), lambda a, s: a.free(s))


def _same(a: P.BlockAllocator, o: OracleAlloc, seqs):
    for s in seqs:
        assert a.table(s) == o.table(s)
        assert a.num_tokens(s) == o.num_tokens[s]
    assert [a.refcount(b) for b in range(o.num_blocks)] == o.refcount
    st = a.stats()
    ost = o.stats()
    assert (st["free"], st["used"], st["shared"], st["tokens"]) == (
        ost["free"], ost["used"], ost["shared"], ost["tokens"])


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_random_ops_match_oracle(seed):
    rng = random.Random(seed)
    N, B = 48, rng.choice([2, 4, 16])
    order = rng.sample(range(N), N)
    a = P.BlockAllocator(N, B, order)
    o = OracleAlloc(N, B, order)
    live, nxt, out = [], 0, []
    for step in range(2000):
        op = rng.random()
        if op < 0.2 or not live:
            args, name = (nxt, rng.randint(0, 3 * B)), "allocate"
        elif op < 0.3:
            args, name = (rng.choice(live), nxt), "fork"
        elif op < 0.4:
            args, name = (rng.choice(live),), "free"
        elif op < 0.43:
            args, name = (10_000 + rng.randint(0, 5),), "append_slot"   # unknown sequence
        elif op < 0.47:
            args, name = (rng.choice(live),), "swap_out"
        elif op < 0.51:
            # a swapped-out sequence mostly, sometimes a live one (an error)
            args, name = (rng.choice(out) if out and rng.random() < 0.8 else rng.choice(live),), "swap_in"
        elif op < 0.52 and out:
            args, name = (rng.choice(out),), "append_slot"              # swapped out: unknown
        else:
            args, name = (rng.choice(live),), "append_slot"
        err_o = err_a = None
        try:
            ro = getattr(o, name)(*args)
        except AllocError as e:
            err_o = e.code
        try:
            ra = getattr(a, name)(*args)
        except P.PkvError as e:
            err_a = e.status
        assert err_o == err_a, (step, name, args, err_o, err_a)
        if err_o is None:
            if name in ("append_slot", "swap_out", "swap_in"):
                assert ra == ro
            if name in ("allocate", "fork"):
                live.append(nxt)
                nxt += 1
            if name == "free":
                live.remove(args[0])
            if name == "swap_out":
                live.remove(args[0])
                out.append(args[0])
            if name == "swap_in":
                out.remove(args[0])
                live.append(args[0])
        _same(a, o, live)


def test_build_block_tables_pads_and_checks():
    a = P.BlockAllocator(16, 4)
    a.allocate(7, 9)
    a.allocate(8, 0)
    table, lens = a.build_block_tables([8, 7], 4)
    assert table.tolist() == [[-1, -1, -1, -1], [0, 1, 2, -1]]
    assert lens.tolist() == [0, 9]
    with pytest.raises(P.PkvError) as e:
        a.build_block_tables([7], 2)           # 3 blocks do not fit in 2
    assert e.value.status == P.PKV_ERR_INVALID_ARG
    with pytest.raises(P.PkvError) as e:
        a.build_block_tables([9], 4)
    assert e.value.status == P.PKV_ERR_UNKNOWN_SEQ


def test_prefix_script_same_as_oracle():
    s = W.spec("prefix_13b")
    sc = W.prefix_script(s)
    a = P.BlockAllocator(sc.num_blocks, s.block_size, sc.free_order)
    o = OracleAlloc(sc.num_blocks, s.block_size, sc.free_order)
    a.run(sc.setup)
    o.run(sc.setup)
    steps_a = [a.append_slot(r) for r in sc.step_appends]
    steps_o = [o.append_slot(r) for r in sc.step_appends]
    assert steps_a == steps_o
    _same(a, o, sc.seqs)


def test_errors_are_atomic():
    a = P.BlockAllocator(2, 4)
    a.allocate(1, 6)
    a.fork(1, 2)
    with pytest.raises(P.PkvError) as e:
        a.append_slot(1)          # copy-on-write needs a free block
    assert e.value.status == P.PKV_ERR_OOM
    assert a.table(1) == [0, 1] and a.num_tokens(1) == 6 and a.refcount(1) == 2
    with pytest.raises(P.PkvError) as e:
        P.BlockAllocator(3, 4, [0, 0, 1])
    assert e.value.status == P.PKV_ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# pkv_prefix_groups against the oracle's definition (bit-exact)
# ---------------------------------------------------------------------------

def _fork_tree_layout(seed, B=4):
    rng = np.random.default_rng(seed)
    a = OracleAlloc(600, B)
    seqs = []
    for i in range(int(rng.integers(1, 6))):
        a.allocate(i, int(rng.integers(0, 30)))
        seqs.append(i)
    nxt = len(seqs)
    for _ in range(40):
        op = rng.integers(4)
        if op == 0:
            a.fork(int(rng.choice(seqs)), nxt)
            seqs.append(nxt)
            nxt += 1
        else:
            r = int(rng.choice(seqs))
            for _ in range(int(rng.integers(1, 9))):
                a.append_slot(r)
    rng.shuffle(seqs)
    rows = [a.table(r) for r in seqs]
    width = max(1, max(len(r) for r in rows))
    t = np.full((len(rows), width), -1, dtype=np.int32)
    for i, r in enumerate(rows):
        t[i, :len(r)] = r
    return t, np.array([a.num_tokens[r] for r in seqs], dtype=np.int32)


@pytest.mark.parametrize("seed", range(20))
def test_prefix_groups_match_oracle(seed):
    import torch
    from oracle.prefix import prefix_groups as oracle_groups
    tables, lens = _fork_tree_layout(seed)
    for mm in (1, 2, 3):
        gs, mem, pb = P.prefix_groups(torch.from_numpy(tables), torch.from_numpy(lens), 4, mm)
        ogs, omem, opb = oracle_groups(tables, lens, 4, mm)
        assert gs.tolist() == ogs and mem.tolist() == omem and pb.tolist() == opb, (seed, mm)


def test_prefix_groups_rejects_bad_arguments():
    import torch
    t = torch.zeros((2, 2), dtype=torch.int32)
    ln = torch.full((2,), 8, dtype=torch.int32)
    with pytest.raises(P.PkvError):
        P.prefix_groups(t, ln, 0)
    with pytest.raises(P.PkvError):
        P.prefix_groups(t, ln, 4, 0)
    gs, mem, pb = P.prefix_groups(t[:0], ln[:0], 4)
    assert gs.tolist() == [0] and mem.tolist() == [] and pb.tolist() == []


# ---------------------------------------------------------------------------
# Prefix cache, prefix allocation and utilisation against the oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [4, 5, 6])
def test_prefix_cache_random_ops_match_oracle(seed):
    from oracle.radix import PrefixCache as OracleCache, allocate_prefix
    rng = random.Random(seed)
    N, B = 200, rng.choice([1, 2, 4])
    a = P.BlockAllocator(N, B)
    o = OracleAlloc(N, B)
    ca, co = P.PrefixCache(a), OracleCache(o)
    prompts = [[rng.randint(0, 2) for _ in range(rng.randint(0, 6 * B))] for _ in range(4)]
    live, toks, nxt = [], {}, 0
    for step in range(600):
        r = rng.random()
        if r < 0.25 or not live:
            # a new request: a prompt plus a suffix, reusing what the cache holds
            t = rng.choice(prompts) + [rng.randint(0, 2) for _ in range(rng.randint(0, 3 * B))]
            ma, mo = ca.match(t), co.match(t)
            assert ma == mo, step
            err_a = err_o = None
            try:
                a.allocate_prefix(nxt, ma, len(t))
            except P.PkvError as e:
                err_a = e.status
            try:
                allocate_prefix(o, nxt, mo, len(t))
            except AllocError as e:
                err_o = e.code
            assert err_a == err_o
            if err_a is None:
                live.append(nxt)
                toks[nxt] = t
            nxt += 1
        elif r < 0.45:
            s = rng.choice(live)
            assert ca.insert(s, toks[s]) == co.insert(s, toks[s])
        elif r < 0.6:
            s = rng.choice(live)
            a.free(s)
            o.free(s)
            live.remove(s)
        elif r < 0.7:
            n = rng.randint(0, 4)
            assert ca.evict(n) == co.evict(n)
        else:
            s = rng.choice(live)
            err_a = err_o = None
            try:
                ra = a.append_slot(s)
            except P.PkvError as e:
                err_a = e.status
            try:
                ro = o.append_slot(s)
            except AllocError as e:
                err_o = e.code
            assert err_a == err_o
            if err_a is None:
                assert ra == ro
                toks[s].append(rng.randint(0, 2))
        assert ca.nodes == co.nodes
        _same(a, o, live)
        u, ost = a.utilisation(), o.stats()
        assert u["blocks_without_sharing"] == ost["table_blocks"] and u["sequences"] == ost["sequences"]
    ca.close()


def test_cache_outliving_its_allocator_is_detached():
    a = P.BlockAllocator(8, 2)
    c = P.PrefixCache(a)
    a.allocate(1, 4)
    assert c.insert(1, [1, 2, 3, 4]) == 2
    lib = P.lib()
    lib.pkv_alloc_destroy(a._h)          # the allocator goes first
    a._h = None
    buf, n = (ctypes.c_int32 * 2)(), ctypes.c_int32()
    assert lib.pkv_cache_evict(c._h, 2, buf, ctypes.byref(n)) == P.PKV_ERR_INVALID_ARG
    c.close()                            # safe: nothing left to release

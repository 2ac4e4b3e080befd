"""Prefix-aware decode (paged_attn_decode_cascade) against the fp64 oracle.

The cascade computes the attention paged_attn_decode defines; the oracle is
the same paged_decode (each sequence's K/V gathered through its own table), so
a grouping, chunking or merge mistake shows up as an error against it.
Layouts come from allocator runs (shared prompt, forks, private suffixes,
copy-on-write of a partly filled shared block).
"""
import dataclasses

import numpy as np
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, max_err, oracle_decode, run_decode, check_no_device_error
from oracle.allocator import BlockAllocator

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()


def _layout(spec, groups, solo, seed):
    """groups: [(prefix tokens, [suffix tokens per member])]; solo: [tokens].
    Returns a Layout whose rows are all members then the solo rows, shuffled."""
    rng = np.random.default_rng(seed)
    B = spec.block_size
    need = sum(-(-P // B) + sum(-(-x // B) + 1 for x in sfx) for P, sfx in groups)
    need += sum(-(-x // B) for x in solo)
    nblk = int(need * 1.1) + 8
    a = BlockAllocator(nblk, B, [int(x) for x in rng.permutation(nblk)])
    rows, nxt = [], 0
    for P, sfx in groups:
        holder = 10 ** 6 + nxt
        a.allocate(holder, P)
        for x in sfx:
            a.fork(holder, nxt)
            for _ in range(x):
                a.append_slot(nxt)
            rows.append(nxt)
            nxt += 1
        a.free(holder)
    for x in solo:
        a.allocate(nxt, x)
        rows.append(nxt)
        nxt += 1
    rows = [rows[i] for i in rng.permutation(len(rows))]
    lens = torch.tensor([a.num_tokens[r] for r in rows], dtype=torch.int32)
    width = max(1, max(len(a.table(r)) for r in rows))
    tables = torch.full((len(rows), width), -1, dtype=torch.int32)
    for i, r in enumerate(rows):
        tables[i, :len(a.table(r))] = torch.tensor(a.table(r), dtype=torch.int32)
    s = spec.replace(num_seqs=len(rows), append=False, pool_blocks=nblk)
    return s, W.Layout(s, nblk, lens, tables, lens.clone(), tables.clone())


def _run_cascade(s, lay, t, min_members=2):
    groups = P.PrefixGroups(lay.tables, lay.lens, s.block_size, min_members)
    out = torch.full_like(t.q, float("nan"))
    P.paged_attn_decode_cascade(t.q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), groups,
                                s.num_kv_heads, s.scale, s.block_size, out,
                                k_scale=t.k_scale, v_scale=t.v_scale)
    return out, groups


def _spec(cd, Hq, Hk, D, B):
    return W.spec("llama3_8b").replace(num_q_heads=Hq, num_kv_heads=Hk, head_dim=D, block_size=B,
                                       cache_dtype=cd, q_dtype=cd, table_width=None)


CASES = {
    # dtype, Hq, Hk, D, B, groups, solo
    "mha_f16_b16": ("f16", 4, 4, 128, 16, [(100, [5, 0, 17, 31, 16]), (48, [1, 2])], [7, 40]),
    "gqa_bf16_b16": ("bf16", 32, 8, 128, 16, [(300, [10, 20, 0, 64])], [500, 1]),
    "g8_bf16_b32": ("bf16", 64, 8, 128, 32, [(257, [3, 40, 96]), (64, [0, 0, 33])], [90]),
    "d64_f16_b32": ("f16", 8, 2, 64, 32, [(96, [1, 63, 64, 65])], [0, 31]),
    "many_members": ("f16", 2, 2, 128, 16, [(64, list(range(0, 140, 2)))], []),  # 70 members: 3 column chunks
    "long_prefix": ("bf16", 16, 4, 128, 16, [(3000, [9, 100, 250])], [1000]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_cascade_matches_oracle(name):
    cd, Hq, Hk, D, B, groups, solo = CASES[name]
    s, lay = _layout(_spec(cd, Hq, Hk, D, B), groups, solo, seed=sum(map(ord, name)))
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda", seed=7)
    out, gr = _run_cascade(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert gr.num_groups == len(groups)
    ref = oracle_decode(s, lay, t)
    assert max_err(out, ref) <= TOL[cd], name
    plain = run_decode(s, lay, t)
    torch.cuda.synchronize()
    assert max_err(plain, ref) <= TOL[cd]


def test_cascade_prefix_workload_full_size():
    # 50 requests behind one 800-token prompt, after the copy-on-write step,
    # laid out by the library's allocator; every row compared.
    s = W.spec("prefix_13b")
    sc = W.prefix_script(s)
    a = P.BlockAllocator(sc.num_blocks, s.block_size, sc.free_order)
    a.run(sc.setup)
    for r in sc.step_appends:
        a.append_slot(r)
    width = -(-max(sc.final_lens) // s.block_size)
    tables, lens = a.build_block_tables(sc.seqs, width)
    s = s.replace(append=False)
    lay = W.Layout(s, sc.num_blocks, lens, tables, lens.clone(), tables.clone())
    t = W.make_tensors(s, lay.num_blocks, tables, lens, device="cuda")
    out, gr = _run_cascade(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert gr.num_groups == 1 and gr.max_group_size == 50 and gr.max_prefix_blocks == 50
    ref = oracle_decode(s, lay, t)
    assert max_err(out, ref) <= TOL["f16"]


def test_cascade_repeated_calls_and_shapes():
    # consecutive calls of different shapes reuse the library's buffers
    outs = []
    for name in ("gqa_bf16_b16", "many_members", "gqa_bf16_b16"):
        cd, Hq, Hk, D, B, groups, solo = CASES[name]
        s, lay = _layout(_spec(cd, Hq, Hk, D, B), groups, solo, seed=3)
        t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda", seed=11)
        out, _ = _run_cascade(s, lay, t)
        torch.cuda.synchronize()
        assert max_err(out, oracle_decode(s, lay, t)) <= TOL[cd], name
        outs.append(out)
    check_no_device_error()


def test_cascade_bad_prefix_is_flagged():
    cd, Hq, Hk, D, B, groups, solo = CASES["mha_f16_b16"]
    s, lay = _layout(_spec(cd, Hq, Hk, D, B), groups, solo, seed=5)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda", seed=5)
    gr = P.PrefixGroups(lay.tables, lay.lens, s.block_size)
    pb = gr.prefix_blocks.clone()
    row = int(gr.members[0])
    pb[row] = int(lay.lens[row]) // B + 3  # more prefix blocks than the sequence holds
    gr.prefix_blocks = pb
    out = torch.zeros_like(t.q)
    P.paged_attn_decode_cascade(t.q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), gr,
                                s.num_kv_heads, s.scale, s.block_size, out)
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    check_no_device_error()


# fp8-e4m3 caches (paged_attn_decode_cascade_fp8): q dtype, Hq, Hk, B, groups, solo; D = 128
FP8_CASES = {
    "fp8_gqa_bf16q_b16": ("bf16", 32, 8, 16, [(300, [10, 20, 0, 64])], [500, 1]),
    "fp8_g8_f16q_b32": ("f16", 64, 8, 32, [(257, [3, 40, 96]), (64, [0, 0, 33])], [90]),
    "fp8_mha_many_members": ("bf16", 2, 2, 16, [(64, list(range(0, 140, 2)))], []),  # 3 column chunks
    "fp8_long_prefix": ("bf16", 16, 4, 16, [(3000, [9, 100, 250])], [1000]),
}


def _fp8_spec(qd, Hq, Hk, B):
    return W.spec("llama3_8b").replace(num_q_heads=Hq, num_kv_heads=Hk, head_dim=128, block_size=B,
                                       cache_dtype="fp8_e4m3", q_dtype=qd, table_width=None)


@pytest.mark.parametrize("name", list(FP8_CASES))
def test_cascade_fp8_matches_oracle(name):
    qd, Hq, Hk, B, groups, solo = FP8_CASES[name]
    s, lay = _layout(_fp8_spec(qd, Hq, Hk, B), groups, solo, seed=sum(map(ord, name)))
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda", seed=9)
    out, gr = _run_cascade(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert gr.num_groups == len(groups)
    ref = oracle_decode(s, lay, t)
    assert max_err(out, ref) <= TOL["fp8_e4m3"], name
    plain = run_decode(s, lay, t)
    torch.cuda.synchronize()
    assert max_err(plain, ref) <= TOL["fp8_e4m3"]


def test_cascade_fp8_bf16_q_rows_beyond_f16_range():
    # Members' bf16 q rows of 2^17 and more: the prefix pass scales such a row
    # by a power of two before rounding it to f16 and takes it back in the
    # logit scale, as the decode does.
    qd, Hq, Hk, B, groups, solo = FP8_CASES["fp8_gqa_bf16q_b16"]
    s, lay = _layout(_fp8_spec(qd, Hq, Hk, B), groups, solo, seed=21)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda", seed=23)
    gr = P.PrefixGroups(lay.tables, lay.lens, s.block_size)
    big = [int(x) for x in gr.members[:2]]
    q = t.q.clone()
    q[big[0]] *= 2.0 ** 17
    q[big[1], :Hq // 2] *= 3.0e5
    t = dataclasses.replace(t, q=q)
    out, _ = _run_cascade(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert torch.isfinite(out.float()).all()
    assert max_err(out, oracle_decode(s, lay, t)) <= TOL["fp8_e4m3"]

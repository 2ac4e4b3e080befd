"""Structure checks of the seeded input generator (no method arithmetic)."""
import torch

import workloads as W
from oracle.allocator import BlockAllocator
from oracle.cache_ops import slot_of


def test_tiny_layout():
    s = W.spec("tiny")
    lay = W.make_layout(s)
    assert lay.lens.tolist() == [1, 17, 40, 100] and lay.num_blocks == 64
    used = lay.tables[lay.tables >= 0]
    assert used.numel() == 1 + 2 + 3 + 7 and len(set(used.tolist())) == used.numel()
    assert int(used.max()) < 64


def test_uniform_lens_and_append_slots():
    s = W.spec("llama3_8b")
    lay = W.make_layout(s)
    assert lay.lens.min() >= 512 and lay.lens.max() <= 4096 and lay.tables.shape == (64, 256)
    for i in range(64):
        assert int(lay.slot_mapping[i]) == slot_of(lay.tables[i].tolist(), int(lay.lens[i]) - 1, 16)
    needed = int((-(-lay.lens // 16)).sum())
    assert lay.num_blocks == -(-needed * 11 // 10) or abs(lay.num_blocks - needed * 1.1) < 1


def test_skewed_lens():
    s = W.spec("long_skewed")
    g = torch.Generator().manual_seed(s.seed)
    lens = W.draw_lens(s, g)
    long_ = [L for L in lens if L >= 32768]
    assert len(long_) == 8 and all(L <= 131072 for L in long_)
    assert sum(1 for L in lens if 64 <= L <= 512) == 248


def test_values_and_poison():
    s = W.spec("tiny")
    lay = W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens)
    assert t.q.shape == (4, 8, 64) and t.q.dtype == torch.float16
    k = t.k_cache
    # the 100-token sequence's last block holds 4 tokens, the rest is NaN
    last = int(lay.tables[3, 6])
    assert torch.isfinite(k[last, :, :4]).all() and torch.isnan(k[last, :, 4:]).all()
    free = set(range(64)) - set(lay.tables[lay.tables >= 0].tolist())
    assert all(torch.isnan(k[b]).all() for b in free)


def test_fp8_values():
    s = W.scaled_down(W.spec("long_skewed"), 8, 256, cache_dtype="fp8_e4m3")
    lay = W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens)
    assert t.k_cache.dtype == torch.uint8 and t.k_scale.shape == (8,)
    free = set(range(lay.num_blocks)) - set(lay.tables[lay.tables >= 0].tolist())
    assert all((t.k_cache[b] == W.FP8_NAN_CODE).all() for b in free)


def test_prefix_script_builds_shared_layout():
    s = W.spec("prefix_13b")
    sc = W.prefix_script(s)
    a = BlockAllocator(sc.num_blocks, s.block_size, sc.free_order)
    a.run(sc.setup)
    pre = [a.table(r) for r in range(50)]
    assert all(t[:50] == pre[0][:50] for t in pre)                 # 50 shared prefix blocks
    assert all(a.refcount[b] == 50 for b in pre[0][:50])
    assert pre[49] == pre[0]
    slots = [a.append_slot(r) for r in sc.step_appends]
    cows = [(src, dst) for _, src, dst in slots if src >= 0]
    assert len(cows) == 1 and cows[0][0] == pre[0][-1]             # request 0 copies its last block
    assert [a.num_tokens[r] for r in range(50)] == sc.final_lens

"""reshape_and_cache, its fp8 variant and copy_blocks on the GPU: bit-exact
against the oracle. Plus the whole decode step (copy-on-write copies, cache
write, decode) against the oracle chain on the same inputs."""
import numpy as np
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, max_err, check_no_device_error
from oracle.allocator import BlockAllocator as OracleAlloc
from oracle.attention import paged_decode
from oracle.cache_ops import reshape_and_cache, reshape_and_cache_fp8, copy_blocks
from oracle_io import raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()


def _pools(NB, Hk, B, D, dtype, gen):
    if dtype == torch.uint8:
        return (torch.randint(0, 256, (NB, Hk, B, D), generator=gen, dtype=torch.uint8).cuda(),
                torch.randint(0, 256, (NB, Hk, B, D), generator=gen, dtype=torch.uint8).cuda())
    return (torch.randn(NB, Hk, B, D, generator=gen).to(dtype).cuda(),
            torch.randn(NB, Hk, B, D, generator=gen).to(dtype).cuda())


@pytest.mark.parametrize("dtype,B,D,T", [(torch.bfloat16, 16, 128, 64), (torch.float16, 32, 64, 37),
                                         (torch.bfloat16, 16, 64, 1), (torch.float16, 16, 128, 300)])
def test_reshape_and_cache_bit_exact(dtype, B, D, T):
    gen = torch.Generator().manual_seed(T)
    NB, Hk = 64 + T // 4, 4
    kc, vc = _pools(NB, Hk, B, D, dtype, gen)
    k = torch.randn(T, Hk, D, generator=gen).to(dtype).cuda()
    v = torch.randn(T, Hk, D, generator=gen).to(dtype).cuda()
    slots = torch.randperm(NB * B, generator=gen)[:T].to(torch.int64)
    slots[::5] = -1                                          # padding tokens are skipped
    ek, ev = reshape_and_cache(raw(k), raw(v), raw(kc), raw(vc), slots.numpy(), B)
    P.reshape_and_cache(k, v, kc, vc, slots.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(raw(kc), ek) and np.array_equal(raw(vc), ev)
    check_no_device_error()


@pytest.mark.parametrize("xdtype,B", [(torch.bfloat16, 16), (torch.float16, 32)])
def test_reshape_and_cache_fp8_bit_exact(xdtype, B):
    gen = torch.Generator().manual_seed(11)
    NB, Hk, D, T = 40, 8, 128, 64
    kc, vc = _pools(NB, Hk, B, D, torch.uint8, gen)
    k = (torch.randn(T, Hk, D, generator=gen) * 3).to(xdtype)
    v = (torch.randn(T, Hk, D, generator=gen) * 3).to(xdtype)
    k[0, 0, :4] = torch.tensor([float("nan"), float("inf"), -float("inf"), -0.0])   # special values
    k[1, 0, :3] = torch.tensor([1e4, -1e4, 1e-8])                                     # saturate / underflow
    ks = (torch.rand(Hk, generator=gen) * 0.05 + 0.005).float()
    vs = (torch.rand(Hk, generator=gen) * 0.05 + 0.005).float()
    slots = torch.randperm(NB * B, generator=gen)[:T].to(torch.int64)
    ek, ev = reshape_and_cache_fp8(raw(k), raw(v), raw(kc), raw(vc), slots.numpy(), B,
                                   "bf16" if xdtype == torch.bfloat16 else "f16", ks.numpy(), vs.numpy())
    P.reshape_and_cache_fp8(k.cuda(), v.cuda(), kc, vc, slots.cuda(), ks.cuda(), vs.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(raw(kc), ek) and np.array_equal(raw(vc), ev)
    check_no_device_error()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.uint8])
def test_copy_blocks_bit_exact(dtype):
    gen = torch.Generator().manual_seed(5)
    NB, Hk, B, D = 50, 8, 16, 128
    kc, vc = _pools(NB, Hk, B, D, dtype, gen)
    perm = torch.randperm(NB, generator=gen)
    pairs = torch.stack([perm[:7], perm[7:14]], dim=1).to(torch.int32)
    ek, ev = copy_blocks(raw(kc), raw(vc), pairs.numpy())
    P.copy_blocks(kc, vc, pairs.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(raw(kc), ek) and np.array_equal(raw(vc), ev)
    check_no_device_error()


def test_copy_blocks_overlapping_pairs_refused():
    # A pair whose destination another pair reads (or also writes), or whose
    # source another pair writes, would make the result depend on the order
    # of the copies: it is not copied and the call is flagged; the other
    # pairs are copied bit for bit (as the oracle copies them).
    gen = torch.Generator().manual_seed(9)
    kc, vc = _pools(12, 4, 16, 64, torch.float16, gen)
    k0, v0 = kc.clone(), vc.clone()
    pairs = torch.tensor([[0, 2], [2, 1], [3, 4], [5, 5], [6, 7], [8, 7], [9, 10]], dtype=torch.int32)
    P.copy_blocks(kc, vc, pairs.cuda())
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    ek, ev = copy_blocks(raw(k0), raw(v0), np.array([[3, 4], [5, 5], [9, 10]]))
    assert np.array_equal(raw(kc), ek) and np.array_equal(raw(vc), ev)
    for blk in (1, 2, 7):                  # chained (0 -> 2 -> 1) and shared destination (7): untouched
        assert torch.equal(kc[blk], k0[blk]) and torch.equal(vc[blk], v0[blk])
    check_no_device_error()


def test_bad_slot_is_flagged_and_skipped():
    gen = torch.Generator().manual_seed(3)
    kc, vc = _pools(4, 2, 16, 64, torch.float16, gen)
    before = kc.clone()
    k = torch.randn(2, 2, 64, generator=gen).half().cuda()
    P.reshape_and_cache(k, k, kc, vc, torch.tensor([4 * 16 + 3, -1], dtype=torch.int64).cuda())
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    assert torch.equal(kc, before)


def _step_oracle(s, tables, lens, q, kp, vp, k_new, v_new, slots, pairs, ks=None, vs=None):
    """Oracle chain: copy-on-write copies, cache write, decode (raw numpy in, fp64 out)."""
    kp, vp = copy_blocks(kp, vp, pairs)
    if s.cache_dtype == "fp8_e4m3":
        kp, vp = reshape_and_cache_fp8(k_new, v_new, kp, vp, slots, s.block_size, s.q_dtype, ks, vs)
    else:
        kp, vp = reshape_and_cache(k_new, v_new, kp, vp, slots, s.block_size)
    return paged_decode(q, kp, vp, tables, lens, s.scale, s.block_size, s.q_dtype, s.cache_dtype,
                        k_scale=ks, v_scale=vs)


@pytest.mark.parametrize("variant", ["bf16", "fp8_e4m3"])
def test_append_step_matches_oracle_chain(variant):
    # llama3_8b-shaped step at reduced size: one new token per sequence, written
    # by reshape_and_cache, then decode over the post-append lengths.
    s = W.scaled_down(W.spec("llama3_8b"), 12, 600, cache_dtype=variant)
    lay = W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cuda")
    ref = _step_oracle(s, lay.tables.numpy(), lay.lens.numpy(), raw(t.q), raw(t.k_cache), raw(t.v_cache),
                       raw(t.k_new), raw(t.v_new), lay.slot_mapping.numpy(), np.zeros((0, 2)),
                       None if t.k_scale is None else t.k_scale.cpu().numpy(),
                       None if t.v_scale is None else t.v_scale.cpu().numpy())
    tables, lens = lay.tables.cuda(), lay.lens.cuda()
    out = torch.empty_like(t.q)
    if variant == "fp8_e4m3":
        P.reshape_and_cache_fp8(t.k_new, t.v_new, t.k_cache, t.v_cache, lay.slot_mapping.cuda(), t.k_scale,
                                t.v_scale)
        P.paged_attn_decode_fp8(t.q, t.k_cache, t.v_cache, t.k_scale, t.v_scale, tables, lens,
                                s.num_kv_heads, s.scale, s.block_size, out)
    else:
        P.reshape_and_cache(t.k_new, t.v_new, t.k_cache, t.v_cache, lay.slot_mapping.cuda())
        P.paged_attn_decode(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale,
                            s.block_size, out)
    torch.cuda.synchronize()
    check_no_device_error()
    assert max_err(out, ref) <= TOL[variant]


@pytest.mark.parametrize("scaled", [True, False])
def test_prefix_sharing_copy_on_write_step(scaled):
    # prefix_13b: the block layout comes from the allocator script; the product
    # allocator (C++) drives the kernels, the oracle allocator drives the oracle,
    # and the two must agree bit for bit on tables, slots and copy pairs.
    s = W.spec("prefix_13b")
    if scaled:
        s = s.replace(num_seqs=6, num_q_heads=4, num_kv_heads=4, lens=("prefix", 64, 3, 40))
    sc = W.prefix_script(s)
    a = P.BlockAllocator(sc.num_blocks, s.block_size, sc.free_order)
    o = OracleAlloc(sc.num_blocks, s.block_size, sc.free_order)
    a.run(sc.setup)
    o.run(sc.setup)
    pre_tables, pre_lens = a.build_block_tables(sc.seqs, -(-max(sc.final_lens) // s.block_size))
    step_a = [a.append_slot(r) for r in sc.step_appends]
    step_o = [o.append_slot(r) for r in sc.step_appends]
    assert step_a == step_o
    width = pre_tables.shape[1]
    tables, lens = a.build_block_tables(sc.seqs, width)
    o_tables = np.full((len(sc.seqs), width), -1, dtype=np.int64)
    for i, r in enumerate(sc.seqs):
        row = o.table(r)
        o_tables[i, :len(row)] = row
    assert np.array_equal(tables.numpy(), o_tables) and lens.tolist() == sc.final_lens
    slots = torch.tensor([x[0] for x in step_a], dtype=torch.int64)
    pairs = torch.tensor([[x[1], x[2]] for x in step_a if x[1] >= 0], dtype=torch.int32).reshape(-1, 2)
    assert pairs.shape[0] == 1
    t = W.make_tensors(s, sc.num_blocks, pre_tables, pre_lens, device="cuda")
    ref = _step_oracle(s, o_tables, np.array(sc.final_lens), raw(t.q), raw(t.k_cache), raw(t.v_cache),
                       raw(t.k_new), raw(t.v_new), slots.numpy(), pairs.numpy())
    out = torch.empty_like(t.q)
    P.copy_blocks(t.k_cache, t.v_cache, pairs.cuda())
    P.reshape_and_cache(t.k_new, t.v_new, t.k_cache, t.v_cache, slots.cuda())
    P.paged_attn_decode(t.q, t.k_cache, t.v_cache, tables.cuda(), lens.cuda(), s.num_kv_heads, s.scale,
                        s.block_size, out)
    torch.cuda.synchronize()
    check_no_device_error()
    assert max_err(out, ref) <= TOL["f16"]
    # the fork (last request) and request 0 share the prefix and differ after it
    assert not torch.equal(out[0], out[-1])

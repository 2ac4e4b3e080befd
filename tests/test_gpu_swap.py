"""Preemption by swapping on the GPU: swap_out_blocks / swap_in_blocks against
the oracle copies (bit-exact), and a preempt-resume cycle driven by the
library's allocator with the decode checked against the oracle afterwards."""
import numpy as np
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, check_no_device_error, max_err, oracle_decode, run_decode
from oracle import cache_ops
from oracle_io import raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()


def _pools(dtype, NB=40, Hk=4, B=16, D=128, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    if dtype == "fp8":
        k = torch.randint(0, 256, (NB, Hk, B, D), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
        v = torch.randint(0, 256, (NB, Hk, B, D), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    else:
        dt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
        k = torch.randn((NB, Hk, B, D), generator=g, device="cuda").to(dt)
        v = torch.randn((NB, Hk, B, D), generator=g, device="cuda").to(dt)
    return k, v


@pytest.mark.parametrize("dtype,B,D", [("bf16", 16, 128), ("f16", 32, 64), ("fp8", 16, 128)])
def test_swap_out_then_in_bit_exact(dtype, B, D):
    k, v = _pools(dtype, B=B, D=D)
    src = [5, 0, 39, 17, 5]
    dst = [1, 2, 3, 4, 6]
    rec = P.swap_record_bytes(k)
    host = torch.empty(len(src) * rec, dtype=torch.uint8).pin_memory()
    P.swap_out_blocks(k, v, torch.tensor(src, dtype=torch.int32, device="cuda"), host)
    torch.cuda.synchronize()
    want = cache_ops.swap_out(raw(k), raw(v), src)
    assert np.array_equal(host.numpy().reshape(len(src), -1), want)
    k0, v0 = raw(k), raw(v)
    P.swap_in_blocks(host, torch.tensor(dst, dtype=torch.int32, device="cuda"), k, v)
    torch.cuda.synchronize()
    ek, ev = cache_ops.swap_in(want, k0, v0, dst)
    assert np.array_equal(raw(k), ek) and np.array_equal(raw(v), ev)
    check_no_device_error()


def test_swap_rejects_bad_host_memory_and_flags_bad_blocks():
    k, v = _pools("bf16")
    blocks = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    rec = P.swap_record_bytes(k)
    with pytest.raises(P.PkvError) as e:                       # pageable host memory
        P.swap_out_blocks(k, v, blocks, torch.empty(2 * rec, dtype=torch.uint8))
    assert e.value.status == P.PKV_ERR_INVALID_ARG
    with pytest.raises(P.PkvError) as e:                       # one record short
        P.swap_out_blocks(k, v, blocks, torch.empty(rec, dtype=torch.uint8).pin_memory())
    assert e.value.status == P.PKV_ERR_INVALID_ARG
    host = torch.zeros(2 * rec, dtype=torch.uint8).pin_memory()
    P.swap_out_blocks(k, v, torch.tensor([1, 10 ** 6], dtype=torch.int32, device="cuda"), host)
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    assert np.array_equal(host.numpy()[:rec], cache_ops.swap_out(raw(k), raw(v), [1])[0])
    assert not host.numpy()[rec:].any()                        # the bad block's record is skipped
    check_no_device_error()


def test_preempt_and_resume_decode():
    # Sequences laid out by the library's allocator; sequence 2 is swapped out,
    # its freed blocks are reused (and overwritten) by a new sequence, then it
    # is swapped back into fresh blocks and the batch decodes as before.
    s = W.spec("llama3_8b").replace(num_seqs=4, table_width=None, append=False)
    B = s.block_size
    lens = [700, 1000, 333, 64]
    nb = 300
    a = P.BlockAllocator(nb, B, list(np.random.default_rng(1).permutation(nb)))
    for i, L in enumerate(lens):
        a.allocate(i, L)
    width = 80
    tables, lens_t = a.build_block_tables(range(4), width)
    lay = W.Layout(s, nb, lens_t, tables, lens_t.clone(), tables.clone())
    t = W.make_tensors(s, nb, tables, lens_t, device="cuda")
    ref = oracle_decode(s, lay, t)

    out_blocks = a.swap_out(2)
    rec = P.swap_record_bytes(t.k_cache)
    host = torch.empty(len(out_blocks) * rec, dtype=torch.uint8).pin_memory()
    P.swap_out_blocks(t.k_cache, t.v_cache, torch.tensor(out_blocks, dtype=torch.int32, device="cuda"), host)
    # a new sequence takes all but 9 free blocks, reaching the swapped-out ones
    # at the tail of the free list, overwrites them and finishes
    a.allocate(9, (a.num_free() - 9) * B)
    reused = a.table(9)
    assert set(out_blocks) & set(reused)
    t.k_cache[reused] = 0
    t.v_cache[reused] = 0
    a.free(9)
    in_blocks = a.swap_in(2)
    assert len(in_blocks) == len(out_blocks) and a.num_tokens(2) == lens[2]
    P.swap_in_blocks(host, torch.tensor(in_blocks, dtype=torch.int32, device="cuda"), t.k_cache, t.v_cache)
    tables2, lens2 = a.build_block_tables(range(4), width)
    lay2 = W.Layout(s, nb, lens2, tables2, lens2.clone(), tables2.clone())
    out = run_decode(s, lay2, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert max_err(out, ref) <= TOL[s.cache_dtype]

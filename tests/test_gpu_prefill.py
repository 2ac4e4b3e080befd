"""Multi-token (causal) paged attention on the GPU against the fp64 oracle
(paged_prefill), through the C ABI. Tolerances as for the decode."""
import numpy as np
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, check_no_device_error, max_err
from oracle.attention import paged_prefill
from oracle_io import raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()


def _case(spec, nq, seed=5):
    """Layout and pool from the workload; nq[s] new tokens per sequence (the
    last ones of its context), their queries drawn here."""
    s = spec.replace(append=False)
    lay = W.make_layout(s, seed=seed)
    t = W.make_tensors(s, lay.num_blocks, lay.tables, lay.lens, device="cuda", seed=seed)
    nq = [min(int(n), int(L)) for n, L in zip(nq, lay.lens.tolist())]
    q_start = torch.tensor(np.concatenate([[0], np.cumsum(nq)]), dtype=torch.int32)
    T = int(q_start[-1])
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16}[s.q_dtype]
    q = torch.randn((T, s.num_q_heads, s.head_dim), generator=g, device="cuda").to(dt)
    return s, lay, t, q, q_start, max(nq) if nq else 0


def _run(s, lay, t, q, q_start, max_q):
    out = torch.full_like(q, float("nan"))
    P.paged_attn_prefill(q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), q_start.cuda(), max_q,
                         s.num_kv_heads, s.scale, s.block_size, out, k_scale=t.k_scale, v_scale=t.v_scale)
    torch.cuda.synchronize()
    return out


def _oracle(s, lay, t, q, q_start, seqs=None):
    ks = None if t.k_scale is None else t.k_scale.cpu().numpy()
    vs = None if t.v_scale is None else t.v_scale.cpu().numpy()
    return paged_prefill(raw(q), raw(t.k_cache), raw(t.v_cache), lay.tables.numpy(), lay.lens.numpy(),
                         q_start.numpy(), s.scale, s.block_size, s.q_dtype, s.cache_dtype,
                         k_scale=ks, v_scale=vs, seqs=seqs)


CASES = {
    # spec, new tokens per sequence
    "verify_gqa": (W.scaled_down(W.spec("llama3_8b"), 8, 900), [4] * 8),
    "verify_g8_b32": (W.scaled_down(W.spec("llama3_70b"), 4, 700, block_size=32).replace(lens=("uniform", 40, 700)),
                      [5, 1, 7, 3]),
    "chunk_mha_f16": (W.spec("llama3_8b").replace(num_seqs=3, num_q_heads=4, num_kv_heads=4, cache_dtype="f16",
                                                  q_dtype="f16", lens=("fixed", [700, 300, 129]), table_width=None),
                      [300, 300, 17]),
    "whole_prompt_d64": (W.spec("tiny").replace(cache_dtype="bf16", q_dtype="bf16", block_size=32,
                                                lens=("fixed", [1, 33, 64, 70]), pool_blocks=None),
                         [1, 33, 64, 70]),
    "mixed_counts": (W.spec("llama3_8b").replace(num_seqs=6, lens=("fixed", [16, 17, 1, 500, 48, 2]),
                                                 table_width=None),
                     [16, 0, 1, 40, 33, 2]),
    # 128-row tiles on the tensor cores (D = 128, at least 128 query rows)
    "tc_chunk_g8_b32": (W.spec("llama3_70b").replace(num_seqs=2, block_size=32, lens=("fixed", [900, 601]),
                                                     table_width=None),
                        [300, 129]),
    "tc_chunk_gqa_f16": (W.spec("llama3_8b").replace(num_seqs=3, cache_dtype="f16", q_dtype="f16",
                                                     lens=("fixed", [333, 129, 700]), table_width=None),
                         [333, 64, 250]),
    # 64 rows at most: one half-filled tensor-core tile per (sequence, head)
    "tc_half_tile": (W.spec("llama3_8b").replace(num_seqs=4, lens=("fixed", [200, 16, 77, 1000]),
                                                 table_width=None),
                     [16, 9, 1, 16]),
    # fp8-e4m3 caches (paged_attn_prefill_fp8): the warp-MMA kernel at every
    # row count, with and without the KV split
    "fp8_verify_gqa": (W.scaled_down(W.spec("llama3_8b"), 8, 900, cache_dtype="fp8_e4m3"), [4] * 8),
    "fp8_chunk_g8_b32": (W.spec("llama3_70b").replace(num_seqs=2, block_size=32, cache_dtype="fp8_e4m3",
                                                      lens=("fixed", [900, 601]), table_width=None),
                         [300, 129]),
    "fp8_mixed_f16q": (W.spec("llama3_8b").replace(num_seqs=6, cache_dtype="fp8_e4m3", q_dtype="f16",
                                                   lens=("fixed", [16, 17, 1, 500, 48, 2]), table_width=None),
                       [16, 0, 1, 40, 33, 2]),
    # fp8 with several warps per CTA: 16 tokens x 4 heads over long contexts
    # (4 warps, KV split), and 2 warps on 32-token blocks with partly filled
    # last blocks
    "fp8_q16_split": (W.scaled_down(W.spec("llama3_8b"), 6, 2500, cache_dtype="fp8_e4m3"), [16] * 6),
    "fp8_q8_b32": (W.spec("llama3_8b").replace(num_seqs=3, block_size=32, cache_dtype="fp8_e4m3",
                                               lens=("fixed", [70, 33, 300]), table_width=None),
                   [8, 5, 8]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_oracle(name):
    spec, nq = CASES[name]
    s, lay, t, q, q_start, max_q = _case(spec, nq)
    out = _run(s, lay, t, q, q_start, max_q)
    check_no_device_error()
    ref = _oracle(s, lay, t, q, q_start)
    assert max_err(out, ref) <= TOL[s.cache_dtype], name


def test_one_token_per_sequence_is_the_decode_step():
    # T = S and max_q_tokens = 1: served by the decode kernels
    spec = W.scaled_down(W.spec("llama3_8b"), 8, 700)
    s, lay, t, q, q_start, max_q = _case(spec, [1] * 8)
    out = _run(s, lay, t, q, q_start, max_q)
    dec = torch.full_like(q, float("nan"))
    P.paged_attn_decode(q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), s.num_kv_heads, s.scale,
                        s.block_size, dec)
    torch.cuda.synchronize()
    check_no_device_error()
    # same kernels; work stealing may cut units differently between calls,
    # so the merge order (and the last bit) can differ
    assert (out.float() - dec.float()).abs().max().item() <= TOL[s.cache_dtype]
    assert max_err(out, _oracle(s, lay, t, q, q_start)) <= TOL[s.cache_dtype]


def test_one_token_for_some_sequences_uses_the_multi_token_path():
    # max_q_tokens = 1 but fewer rows than sequences: the multi-token kernel
    spec = W.scaled_down(W.spec("llama3_8b"), 6, 500)
    s, lay, t, q, q_start, max_q = _case(spec, [1, 0, 1, 1, 0, 1])
    out = _run(s, lay, t, q, q_start, max_q)
    check_no_device_error()
    assert max_err(out, _oracle(s, lay, t, q, q_start)) <= TOL[s.cache_dtype]


def test_full_size_verification_sampled():
    # llama3_8b-shaped batch verifying 4 speculative tokens per sequence
    spec = W.spec("llama3_8b")
    s, lay, t, q, q_start, max_q = _case(spec, [4] * spec.num_seqs)
    out = _run(s, lay, t, q, q_start, max_q)
    check_no_device_error()
    seqs = [0, 17, 40, 63]
    ref = _oracle(s, lay, t, q, q_start, seqs=seqs)
    rows = [r for sq in seqs for r in range(int(q_start[sq]), int(q_start[sq + 1]))]
    assert max_err(out, ref, rows) <= TOL[s.cache_dtype]
    assert torch.isfinite(out).all()


def test_full_size_chunk_sampled():
    # llama3_8b-shaped batch with a 64-token chunk per sequence (256 query rows
    # per kv head: tensor-core tiles)
    spec = W.spec("llama3_8b")
    s, lay, t, q, q_start, max_q = _case(spec, [64] * spec.num_seqs)
    out = _run(s, lay, t, q, q_start, max_q)
    check_no_device_error()
    seqs = [3, 31, 62]
    ref = _oracle(s, lay, t, q, q_start, seqs=seqs)
    rows = [r for sq in seqs for r in range(int(q_start[sq]), int(q_start[sq + 1]))]
    assert max_err(out, ref, rows) <= TOL[s.cache_dtype]
    assert torch.isfinite(out).all()


def test_inconsistent_rows_are_flagged():
    spec = W.scaled_down(W.spec("llama3_8b"), 4, 300)
    s, lay, t, q, q_start, max_q = _case(spec, [3] * 4)
    lens = lay.lens.clone()
    lens[1] = 2                                   # fewer tokens than new ones
    out = torch.zeros_like(q)
    P.paged_attn_prefill(q, t.k_cache, t.v_cache, lay.tables.cuda(), lens.cuda(), q_start.cuda(), max_q,
                         s.num_kv_heads, s.scale, s.block_size, out)
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    check_no_device_error()


def test_fp8_one_token_per_sequence_is_the_fp8_decode_step():
    spec = W.scaled_down(W.spec("long_skewed"), 8, 1500, cache_dtype="fp8_e4m3")
    s, lay, t, q, q_start, max_q = _case(spec, [1] * 8)
    out = _run(s, lay, t, q, q_start, max_q)
    dec = torch.full_like(q, float("nan"))
    P.paged_attn_decode_fp8(q, t.k_cache, t.v_cache, t.k_scale, t.v_scale, lay.tables.cuda(), lay.lens.cuda(),
                            s.num_kv_heads, s.scale, s.block_size, dec)
    torch.cuda.synchronize()
    check_no_device_error()
    assert (out.float() - dec.float()).abs().max().item() <= TOL["fp8_e4m3"]
    assert max_err(out, _oracle(s, lay, t, q, q_start)) <= TOL["fp8_e4m3"]


def test_fp8_bf16_q_rows_beyond_f16_range():
    # bf16 query rows past the f16 maximum on an fp8 cache: each such row is
    # scaled by a power of two before its f16 rounding (its logit scale takes
    # it back), so the outputs stay finite and within tolerance
    spec = W.scaled_down(W.spec("llama3_8b"), 4, 600, cache_dtype="fp8_e4m3")
    s, lay, t, q, q_start, max_q = _case(spec, [5, 3, 8, 2])
    q = q.float()
    q[::2] *= 2.5e4
    q[1, 3] = 0.0
    q[1, 3, 5] = -1.2e5
    q = q.to(torch.bfloat16)
    assert q.float().abs().max() > 65504
    out = _run(s, lay, t, q, q_start, max_q)
    check_no_device_error()
    assert torch.isfinite(out.float()).all()
    assert max_err(out, _oracle(s, lay, t, q, q_start)) <= TOL["fp8_e4m3"]

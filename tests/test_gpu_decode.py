"""Decode attention on the GPU against the fp64 oracle (through the C ABI).

Small cases compare every output element; the full-size workloads compare
sampled sequences. Tolerances (max abs error vs the oracle on the stored,
dequantised cache): fp16 2e-3, bf16 1e-2, fp8-e4m3 3e-2.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, decode_case, run_decode, oracle_decode, max_err, check_no_device_error
from oracle.numerics import decode_e4m3
from oracle_io import raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()
    torch.cuda.init()


def _small(name, **kw):
    base = W.spec(name)
    return base.replace(**kw)


SMALL = {
    "tiny": W.spec("tiny"),
    "8b_small": W.scaled_down(W.spec("llama3_8b"), 8, 700),
    "70b_small": W.scaled_down(W.spec("llama3_70b"), 4, 900).replace(lens=("uniform", 300, 900)),
    "mha_f16": W.spec("llama3_8b").replace(num_seqs=5, num_q_heads=6, num_kv_heads=6, cache_dtype="f16",
                                           q_dtype="f16", lens=("uniform", 1, 400), table_width=None),
    "skewed_b16": W.scaled_down(W.spec("long_skewed"), 16, 3000),
    "skewed_b32": W.scaled_down(W.spec("long_skewed"), 16, 3000, block_size=32),
    "skewed_fp8_b16": W.scaled_down(W.spec("long_skewed"), 16, 3000, cache_dtype="fp8_e4m3"),
    "skewed_fp8_b32": W.scaled_down(W.spec("long_skewed"), 16, 3000, cache_dtype="fp8_e4m3",
                                    block_size=32),
    "fp8_f16q": W.scaled_down(W.spec("long_skewed"), 6, 500, cache_dtype="fp8_e4m3", q_dtype="f16"),
    "d64_bf16_b32": W.spec("tiny").replace(cache_dtype="bf16", q_dtype="bf16", block_size=32,
                                           pool_blocks=None, lens=("fixed", [5, 33, 64, 70])),
    "d64_f16_b16_g1": W.spec("tiny").replace(num_q_heads=2, lens=("fixed", [3, 16, 31, 48])),
    "f16_b32_g8": W.spec("llama3_70b").replace(num_seqs=3, cache_dtype="f16", q_dtype="f16",
                                               block_size=32, lens=("fixed", [33, 100, 257]),
                                               table_width=None),
    "g3": W.spec("llama3_8b").replace(num_seqs=3, num_q_heads=6, num_kv_heads=2,
                                      lens=("fixed", [40, 1, 77]), table_width=None),
    "g6": W.spec("llama3_8b").replace(num_seqs=3, num_q_heads=12, num_kv_heads=2,
                                      lens=("fixed", [140, 16, 17]), table_width=None),
    "edge_lens": W.spec("llama3_8b").replace(num_seqs=9, lens=("fixed", [0, 1, 15, 16, 17, 31, 32, 33, 0]),
                                             table_width=None),
    "many_short": W.spec("llama3_8b").replace(num_seqs=300, num_q_heads=8, num_kv_heads=2,
                                              lens=("uniform", 0, 40), table_width=None),
    "one_long": W.spec("llama3_8b").replace(num_seqs=1, lens=("fixed", [6000]), table_width=None),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_matches_oracle_small(name):
    s, lay, t = decode_case(SMALL[name], seed=SMALL[name].seed + 99)
    out = run_decode(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    ref = oracle_decode(s, lay, t)
    err = max_err(out, ref)
    assert err <= TOL[s.cache_dtype], (name, err)


def test_one_token_context_returns_v0_exactly():
    for cd in ("f16", "bf16"):
        s = W.spec("llama3_70b").replace(num_seqs=3, cache_dtype=cd, q_dtype=cd, lens=("fixed", [1, 1, 1]),
                                         table_width=None)
        s, lay, t = decode_case(s)
        out = run_decode(s, lay, t)
        for i in range(3):
            blk = int(lay.tables[i, 0])
            for h in range(s.num_q_heads):
                v0 = t.v_cache[blk, h // s.group, 0]
                assert torch.equal(out[i, h], v0), (cd, i, h)
    check_no_device_error()


def test_repeated_calls_and_explicit_workspace():
    # Work is rebalanced between warps at run time, so repeated calls may cut
    # units differently (last-bit differences); each result meets the tolerance.
    s, lay, t = decode_case(W.scaled_down(W.spec("long_skewed"), 16, 3000))
    ref = oracle_decode(s, lay, t)
    nbytes = P.workspace_bytes(s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, P.PKV_BF16,
                               torch.cuda.current_device())
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for i in range(6):
        out = run_decode(s, lay, t, workspace=ws if i % 2 else None)
        torch.cuda.synchronize()
        assert max_err(out, ref) <= TOL[s.cache_dtype], i
    with pytest.raises(P.PkvError) as e:
        run_decode(s, lay, t, workspace=ws[: nbytes // 2])
    assert e.value.status == P.PKV_ERR_WORKSPACE
    check_no_device_error()


def test_fp8_widening_of_every_code():
    # One token whose V row holds 128 codes: out = decode(code) * v_scale exactly
    # (every e4m3 value is exact in bf16), for both halves of the code space.
    for half in range(2):
        s = W.spec("long_skewed").replace(num_seqs=1, num_q_heads=1, num_kv_heads=1, cache_dtype="fp8_e4m3",
                                          lens=("fixed", [1]), table_width=None, pool_blocks=4)
        s, lay, t = decode_case(s)
        codes = torch.arange(128 * half, 128 * half + 128, dtype=torch.int64)
        codes[codes == 0x7F] = 0x7E
        codes[codes == 0xFF] = 0xFE
        blk = int(lay.tables[0, 0])
        t.v_cache[blk, 0, 0] = codes.to(torch.uint8).cuda()
        t.v_scale.fill_(1.0)
        out = run_decode(s, lay, t)
        expect = torch.tensor(decode_e4m3(codes.numpy()), dtype=torch.float64)
        assert torch.equal(out[0, 0].double().cpu(), expect), half
    check_no_device_error()


def test_bad_inputs_are_flagged_not_faulted():
    s, lay, t = decode_case(W.spec("tiny"))
    tables = lay.tables.clone()
    tables[1, 0] = 10 ** 6                       # block id outside the pool
    out = torch.empty_like(t.q)
    P.paged_attn_decode(t.q, t.k_cache, t.v_cache, tables.cuda(), lay.lens.cuda(), s.num_kv_heads, s.scale,
                        s.block_size, out)
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    lens = lay.lens.clone()
    lens[2] = lay.tables.shape[1] * s.block_size + 5   # longer than the table row
    P.paged_attn_decode(t.q, t.k_cache, t.v_cache, lay.tables.cuda(), lens.cuda(), s.num_kv_heads, s.scale,
                        s.block_size, out)
    assert P.device_error(torch.cuda.current_device()) == P.PKV_ERR_DEVICE_CHECK
    check_no_device_error()                       # the flag was cleared
    with pytest.raises(P.PkvError) as e:         # host-side shape check
        P.paged_attn_decode(t.q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), 3, s.scale,
                            s.block_size, out)
    assert e.value.status == P.PKV_ERR_INVALID_ARG


def _sample(lens, k, rng):
    order = np.argsort(lens)
    pick = set(int(i) for i in order[-2:]) | set(int(i) for i in order[:2])
    pick |= set(int(i) for i in rng.choice(len(lens), size=min(k, len(lens)), replace=False))
    return sorted(pick)


@pytest.mark.parametrize("name,over", [
    ("llama3_8b", {}),
    ("llama3_70b", {}),
    ("long_skewed", {}),
    ("long_skewed", {"block_size": 32}),
    ("long_skewed", {"cache_dtype": "fp8_e4m3"}),
    ("long_skewed", {"cache_dtype": "fp8_e4m3", "block_size": 32}),
])
def test_decode_full_size_sampled(name, over):
    spec = W.spec(name, **over)
    s, lay, t = decode_case(spec)
    out = run_decode(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    seqs = _sample(lay.lens.numpy(), 4, np.random.default_rng(0))
    ref = oracle_decode(s, lay, t, seqs=seqs)
    err = max_err(out, ref, seqs)
    assert err <= TOL[s.cache_dtype], (name, over, err)
    # every other row is finite and bounded by the largest |v| of the pool
    assert torch.isfinite(out).all()


def test_one_workspace_shared_by_configurations():
    # Kernel configurations differ in grid size (one or two CTAs per SM); the
    # work-claiming state of one must not be disturbed by another's scratch.
    cases = [decode_case(SMALL[n], seed=SMALL[n].seed + 7)
             for n in ("skewed_b32", "8b_small", "d64_f16_b16_g1", "skewed_fp8_b16", "tiny")]
    dev = torch.cuda.current_device()
    code = {"bf16": P.PKV_BF16, "f16": P.PKV_F16, "fp8_e4m3": P.PKV_FP8_E4M3}
    nbytes = max(P.workspace_bytes(s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size,
                                   code[s.cache_dtype], dev) for s, _, _ in cases)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    refs = [oracle_decode(*c) for c in cases]
    for rnd in range(3):
        for (s, lay, t), ref in zip(cases, refs):
            out = run_decode(s, lay, t, workspace=ws)
            torch.cuda.synchronize()
            assert max_err(out, ref) <= TOL[s.cache_dtype], (rnd, s.name)
    check_no_device_error()


def test_cut_unit_with_more_pieces_than_one_merge_pass():
    # One (sequence, kv head) unit spread over the whole persistent grid: at
    # D = 64 and 16-token blocks a B200 runs 2 CTAs of 4 warps per SM (1184
    # warps), and 40000 tokens give every warp part of the unit, so the merge
    # folds more pieces than its list holds (1024) in more than one pass.
    for g, cd in ((1, "f16"), (8, "bf16")):
        s = W.spec("tiny").replace(num_seqs=1, num_q_heads=g, num_kv_heads=1, cache_dtype=cd, q_dtype=cd,
                                   lens=("fixed", [40000]), pool_blocks=None, table_width=None)
        s, lay, t = decode_case(s)
        out = run_decode(s, lay, t)
        torch.cuda.synchronize()
        check_no_device_error()
        assert max_err(out, oracle_decode(s, lay, t)) <= TOL[cd], (g, cd)


def test_fp8_bf16_q_rows_beyond_f16_range():
    # bf16 q rows up to ~1e5 (past the f16 maximum 65504) on an fp8 cache: the
    # row is scaled by a power of two before its f16 rounding, so the output
    # stays finite and within tolerance; ordinary rows of the same batch are
    # unaffected.
    s, lay, t = decode_case(W.scaled_down(W.spec("long_skewed"), 8, 1500, cache_dtype="fp8_e4m3"))
    q = t.q.float()
    q[::2] *= 2.5e4                       # every other sequence: |q| up to about 1e5
    q[1, 3] = 0.0
    q[1, 3, 5] = -1.2e5                   # one element far past 65504, rest of that row 0
    t.q.copy_(q.to(t.q.dtype))
    assert t.q.float().abs().max() > 65504
    out = run_decode(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert max_err(out, oracle_decode(s, lay, t)) <= TOL["fp8_e4m3"]


@pytest.mark.parametrize("name", ["skewed_b16", "skewed_fp8_b16", "one_long", "d64_f16_b16_g1"])
def test_deterministic_flag_gives_identical_bits(name):
    s, lay, t = decode_case(SMALL[name], seed=SMALL[name].seed + 5)
    code = {"bf16": P.PKV_BF16, "f16": P.PKV_F16, "fp8_e4m3": P.PKV_FP8_E4M3}[s.cache_dtype]
    nbytes = P.workspace_bytes(s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, code,
                               torch.cuda.current_device())
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    tables, lens = lay.tables.cuda(), lay.lens.cuda()
    outs = []
    for _ in range(5):
        out = torch.full_like(t.q, float("nan"))
        P.paged_attn_decode_ex(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale, s.block_size,
                               out, ws, t.k_scale, t.v_scale, flags=P.PKV_DECODE_DETERMINISTIC)
        outs.append(out)
    torch.cuda.synchronize()
    check_no_device_error()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16)), name
    assert max_err(outs[0], oracle_decode(s, lay, t)) <= TOL[s.cache_dtype], name
    with pytest.raises(P.PkvError) as e:
        P.paged_attn_decode_ex(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale, s.block_size,
                               outs[0], ws, t.k_scale, t.v_scale, flags=2)
    assert e.value.status == P.PKV_ERR_INVALID_ARG


def test_fp8_adaptive_partition_across_shapes():
    # The fp8 decode cuts its static ranges by weights the previous call
    # learned (kept in the workspace) when the batch has at least as many
    # (sequence, kv head) units as warp ranges (1184 on a B200). Alternate
    # two such batches of one kernel configuration on one workspace, so that
    # most calls run on a partition learned from the other batch: every call
    # must still match the oracle, and a PKV_DECODE_DETERMINISTIC call (equal
    # ranges, no stealing) must give the same bits whatever the learned state.
    a = decode_case(W.scaled_down(W.spec("long_skewed"), 160, 3000, cache_dtype="fp8_e4m3"), seed=71)
    b = decode_case(W.scaled_down(W.spec("llama3_8b"), 150, 900, cache_dtype="fp8_e4m3"), seed=72)
    assert a[0].num_seqs * a[0].num_kv_heads >= 1184 and b[0].num_seqs * b[0].num_kv_heads >= 1184
    s0 = a[0]
    nbytes = P.workspace_bytes(s0.num_q_heads, s0.num_kv_heads, s0.head_dim, s0.block_size,
                               P.PKV_FP8_E4M3, torch.cuda.current_device())
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    refs = [oracle_decode(*c) for c in (a, b)]
    dev_args = [(lay.tables.cuda(), lay.lens.cuda()) for _, lay, _ in (a, b)]

    def call(i, flags=0):
        s, lay, t = (a, b)[i]
        out = torch.full_like(t.q, float("nan"))
        P.paged_attn_decode_ex(t.q, t.k_cache, t.v_cache, *dev_args[i], s.num_kv_heads, s.scale,
                               s.block_size, out, ws, t.k_scale, t.v_scale, flags=flags)
        return out

    det0 = call(0, P.PKV_DECODE_DETERMINISTIC)
    for r in range(6):
        for i in (0, 1):
            out = call(i)
            torch.cuda.synchronize()
            assert max_err(out, refs[i]) <= TOL["fp8_e4m3"], (r, i)
    det1 = call(0, P.PKV_DECODE_DETERMINISTIC)
    torch.cuda.synchronize()
    check_no_device_error()
    assert torch.equal(det0.view(torch.int16), det1.view(torch.int16))


@pytest.mark.parametrize("block_size", [16, 32])
def test_fp8_logits_climbing_and_jumping_along_the_context(block_size):
    # The fp8 decode moves a column's exponent base only when a score passes
    # it by more than 8, so its softmax weights reach 2^8 between moves. Keys
    # whose logits climb along the context (about 60 in the exp2 domain from
    # first to last token: many moves, weights up to 2^8 in between) and, on
    # every other sequence, a jump of about 30 over the last tenth of the
    # context (O rescaled late) must still match the oracle.
    from oracle.numerics import encode_e4m3
    s, lay, t = decode_case(W.scaled_down(W.spec("long_skewed"), 6, 3000, cache_dtype="fp8_e4m3",
                                          block_size=block_size), seed=91)
    g, Hk, B = s.num_q_heads // s.num_kv_heads, s.num_kv_heads, s.block_size
    ks = t.k_scale.cpu().numpy().astype(np.float64)
    log2e = 1.0 / np.log(2.0)
    # q = (A_h, 0, ..., 0): the exp2-domain logit of a key is A_h * scale *
    # k_scale[h] * log2(e) * K[0], and K[0] = 448 (the e4m3 maximum) maps to 60
    amp = 60.0 / (448.0 * s.scale * ks * log2e)
    q = torch.zeros(t.q.shape, dtype=torch.float32)
    for hq in range(s.num_q_heads):
        q[:, hq, 0] = float(amp[hq // g])
    t.q.copy_(q.to(t.q.dtype))
    kc = t.k_cache.cpu().numpy()
    tables, lens = lay.tables.numpy(), lay.lens.numpy()
    for si in range(s.num_seqs):
        L = int(lens[si])
        if L == 0:
            continue
        j = np.arange(L)
        if si % 2 == 0:
            val = 448.0 * j / max(L - 1, 1)
        else:
            val = np.where(j >= int(0.9 * L), 448.0, 224.0 * j / max(L - 1, 1))
        codes = encode_e4m3(val)
        phys = tables[si, j // B]
        for h in range(Hk):
            kc[phys, h, j % B, 0] = codes
    t.k_cache.copy_(torch.from_numpy(kc))
    out = run_decode(s, lay, t)
    torch.cuda.synchronize()
    check_no_device_error()
    assert max_err(out, oracle_decode(s, lay, t)) <= TOL["fp8_e4m3"]

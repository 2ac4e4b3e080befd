"""Seeded synthetic inputs for the paged-KV decode path.

This module draws random numbers and places blocks in a pool; it holds none of
the method's arithmetic (no attention, softmax, quantisation rule or
allocator policy). Both the CUDA path and the CPU oracle take their inputs
from here, and nothing here imports either of them.

Workloads (the five decode shapes the PagedAttention pages motivate: the
13B-class sizing in "Why the cache exists, and why it's so hungry" of
"KV-Cache Management and PagedAttention", the Llama-3 sizing example and the
shared-prompt flowchart of "PagedAttention and KV Cache Management"):

  tiny          4 seqs, lens {1,17,40,100}, 8 q / 2 kv heads, D=64, B=16, fp16,
                pool of 64 blocks in seeded random order
  llama3_8b     64 seqs, lens ~ U[512,4096], 32 q / 8 kv heads, D=128, B=16,
                bf16, pool = needed blocks + 10 %, shuffled; the step appends
                one new token per sequence (64 tokens) before the decode
  llama3_70b    64 seqs, all lens 4096, 64 q / 8 kv heads, D=128, B=16, bf16
  prefix_13b    50 requests sharing an 800-token prefix (50 full blocks held
                once), private suffixes ~ U[32,256], 40 q = 40 kv heads, D=128,
                fp16; the block layout is given as an operation script that a
                block allocator executes (a fork makes one partially filled
                last block shared, so the step's append copies it on write)
  long_skewed   8 seqs ~ U[32768,131072] + 248 seqs ~ U[64,512], 32 q / 8 kv
                heads, D=128, B=16 or 32, bf16 or fp8-e4m3 with per-head fp32
                scales

Values: q, k, v ~ N(0,1) drawn in fp32 and rounded to the storage type.
Unused slots of the pool (free blocks, the tail of each last block, the slot a
step's new token will fill) hold NaN (fp8: code 0x7F), so a kernel that reads
them into a result shows it.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import torch

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
FP8_NAN_CODE = 0x7F
FP8_MAX = 448.0

SEED_BASE = 0x5EED0000


@dataclasses.dataclass(frozen=True)
class Spec:
    """Shape of one decode workload."""

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    cache_dtype: str  # "f16" | "bf16" | "fp8_e4m3"
    q_dtype: str  # "f16" | "bf16"
    lens: Tuple  # ("fixed", [...]) | ("uniform", lo, hi) | ("skewed", n_long, lo, hi, n_short, lo, hi) | ("prefix", P, lo, hi)
    pool_blocks: Optional[int] = None  # fixed pool size; else needed * (1 + slack)
    pool_slack: float = 0.10
    table_width: Optional[int] = None  # block-table row width; default: recipe max / B
    append: bool = False  # step writes one new token per sequence first
    seed: int = SEED_BASE

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def cache_elem_bytes(self) -> int:
        return 1 if self.cache_dtype == "fp8_e4m3" else 2

    def replace(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


def spec(name: str, **overrides) -> Spec:
    """The named workload, optionally with fields replaced (e.g. block_size)."""
    base = {
        "tiny": Spec("tiny", 4, 8, 2, 64, 16, "f16", "f16", ("fixed", [1, 17, 40, 100]),
                     pool_blocks=64, seed=SEED_BASE + 1),
        "llama3_8b": Spec("llama3_8b", 64, 32, 8, 128, 16, "bf16", "bf16", ("uniform", 512, 4096),
                          append=True, seed=SEED_BASE + 2),
        "llama3_70b": Spec("llama3_70b", 64, 64, 8, 128, 16, "bf16", "bf16", ("fixed", [4096] * 64),
                           seed=SEED_BASE + 3),
        "prefix_13b": Spec("prefix_13b", 50, 40, 40, 128, 16, "f16", "f16", ("prefix", 800, 32, 256),
                           append=True, seed=SEED_BASE + 4),
        "long_skewed": Spec("long_skewed", 256, 32, 8, 128, 16, "bf16", "bf16",
                            ("skewed", 8, 32768, 131072, 248, 64, 512), seed=SEED_BASE + 5),
    }[name]
    return base.replace(**overrides) if overrides else base


def describe(s: Spec) -> str:
    return (f"{s.name}: S={s.num_seqs} Hq={s.num_q_heads} Hk={s.num_kv_heads} D={s.head_dim} "
            f"B={s.block_size} cache={s.cache_dtype} q={s.q_dtype} lens={s.lens}")


def _uniform_ints(gen: torch.Generator, n: int, lo: int, hi: int) -> List[int]:
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def draw_lens(s: Spec, gen: torch.Generator) -> List[int]:
    kind = s.lens[0]
    if kind == "fixed":
        lens = list(s.lens[1])
        assert len(lens) == s.num_seqs
        return lens
    if kind == "uniform":
        return _uniform_ints(gen, s.num_seqs, s.lens[1], s.lens[2])
    if kind == "skewed":
        _, n_long, llo, lhi, n_short, slo, shi = s.lens
        assert n_long + n_short == s.num_seqs
        lens = _uniform_ints(gen, n_long, llo, lhi) + _uniform_ints(gen, n_short, slo, shi)
        order = torch.randperm(s.num_seqs, generator=gen).tolist()
        return [lens[i] for i in order]
    raise ValueError(f"lens recipe {kind!r} has no direct layout (use prefix_script)")


def _recipe_max_len(s: Spec) -> int:
    kind = s.lens[0]
    if kind == "fixed":
        return max(s.lens[1]) if s.lens[1] else 0
    if kind == "uniform":
        return s.lens[2]
    if kind == "skewed":
        return max(s.lens[3], s.lens[6])
    if kind == "prefix":
        return s.lens[1] + s.lens[3]
    raise ValueError(kind)


@dataclasses.dataclass
class Layout:
    """Where every token of every sequence lives in the pool.

    `tables` / `lens` describe the state the decode reads (after the step's
    append when `spec.append`); `fill_tables` / `fill_lens` describe the state
    before the step, i.e. which slots hold data when the step starts.
    """

    spec: Spec
    num_blocks: int
    lens: torch.Tensor  # int32 [S]
    tables: torch.Tensor  # int32 [S, W], -1 past ceil(L/B)
    fill_lens: torch.Tensor  # int32 [S]
    fill_tables: torch.Tensor  # int32 [S, W]
    slot_mapping: Optional[torch.Tensor] = None  # int64 [S] new token slots (append only)
    cow_pairs: Optional[torch.Tensor] = None  # int32 [n, 2] (src, dst) block copies (append only)


def _table_width(s: Spec) -> int:
    if s.table_width is not None:
        return s.table_width
    return max(1, -(-_recipe_max_len(s) // s.block_size))


def make_layout(s: Spec, seed: Optional[int] = None) -> Layout:
    """Lay each sequence's blocks out at seeded random places in the pool.

    Every sequence gets ceil(L/B) blocks of its own (no sharing); the pool is
    a seeded permutation of block ids, handed out in order.
    """
    if s.lens[0] == "prefix":
        raise ValueError("prefix workloads are laid out by an allocator from prefix_script()")
    gen = torch.Generator().manual_seed(s.seed if seed is None else seed)
    lens = draw_lens(s, gen)
    B = s.block_size
    nb = [-(-L // B) for L in lens]
    needed = sum(nb)
    if s.pool_blocks is not None:
        num_blocks = s.pool_blocks
    else:
        num_blocks = max(1, int(math.ceil(needed * (1.0 + s.pool_slack))))
    assert num_blocks >= needed, (num_blocks, needed)
    width = max(_table_width(s), max(nb) if nb else 1)
    perm = torch.randperm(num_blocks, generator=gen)
    tables = torch.full((s.num_seqs, width), -1, dtype=torch.int32)
    nxt = 0
    for i, n in enumerate(nb):
        tables[i, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    lens_t = torch.tensor(lens, dtype=torch.int32)
    lay = Layout(s, num_blocks, lens_t, tables, lens_t.clone(), tables.clone())
    if s.append:
        # The step's new token is the last one of each sequence: it is not in
        # the pool before the step and lands at position L-1.
        assert min(lens) >= 1
        lay.fill_lens = lens_t - 1
        pos = lens_t.to(torch.int64) - 1
        blk = tables.to(torch.int64).gather(1, (pos // B).unsqueeze(1)).squeeze(1)
        lay.slot_mapping = blk * B + pos % B
        lay.cow_pairs = torch.zeros((0, 2), dtype=torch.int32)
    return lay


# ---------------------------------------------------------------------------
# Prefix-sharing workload: an operation script for a block allocator.
# ---------------------------------------------------------------------------

PREFIX_HOLDER = 1_000_000


@dataclasses.dataclass
class PrefixScript:
    spec: Spec
    num_blocks: int
    free_order: List[int]  # initial free-list order (a seeded permutation)
    setup: List[Tuple]  # ops run before the step
    step_appends: List[int]  # sequence ids appended once each, in order, by the step
    seqs: List[int]  # decode batch order
    final_lens: List[int]


def prefix_script(s: Spec, seed: Optional[int] = None) -> PrefixScript:
    """Ops that build the shared-prefix layout through any block allocator.

    A holder sequence allocates the P-token prefix; every request forks it
    (refcount on each prefix block), the holder is freed, each request appends
    its private suffix up to one token before its final length, request 0 is
    forked into the last request, and the step appends one token to every
    request. Request 0's last block is partially filled and shared with its
    fork when the step appends to it, so that append copies the block first.
    """
    assert s.lens[0] == "prefix"
    _, P, lo, hi = s.lens
    gen = torch.Generator().manual_seed(s.seed if seed is None else seed)
    B = s.block_size
    n_req = s.num_seqs
    suffix = _uniform_ints(gen, n_req - 1, lo, hi)
    # request 0 must end the pre-step state inside a block (not on a boundary)
    while (P + suffix[0] - 1) % B == 0:
        suffix[0] = _uniform_ints(gen, 1, lo, hi)[0]
    final = [P + x for x in suffix] + [P + suffix[0]]
    needed = -(-P // B) + sum(-(-(L - P) // B) for L in final[:-1]) + 1
    num_blocks = int(math.ceil(needed * (1.0 + s.pool_slack)))
    order = torch.randperm(num_blocks, generator=gen).tolist()
    setup: List[Tuple] = [("allocate", PREFIX_HOLDER, P)]
    for r in range(n_req - 1):
        setup.append(("fork", PREFIX_HOLDER, r))
    setup.append(("free", PREFIX_HOLDER))
    for r in range(n_req - 1):
        setup.append(("append", r, final[r] - 1 - P))
    setup.append(("fork", 0, n_req - 1))
    return PrefixScript(s, num_blocks, order, setup, list(range(n_req)), list(range(n_req)), final)


# ---------------------------------------------------------------------------
# Values
# ---------------------------------------------------------------------------

def _randn(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _used_slot_mask(num_blocks: int, block_size: int, tables: torch.Tensor, lens: torch.Tensor) -> torch.Tensor:
    """bool [NB, B]: slot holds a token of some sequence."""
    fill = torch.zeros(num_blocks, dtype=torch.int64)
    B = block_size
    for i in range(tables.shape[0]):
        L = int(lens[i])
        n = -(-L // B)
        for b in range(n):
            blk = int(tables[i, b])
            fill[blk] = max(int(fill[blk]), min(B, L - b * B))
    return torch.arange(B).unsqueeze(0) < fill.unsqueeze(1)


@dataclasses.dataclass
class Tensors:
    q: torch.Tensor  # [S, Hq, D] q dtype
    k_cache: torch.Tensor  # [NB, Hk, B, D] cache dtype (uint8 codes for fp8)
    v_cache: torch.Tensor
    k_new: Optional[torch.Tensor] = None  # [S, Hk, D] q dtype (append only)
    v_new: Optional[torch.Tensor] = None
    k_scale: Optional[torch.Tensor] = None  # fp32 [Hk] (fp8 only)
    v_scale: Optional[torch.Tensor] = None


def make_tensors(s: Spec, num_blocks: int, fill_tables: torch.Tensor, fill_lens: torch.Tensor,
                 device="cpu", seed: Optional[int] = None, poison: bool = True,
                 chunk_blocks: int = 4096) -> Tensors:
    """Draw q, the pool contents and the step's new K/V for a layout."""
    seed = (s.seed if seed is None else seed) + 0x1234
    gen = torch.Generator(device=device).manual_seed(seed)
    S, Hq, Hk, D, B = s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size
    qdt = TORCH_DTYPES[s.q_dtype]
    q = _randn((S, Hq, D), gen, device).to(qdt)
    k_new = v_new = None
    if s.append:
        k_new = _randn((S, Hk, D), gen, device).to(qdt)
        v_new = _randn((S, Hk, D), gen, device).to(qdt)
    used = _used_slot_mask(num_blocks, B, fill_tables, fill_lens).to(device)
    fp8 = s.cache_dtype == "fp8_e4m3"
    cdt = torch.uint8 if fp8 else TORCH_DTYPES[s.cache_dtype]
    caches = []
    scales = []
    for which in range(2):
        pool = torch.empty((num_blocks, Hk, B, D), dtype=cdt, device=device)
        if fp8:
            # Scale so the largest stored value of each head maps to the top
            # of the e4m3 range; values are N(0,1) quantised by torch's own
            # float8_e4m3fn cast (a library routine, not the method's encoder).
            amax = torch.zeros(Hk, dtype=torch.float32, device=device)
            parts = []
            for b0 in range(0, num_blocks, chunk_blocks):
                x = _randn((min(chunk_blocks, num_blocks - b0), Hk, B, D), gen, device)
                m = used[b0:b0 + x.shape[0]].unsqueeze(1).unsqueeze(-1)
                amax = torch.maximum(amax, (x.abs() * m).amax(dim=(0, 2, 3)))
                parts.append(x)
            new = k_new if which == 0 else v_new
            if new is not None:
                amax = torch.maximum(amax, new.float().abs().amax(dim=(0, 2)))
            scale = (amax / FP8_MAX).clamp_min(1e-12)
            for b0, x in zip(range(0, num_blocks, chunk_blocks), parts):
                codes = (x / scale.view(1, Hk, 1, 1)).to(torch.float8_e4m3fn).view(torch.uint8)
                pool[b0:b0 + x.shape[0]] = codes
            scales.append(scale)
        else:
            for b0 in range(0, num_blocks, chunk_blocks):
                n = min(chunk_blocks, num_blocks - b0)
                pool[b0:b0 + n] = _randn((n, Hk, B, D), gen, device).to(cdt)
        if poison:
            mask = (~used).unsqueeze(1).unsqueeze(-1).expand(num_blocks, Hk, B, D)
            if fp8:
                pool.masked_fill_(mask, FP8_NAN_CODE)
            else:
                pool.masked_fill_(mask, float("nan"))
        caches.append(pool)
    t = Tensors(q, caches[0], caches[1], k_new, v_new)
    if fp8:
        t.k_scale, t.v_scale = scales
    return t


def scaled_down(s: Spec, num_seqs: int, len_cap: int, **kw) -> Spec:
    """A small version of a workload with the same structure (for full parity)."""
    kind = s.lens[0]
    if kind == "fixed":
        lens = ("fixed", [min(L, len_cap) for L in s.lens[1][:num_seqs]])
    elif kind == "uniform":
        lens = ("uniform", min(s.lens[1], len_cap // 2), min(s.lens[2], len_cap))
    elif kind == "skewed":
        n_long = max(1, num_seqs // 16)
        lens = ("skewed", n_long, len_cap // 2, len_cap, num_seqs - n_long,
                max(1, min(s.lens[5], len_cap // 16)), max(2, min(s.lens[6], len_cap // 8)))
    elif kind == "prefix":
        lens = ("prefix", min(s.lens[1], len_cap // 2), 1, max(2, len_cap // 4))
    else:
        raise ValueError(kind)
    return s.replace(num_seqs=num_seqs, lens=lens, table_width=None, **kw)

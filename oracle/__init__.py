"""CPU oracle for the paged-KV decode path. TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct numpy code in fp64, written from the pages
"KV-Cache Management and PagedAttention" (adversariallm.ai),
"PagedAttention and KV Cache Management" (blog.sejan.dev) and
"Managing the KV cache" (xavier-ramirez.com). Each function cites the passage
it follows.

Only `tests/`, `__graft_entry__.smoke()` and the `cpu_baseline` leg of
`bench.py` (plus its `--impl reference` arm) may import this package. The
product (`paged_kv_cache_453_b200`) never imports, links or runs it, and this
package imports nothing from the product; the two share no code. Inputs come
from the seeded generators in `workloads`, which hold none of the method's
arithmetic.

Parity status of each function (how it is pinned, in tests/test_oracle_*.py):
  numerics.decode_e4m3 / encode_e4m3   pinned: format constants, exhaustive
                                       round trip, tie and saturation cases,
                                       torch's float8_e4m3fn cast
  numerics.widen                       pinned: numpy float16, known bf16 bits
  attention.paged_decode               pinned: brute-force contiguous attention
                                       (pure-Python loops), 1-token context,
                                       q = 0 mean, two-token closed form, GQA
                                       head map, placement permutation, shared
                                       prefix = duplicated prefix, NaN slack
  cache_ops.reshape_and_cache(_fp8)    pinned: hand-placed slots, skip of
                                       negative slots
  cache_ops.copy_blocks                pinned: hand-built pool
  allocator.BlockAllocator             pinned: the printed allocator demo of
                                       "Hands-On Implementation", invariants
  sizing.kv_bytes                      pinned: the 13B and Llama-3-70B worked
                                       numbers and the 25-token prompt example
"""
from . import numerics, attention, cache_ops, allocator, sizing  # noqa: F401
from .numerics import widen, decode_e4m3, encode_e4m3  # noqa: F401
from .attention import paged_decode, gather_sequence  # noqa: F401
from .cache_ops import reshape_and_cache, reshape_and_cache_fp8, copy_blocks  # noqa: F401
from .allocator import BlockAllocator, AllocError  # noqa: F401

"""paged_attn_decode_noalloc: decode for callers that cannot allocate device
memory when they call (an engine that gave nearly all of HBM to its own
KV-block pool at start-up, or a latency-critical caller that cannot take the
device synchronisation cudaMalloc brings). Its split-KV scratch is a static
device array of the library, shared by every call on the device.

Checked through the C ABI against the regular entry points, within the
decode tolerances, on consecutive calls (so each call runs on the scratch the
previous call left behind). Collected last on purpose.
"""
import pytest
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from gpu_cases import TOL, decode_case, run_decode, max_err, check_no_device_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def setup():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_453_b200.build import build
    build()


def _noalloc(s, lay, t):
    out = torch.full_like(t.q, float("nan"))
    P.paged_attn_decode_noalloc(t.q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(),
                                s.num_kv_heads, s.scale, s.block_size, out, t.k_scale, t.v_scale)
    return out


def test_noalloc_matches_regular_entry_on_consecutive_calls():
    cases = [decode_case(W.scaled_down(W.spec("llama3_8b"), 16, 2000)),
             decode_case(W.scaled_down(W.spec("long_skewed"), 16, 3000, cache_dtype="fp8_e4m3")),
             decode_case(W.spec("llama3_70b").replace(num_seqs=3, lens=("fixed", [1, 4000, 0]),
                                                       table_width=None))]
    refs = [run_decode(*c).float().cpu().numpy() for c in cases]
    torch.cuda.synchronize()
    # Two rounds of back-to-back calls: every call starts from the scratch
    # contents of a different shape.
    for _ in range(2):
        outs = [_noalloc(*c) for c in cases]
        torch.cuda.synchronize()
        for (s, _, _), out, ref in zip(cases, outs, refs):
            assert max_err(out, ref) <= TOL[s.cache_dtype], s.name
    check_no_device_error()

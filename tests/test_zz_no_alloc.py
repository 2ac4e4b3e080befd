"""paged_attn_decode_noalloc: decode for callers that cannot allocate device
memory when they call (an engine that gave nearly all of HBM to its own
KV-block pool at start-up, or a latency-critical caller that cannot take the
device synchronisation cudaMalloc brings). Its split-KV scratch is a static
device array of the library, shared by every call on the device.

Checked through the C ABI against the regular entry points, within the
decode tolerances, on consecutive calls (so each call runs on the scratch the
previous call left behind), including a shape whose default scratch does not
fit the array (the call keeps fewer steal slots); the device's free memory is
the same before and after the calls. Collected last on purpose.
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


def _noalloc_into(s, lay, t, out, tables, lens):
    P.paged_attn_decode_noalloc(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale,
                                s.block_size, out, t.k_scale, t.v_scale)


def test_noalloc_matches_regular_entry_on_consecutive_calls():
    # The g = 8 fp8 shape needs more than the static array for the default
    # split-KV scratch (the regular entry's workspace query says so), so the
    # call runs with fewer steal slots: that path is compared too.
    g8_fp8 = W.scaled_down(W.spec("llama3_70b"), 8, 3000, cache_dtype="fp8_e4m3").replace(
        lens=("uniform", 1000, 3000))
    dev = torch.cuda.current_device()
    assert P.workspace_bytes(64, 8, 128, 16, P.PKV_FP8_E4M3, dev) > P.NOALLOC_SCRATCH_BYTES
    cases = [decode_case(W.scaled_down(W.spec("llama3_8b"), 16, 2000)),
             decode_case(W.scaled_down(W.spec("long_skewed"), 16, 3000, cache_dtype="fp8_e4m3")),
             decode_case(W.spec("llama3_70b").replace(num_seqs=3, lens=("fixed", [1, 4000, 0]),
                                                       table_width=None)),
             decode_case(g8_fp8)]
    refs = [run_decode(*c).float().cpu().numpy() for c in cases]
    torch.cuda.synchronize()
    # Outputs and index tensors made before the calls, so that nothing below
    # asks torch's allocator for memory either.
    args = [(torch.full_like(t.q, float("nan")), lay.tables.cuda(), lay.lens.cuda()) for _, lay, t in cases]
    for c, a in zip(cases, args):      # first call per device looks the array up
        _noalloc_into(*c, *a)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info(dev)[0]
    # Two rounds of back-to-back calls: every call starts from the scratch
    # contents of a different shape.
    for _ in range(2):
        for c, a in zip(cases, args):
            a[0].fill_(float("nan"))
            _noalloc_into(*c, *a)
        torch.cuda.synchronize()
        outs = [a[0].cpu() for a in args]     # host copies: no device memory asked for
        for (s, _, _), out, ref in zip(cases, outs, refs):
            assert max_err(out, ref) <= TOL[s.cache_dtype], s.name
    assert torch.cuda.mem_get_info(dev)[0] == free_before, "the no-allocation entry point allocated"
    check_no_device_error()

"""The bench's packed step inputs (host side): one buffer holds every input of
a step at 16-byte aligned offsets, and the views read back exactly what was
packed (so one copy moves a whole step's inputs)."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_step_buffers_round_trip_and_alignment():
    g = torch.Generator().manual_seed(3)
    parts = {"q": torch.randn(3, 5, 8, generator=g).to(torch.bfloat16),
             "slots": torch.randint(-5, 1000, (3,), generator=g, dtype=torch.int64),
             "tables": torch.randint(-1, 100, (3, 7), generator=g, dtype=torch.int32),
             "lens": torch.randint(0, 90, (3,), generator=g, dtype=torch.int32),
             "empty": torch.zeros((0, 2), dtype=torch.int32),
             "codes": torch.randint(0, 256, (3, 2, 5), generator=g, dtype=torch.uint8)}
    b = bench.StepBuffers(parts, "cpu", pin=False)
    used = sum(x.numel() * x.element_size() for x in parts.values())
    assert used <= b.nbytes < used + bench.StepBuffers.ALIGN * len(parts)
    for k, x in parts.items():
        v = b.d(k)
        assert v.dtype == x.dtype and tuple(v.shape) == tuple(x.shape)
        assert torch.equal(v, x), k
        assert (v.data_ptr() - b.dev.data_ptr()) % bench.StepBuffers.ALIGN == 0, k


def test_prepared_calls_keep_their_tensors_alive():
    # A prepared call holds raw device pointers; it must also hold the tensors
    # (a temporary such as tables.cuda() passed inline would otherwise be freed
    # and its memory reused under the call). Checked on CPU with the
    # constructor's bookkeeping only: no device call is made.
    import gc
    import weakref
    import torch
    import paged_kv_cache_453_b200 as P

    class T(torch.Tensor):  # a tensor subclass can be weakly referenced
        pass

    x = torch.zeros(4).as_subclass(T)
    ref = weakref.ref(x)
    call = P.Prepared("noop", lambda *a: 0, (), (None, (x,)), stream=0)  # stream 0: no CUDA query
    del x
    gc.collect()
    assert ref() is not None, "Prepared dropped a tensor it was built from"
    del call
    gc.collect()
    assert ref() is None


def test_prefill_roofline_takes_the_binding_bound():
    # 16 new tokens x 4 heads on the llama3_8b batch: ~40 GFLOP against
    # ~648 MB, so the bytes at the HBM peak take longer than the FLOPs at the
    # tensor peak; at 512 new tokens the MMAs bind.
    hbm, tensor = (6650.0, "fallback"), (1590.0, "fallback")
    r = bench.prefill_roofline(40.3e9, 648e6, 132e-6, tensor, hbm)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - 648e6 / 132e-6 / 1e9 / 6650.0) < 1e-12
    assert abs(r["tensor_frac"] - 40.3e9 / 132e-6 / 1e12 / 1590.0) < 1e-12
    r = bench.prefill_roofline(1.29e12, 1.1e9, 1.45e-3, tensor, hbm)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - 1.29e12 / 1.45e-3 / 1e12 / 1590.0) < 1e-12
    assert r["hbm_frac"] < r["frac"]

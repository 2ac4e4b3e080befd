"""Shared helpers of the GPU parity tests: build a decode case on the device,
run the library, run the oracle on the same inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_453_b200 as P
import workloads as W
from oracle.attention import paged_decode
from oracle_io import raw

# Maximum absolute error against the fp64 oracle, by the cache type's output.
TOL = {"f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2}


def decode_case(spec: W.Spec, device="cuda", seed=None):
    """(layout, tensors) with every token already in the pool (no append)."""
    s = spec.replace(append=False)
    lay = W.make_layout(s, seed=seed)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device=device, seed=seed)
    return s, lay, t


def run_decode(s: W.Spec, lay: W.Layout, t: W.Tensors, out=None, workspace=None):
    dev = t.q.device
    tables = lay.tables.to(dev)
    lens = lay.lens.to(dev)
    if out is None:
        out = torch.full_like(t.q, float("nan"))
    if workspace is not None:
        P.paged_attn_decode_ex(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale,
                               s.block_size, out, workspace, t.k_scale, t.v_scale)
    elif s.cache_dtype == "fp8_e4m3":
        P.paged_attn_decode_fp8(t.q, t.k_cache, t.v_cache, t.k_scale, t.v_scale, tables, lens,
                                s.num_kv_heads, s.scale, s.block_size, out)
    else:
        P.paged_attn_decode(t.q, t.k_cache, t.v_cache, tables, lens, s.num_kv_heads, s.scale,
                            s.block_size, out)
    return out


def oracle_decode(s: W.Spec, lay: W.Layout, t: W.Tensors, seqs=None) -> np.ndarray:
    ks = None if t.k_scale is None else t.k_scale.cpu().numpy()
    vs = None if t.v_scale is None else t.v_scale.cpu().numpy()
    return paged_decode(raw(t.q), raw(t.k_cache), raw(t.v_cache), lay.tables.numpy(),
                        lay.lens.numpy(), s.scale, s.block_size, s.q_dtype, s.cache_dtype,
                        k_scale=ks, v_scale=vs, seqs=seqs)


def max_err(out: torch.Tensor, ref: np.ndarray, seqs=None) -> float:
    o = out.float().cpu().numpy().astype(np.float64)
    if seqs is not None:
        o, ref = o[list(seqs)], ref[list(seqs)]
    assert np.all(np.isfinite(o)), "non-finite output"
    return float(np.max(np.abs(o - ref))) if o.size else 0.0


def check_no_device_error():
    st = P.device_error(torch.cuda.current_device())
    assert st == P.PKV_OK, P.status_string(st)

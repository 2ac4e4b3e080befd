"""Benchmark of the paged-KV decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--block-size B] [--cache-dtype bf16|f16|fp8_e4m3]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = the whole hot path over one batch: reshape_and_cache of the step's
new tokens (one per sequence), then paged_attn_decode (decode kernel + merge
kernel) over every sequence, all through the C ABI. Default workload: the
Llama-3-8B-shaped decode (64 sequences, lens ~ U[512, 4096], 32 q / 8 kv
heads, D = 128, B = 16, bf16; about 604 MB of K/V, larger than the 126 MB L2,
so no flush is needed between steps).

metric / value: K+V bytes the decode reads per step (sum of L_s * 2 * Hk * D *
elem) divided by the device time of a step, in GB/s, summed over ranks. With
N > 1 each rank runs its own replica (the path has no exchange step), so
scaling is weak. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on bounded samples of the same
workload on the host cores (the only other place this file runs oracle/).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "paged decode attention HBM GB/s (KV bytes read/s) and % of B200 peak; seqs/s"
UNIT = "GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--cache-dtype", default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--op", default="decode", choices=["decode", "swap", "prefill"],
                    help="swap: preemption by swapping (blocks to page-locked host memory and back); "
                         "prefill: causal attention of --q-tokens new tokens per sequence")
    ap.add_argument("--q-tokens", type=int, default=4,
                    help="new tokens per sequence for --op prefill (4: speculative verification)")
    ap.add_argument("--no-cascade", action="store_true",
                    help="decode a shared-prefix workload with the plain decode")
    return ap.parse_args()


def workload_spec(a) -> W.Spec:
    over = {}
    if a.block_size:
        over["block_size"] = a.block_size
    if a.cache_dtype:
        over["cache_dtype"] = a.cache_dtype
        if a.cache_dtype in ("f16", "bf16"):
            over["q_dtype"] = a.cache_dtype
    return W.spec(a.workload, **over).replace(append=True)


def prefix_layout(s: W.Spec, allocator_cls) -> W.Layout:
    """The shared-prefix layout, built by a block allocator from the
    workload's operation script; the step's appends (one copy-on-write among
    them) give the slot mapping and the block-copy pairs. The timed arm uses
    the library's allocator, the reference arm the oracle's."""
    sc = W.prefix_script(s)
    a = allocator_cls(sc.num_blocks, s.block_size, sc.free_order)
    a.run(sc.setup)
    width = -(-max(sc.final_lens) // s.block_size)

    def tables():
        t = torch.full((len(sc.seqs), width), -1, dtype=torch.int32)
        for i, r in enumerate(sc.seqs):
            row = a.table(r)
            t[i, :len(row)] = torch.tensor(row, dtype=torch.int32)
        return t

    fill_tables = tables()
    step = [a.append_slot(r) for r in sc.step_appends]
    lens = torch.tensor(sc.final_lens, dtype=torch.int32)
    lay = W.Layout(s, sc.num_blocks, lens, tables(), lens - 1, fill_tables)
    lay.slot_mapping = torch.tensor([x[0] for x in step], dtype=torch.int64)
    lay.cow_pairs = torch.tensor([[x[1], x[2]] for x in step if x[1] >= 0], dtype=torch.int32).reshape(-1, 2)
    return lay


def unique_kv_bytes(s: W.Spec, lay) -> int:
    """K+V bytes of the distinct stored tokens the decode reads (a block shared
    by several tables counts once, with its longest use)."""
    B = s.block_size
    fill = {}
    for row, L in zip(lay.tables.tolist(), lay.lens.tolist()):
        for b in range(-(-L // B)):
            fill[row[b]] = max(fill.get(row[b], 0), min(B, L - b * B))
    return sum(fill.values()) * 2 * s.num_kv_heads * s.head_dim * s.cache_elem_bytes


def config_of(s: W.Spec, lay, kv_bytes: int) -> dict:
    return {"workload": W.describe(s), "num_seqs": s.num_seqs,
            "num_q_heads": s.num_q_heads, "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim,
            "block_size": s.block_size, "cache_dtype": s.cache_dtype,
            "tokens": int(lay.lens.sum()), "kv_bytes_per_step": kv_bytes,
            "l2": "inputs larger than L2 (K/V pool > 126 MB), no flush",
            "step": "reshape_and_cache(new token per seq) + paged_attn_decode"}


def kv_bytes_of(s: W.Spec, lens) -> int:
    return int(sum(int(L) for L in lens)) * 2 * s.num_kv_heads * s.head_dim * s.cache_elem_bytes


def decode_alg_bytes(s: W.Spec, lens) -> int:
    """Algorithmic bytes of one decode: K+V of every stored token, q and out,
    the used block-table entries and the lengths (plus fp8 scales)."""
    B = s.block_size
    kv = kv_bytes_of(s, lens)
    qo = 2 * s.num_seqs * s.num_q_heads * s.head_dim * 2
    tab = sum(-(-int(L) // B) for L in lens) * 4 + 4 * s.num_seqs
    sc = 2 * s.num_kv_heads * 4 if s.cache_dtype == "fp8_e4m3" else 0
    return kv + qo + tab + sc


class StepBuffers:
    """One step's inputs packed into a single device buffer with a
    page-locked host twin (16-byte aligned pieces), so the step's inputs
    cross to the device in one copy."""

    ALIGN = 16

    def __init__(self, host_tensors: dict, device, pin: bool = True):
        self.meta = {}
        off = 0
        for k, x in host_tensors.items():
            off = -(-off // self.ALIGN) * self.ALIGN
            nb = x.numel() * x.element_size()
            self.meta[k] = (off, nb, x.dtype, tuple(x.shape))
            off += nb
        self.nbytes = max(self.ALIGN, -(-off // self.ALIGN) * self.ALIGN)
        self.host = torch.zeros(self.nbytes, dtype=torch.uint8, pin_memory=pin)
        self.dev = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        for k, x in host_tensors.items():
            self._view(self.host, k).copy_(x.contiguous())
        self.dev.copy_(self.host)

    def _view(self, buf, k):
        off, nb, dt, sh = self.meta[k]
        return buf[off:off + nb].view(dt).view(sh)

    def d(self, k):
        """The device view of input k."""
        return self._view(self.dev, k)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device: int):
        self.lines = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", ident], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        sms, maxs, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sms.append(float(parts[0]))
                maxs.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


# ---------------------------------------------------------------------------
# roofline helpers
# ---------------------------------------------------------------------------

def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_peak_bf16():
    """Dense bf16 tensor peak (burst: a kernel timed alone), TFLOP/s."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("decode.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_453_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(s: W.Spec):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source and this workload."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    key = f"{s.name}/{s.cache_dtype}/B{s.block_size}"
    e = d.get(key)
    if not e or e.get("kernel_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


def prefill_traffic(s: W.Spec, q_tokens: int, kernel: str):
    """DRAM bytes per tensor-core multi-token launch from the committed ncu
    summary, if it was taken on the current kernel source, this workload
    and this kernel."""
    p = os.path.join(ROOT, "profiles", "prefill_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for name in ("prefill.cuh", "prefill_tc.cuh", "prefill_tc2.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_453_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    e = d.get(f"{s.name}/{s.cache_dtype}/B{s.block_size}/q{q_tokens}")
    if not e or e.get("kernel_sha") != h.hexdigest()[:16] or e.get("kernel") != kernel:
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def _host_cores() -> int:
    """Cores this process may run on (the host's usable cores)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _blas_threads() -> int:
    """Threads the oracle's BLAS calls run on (the cores it actually uses)."""
    try:
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def _host_inputs(s: W.Spec, lay, t):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_io import raw
    ks = None if t.k_scale is None else t.k_scale.cpu().numpy()
    vs = None if t.v_scale is None else t.v_scale.cpu().numpy()
    return raw(t.q), raw(t.k_cache), raw(t.v_cache), lay.tables.numpy(), lay.lens.numpy(), ks, vs


def oracle_rate(s: W.Spec, host, seqs) -> tuple:
    """(seconds, KV bytes) of the oracle over the given sequences."""
    from oracle.attention import paged_decode
    q, kp, vp, tab, lens, ks, vs = host
    t0 = time.perf_counter()
    paged_decode(q, kp, vp, tab, lens, s.scale, s.block_size, s.q_dtype, s.cache_dtype, k_scale=ks,
                 v_scale=vs, seqs=seqs)
    dt = time.perf_counter() - t0
    return dt, kv_bytes_of(s, [lens[i] for i in seqs])


def cpu_baseline(s: W.Spec, host, budget_s: float) -> dict:
    """The oracle over the workload's sequences in order, cycling through them
    until about budget_s seconds of CPU work have been done."""
    S = s.num_seqs
    tot_t, tot_b, done = 0.0, 0, 0
    while tot_t < budget_s:
        dt, nb = oracle_rate(s, host, [done % S])
        tot_t += dt
        tot_b += nb
        done += 1
    return {"value": tot_b / tot_t / 1e9, "unit": UNIT, "cores": _blas_threads(), "host_cores": _host_cores(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle, one sequence per call, cycling over the workload's {S} "
                      f"sequences: {done} sequence decodes ({tot_b} K/V bytes) in {tot_t:.1f} s",
            "seqs_per_s": done / tot_t}


# ---------------------------------------------------------------------------

def dist_setup(a):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return ws, rank, local, pg


def max_over_ranks(vals, dist, device):
    """Each value's maximum over all ranks (a timing: the slowest rank sets
    the job's time). Without a process group the values come back as they are."""
    if not dist:
        return [float(v) for v in vals]
    tt = torch.tensor([float(v) for v in vals], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return [float(x) for x in tt]


def run_reference(a, s: W.Spec, ws: int, rank: int):
    if rank != 0:
        return
    if s.lens[0] == "prefix":
        from oracle.allocator import BlockAllocator
        lay = prefix_layout(s, BlockAllocator)
    else:
        lay = W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device="cpu")
    host = _host_inputs(s, lay, t)
    # Size each step's sample so that warm-up + steps take about 2 minutes.
    dt1, _ = oracle_rate(s, host, [0])
    per_step = 120.0 / max(1, a.steps + a.warmup)
    frac = min(1.0, per_step / max(dt1, 1e-6))
    S = s.num_seqs
    order = list(range(S))

    def step(i):
        seq = order[i % S]
        if frac >= 1.0:
            return oracle_rate(s, host, [seq])
        # part of one sequence: its first ceil(frac * L) tokens
        L = int(host[4][seq])
        n = max(1, int(math.ceil(frac * L)))
        lens = host[4].copy()
        lens[seq] = n
        h2 = host[:4] + (lens,) + host[5:]
        return oracle_rate(s, h2, [seq])

    for i in range(a.warmup):
        step(i)
    tot_t, tot_b = 0.0, 0
    for i in range(a.steps):
        dt, nb = step(a.warmup + i)
        tot_t += dt
        tot_b += nb
    value = tot_b / tot_t / 1e9
    sample = (f"each step: fp64 numpy oracle on one sequence of the workload"
              + ("" if frac >= 1.0 else f", its first {frac:.3%} of tokens"))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * tot_t / max(1, a.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(s, lay, kv_bytes_of(s, lay.lens.tolist())) | {"parallelism": f"replicas x{ws}"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "host_cores": _host_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def run_swap(a, s: W.Spec):
    """Swap a quarter of the workload's sequences out to page-locked host
    memory and back into other blocks, per step; compared with torch's own
    device<->pinned-host copies of the same bytes (the host link's rate)."""
    import paged_kv_cache_453_b200 as P
    from paged_kv_cache_453_b200.build import build
    build()
    torch.cuda.set_device(0)
    lay = W.make_layout(s.replace(append=False))
    t = W.make_tensors(s.replace(append=False), lay.num_blocks, lay.tables, lay.lens, device="cuda:0")
    n_seq = max(1, s.num_seqs // 4)
    blocks = [int(b) for i in range(n_seq) for b in lay.tables[i, :-(-int(lay.lens[i]) // s.block_size)]]
    used = set(int(b) for b in lay.tables.flatten() if b >= 0)
    spare = [b for b in range(lay.num_blocks) if b not in used]
    dst = (spare + blocks)[:len(blocks)]  # into free blocks first (same data if they run out)
    src_t = torch.tensor(blocks, dtype=torch.int32, device="cuda:0")
    dst_t = torch.tensor(dst, dtype=torch.int32, device="cuda:0")
    rec = P.swap_record_bytes(t.k_cache)
    nbytes = len(blocks) * rec
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dev_buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda:0")

    def timed(fn, K):
        for _ in range(max(3, a.warmup)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K / 1e3

    K = max(1, min(a.steps, 200))
    clocks = ClockSampler(0)
    t_out = timed(lambda: P.swap_out_blocks(t.k_cache, t.v_cache, src_t, host), K)
    t_in = timed(lambda: P.swap_in_blocks(host, dst_t, t.k_cache, t.v_cache), K)
    clk = clocks.stop()
    t_d2h = timed(lambda: host.copy_(dev_buf, non_blocking=True), K)
    t_h2d = timed(lambda: dev_buf.copy_(host, non_blocking=True), K)
    st = P.device_error(0)
    if st != P.PKV_OK:
        raise SystemExit(f"device check failed: {P.status_string(st)}")
    link = 2 * nbytes / (t_d2h + t_h2d) / 1e9
    value = 2 * nbytes / (t_out + t_in) / 1e9
    print(json.dumps({
        "metric": "preemption swap GB/s (K+V block bytes out to page-locked host memory and back)",
        "value": value, "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": max(3, a.warmup),
        "ms_per_step": (t_out + t_in) * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": s.cache_dtype, "data": "synthetic",
        "config": {"workload": W.describe(s), "blocks_per_step": len(blocks), "bytes_each_way": nbytes,
                   "step": "swap_out_blocks then swap_in_blocks into other blocks"},
        "swap_out_gbs": nbytes / t_out / 1e9, "swap_in_gbs": nbytes / t_in / 1e9,
        "roofline": {"bound": "host link", "achieved": value, "peak": link, "unit": "GB/s", "frac": value / link,
                     "peak_source": "torch device<->pinned-host copies of the same bytes in this run",
                     "d2h_gbs": nbytes / t_d2h / 1e9, "h2d_gbs": nbytes / t_h2d / 1e9, "traffic": None},
        "clocks": clk, "gpu_launches": 2 * K,
    }))


def prefill_roofline(flops: float, alg_bytes: float, sec: float, tensor_peak, hbm_peak) -> dict:
    """Roofline of a tensor-core multi-token launch: bound by whichever of
    its FLOPs at the tensor peak and its algorithmic bytes at the HBM peak
    takes longer (few new tokens per sequence: HBM; many: the MMAs). The
    other side's fraction is reported beside it."""
    (tp, tsrc), (hp, hsrc) = tensor_peak, hbm_peak
    t_tensor = flops / (tp * 1e12)
    t_hbm = alg_bytes / (hp * 1e9)
    f_tensor = flops / sec / 1e12 / tp
    f_hbm = alg_bytes / sec / 1e9 / hp
    if t_hbm >= t_tensor:
        return {"bound": "hbm", "achieved": alg_bytes / sec / 1e9, "peak": hp, "unit": "GB/s", "frac": f_hbm,
                "peak_source": hsrc, "tensor_frac": f_tensor, "tensor_peak": tp}
    return {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": tp, "unit": "TFLOP/s", "frac": f_tensor,
            "peak_source": tsrc + " (bf16 burst)", "hbm_frac": f_hbm, "hbm_peak": hp}


def run_prefill(a, s: W.Spec):
    """Causal attention of --q-tokens new tokens per sequence (the last ones of
    each context) over the workload's paged cache, inputs resident."""
    import paged_kv_cache_453_b200 as P
    from paged_kv_cache_453_b200.build import build
    build()
    torch.cuda.set_device(0)
    s = s.replace(append=False)
    lay = W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.tables, lay.lens, device="cuda:0")
    lens = lay.lens.tolist()
    nq = [min(a.q_tokens, L) for L in lens]
    q_start = torch.tensor([0] + list(np.cumsum(nq)), dtype=torch.int32)
    T = int(q_start[-1])
    g = torch.Generator(device="cuda:0").manual_seed(s.seed + 77)
    q = torch.randn((T, s.num_q_heads, s.head_dim), generator=g, device="cuda:0").to(t.q.dtype)
    out = torch.empty_like(q)
    call = P.prepare_prefill(q, t.k_cache, t.v_cache, lay.tables.cuda(), lay.lens.cuda(), q_start.cuda(),
                             max(nq), s.num_kv_heads, s.scale, s.block_size, out,
                             k_scale=t.k_scale, v_scale=t.v_scale)
    kv = kv_bytes_of(s, lens)
    alg = kv + 2 * T * s.num_q_heads * s.head_dim * 2 + sum(-(-L // s.block_size) for L in lens) * 4 + 8 * s.num_seqs
    keys = sum(sum(L - n + j + 1 for j in range(n)) for L, n in zip(lens, nq))
    flops = 4.0 * s.head_dim * s.num_q_heads * keys
    for _ in range(max(3, a.warmup)):
        call()
    torch.cuda.synchronize()
    K = a.steps
    clocks = ClockSampler(0)
    time.sleep(0.3 if clocks.proc else 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        call()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    st = P.device_error(0)
    if st != P.PKV_OK:
        raise SystemExit(f"device check failed: {P.status_string(st)}")
    sec = e0.elapsed_time(e1) / K / 1e3
    # tiles of 128 rows (new tokens x group heads) run on the tensor cores
    # from 64 rows (one tile per CTA up to 128 rows, two beyond):
    # that launch is bound by the MMAs, the others by the KV bytes
    g = s.num_q_heads // s.num_kv_heads
    cols = max(nq) * g
    tc = s.cache_dtype != "fp8_e4m3" and s.head_dim == 128 and cols >= 64 and s.scale > 0
    # kernels one call launches: the tensor-core kernel (after the one-CTA
    # longest-first ordering pass when 1 < S <= 1024 and the grid is more
    # than one wave), or the warp-MMA
    # kernel (plus its merge when the KV is cut into chunks)
    decode_step = max(nq) == 1 and T == s.num_seqs  # served by the decode kernels
    if decode_step:
        per_call = 2
    elif tc:
        rows = 256 if cols > 128 else 128  # query rows per CTA
        ctas = s.num_seqs * s.num_kv_heads * -(-cols // rows)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        per_call = 1 + (1 if 1 < s.num_seqs <= 1024 and ctas > sms else 0)
    else:
        ecols = 16 if cols <= 16 else 32 if cols <= 32 else 64
        ncc = -(-cols // ecols)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        per_call = 1 + (1 if s.num_seqs * s.num_kv_heads * ncc < 4 * sms and lay.tables.shape[1] > 32 else 0)
    if tc and not decode_step:
        kern = "prefill_tc2_kernel" if cols > 128 else "prefill_tc_kernel"
        roof = prefill_roofline(flops, alg, sec, measured_peak_bf16(), measured_peak_hbm())
        roof.update({"kernel": kern, "traffic": prefill_traffic(s, a.q_tokens, kern),
                     "alg_bytes_per_launch": alg, "flops_per_launch": flops})
    else:
        peak, src = measured_peak_hbm()
        roof = {"kernel": "decode_kernel + decode_merge_kernel" if decode_step else "prefill_kernel",
                "bound": "hbm", "achieved": alg / sec / 1e9, "peak": peak,
                "unit": "GB/s", "frac": alg / sec / 1e9 / peak, "peak_source": src, "traffic": None,
                "alg_bytes_per_launch": alg, "flops_per_launch": flops}
    print(json.dumps({
        "metric": "multi-token paged attention HBM GB/s (KV bytes read/s) and TFLOP/s",
        "value": kv / sec / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": max(3, a.warmup),
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": s.cache_dtype, "data": "synthetic",
        "config": {"workload": W.describe(s), "new_tokens_per_seq": a.q_tokens, "query_rows": T,
                   "kv_bytes": kv, "l2": "inputs larger than L2 (K/V pool > 126 MB), no flush"},
        "tflops": flops / sec / 1e12,
        "roofline": roof,
        "clocks": clk, "gpu_launches": per_call * K,
    }))


def main():
    a = parse()
    s = workload_spec(a)
    if a.op == "swap":
        run_swap(a, s)
        return
    if a.op == "prefill":
        run_prefill(a, s)
        return
    ws, rank, local, dist = dist_setup(a)
    if a.impl == "reference":
        run_reference(a, s, ws, rank)
        if dist:
            dist.destroy_process_group()
        return

    import paged_kv_cache_453_b200 as P
    from paged_kv_cache_453_b200.build import build
    if rank == 0:
        build()
    if dist:
        dist.barrier()
    dev = local
    torch.cuda.set_device(dev)
    shared = s.lens[0] == "prefix"
    lay = prefix_layout(s, P.BlockAllocator) if shared else W.make_layout(s)
    t = W.make_tensors(s, lay.num_blocks, lay.fill_tables, lay.fill_lens, device=f"cuda:{dev}")
    fp8 = s.cache_dtype == "fp8_e4m3"
    n_cow = int(lay.cow_pairs.shape[0])
    cascade = shared and not a.no_cascade
    groups = P.PrefixGroups(lay.tables, lay.lens, s.block_size, device="cpu") if cascade else None

    # A step's inputs (q, the new tokens' K/V and slots, the block tables and
    # lengths, copy-on-write pairs and prefix groups) sit packed in one device
    # buffer with a page-locked host twin: the end-to-end leg moves them with
    # one host->device copy per step. Two such buffers alternate there; the
    # device-timed leg runs on the first, its inputs resident.
    host_in = {"q": t.q.cpu(), "k_new": t.k_new.cpu(), "v_new": t.v_new.cpu(), "slots": lay.slot_mapping,
               "tables": lay.tables, "lens": lay.lens}
    if n_cow:
        host_in["cow_pairs"] = lay.cow_pairs
    if cascade:
        for k_ in ("prefix_blocks", "group_start", "members"):
            host_in[k_] = getattr(groups, k_)
    bufs = [StepBuffers(host_in, f"cuda:{dev}") for _ in range(2)]

    def step_calls(b: "StepBuffers"):
        out = torch.empty_like(t.q)
        write = P.prepare_reshape(b.d("k_new"), b.d("v_new"), t.k_cache, t.v_cache, b.d("slots"), t.k_scale,
                                  t.v_scale)
        if n_cow:
            cow = P.prepare_copy_blocks(t.k_cache, t.v_cache, b.d("cow_pairs"))

            def reshape():
                cow()
                write()
        else:
            reshape = write
        if cascade:
            g = P.PrefixGroups.on_device(b.d("prefix_blocks"), b.d("group_start"), b.d("members"),
                                         groups.num_groups, groups.max_group_size, groups.max_prefix_blocks)
            decode = P.prepare_decode_cascade(b.d("q"), t.k_cache, t.v_cache, b.d("tables"), b.d("lens"), g,
                                              s.num_kv_heads, s.scale, s.block_size, out,
                                              k_scale=t.k_scale, v_scale=t.v_scale)
        else:
            decode = P.prepare_decode(b.d("q"), t.k_cache, t.v_cache, b.d("tables"), b.d("lens"), s.num_kv_heads,
                                      s.scale, s.block_size, out, t.k_scale, t.v_scale)
        return reshape, decode, out

    calls = [step_calls(b) for b in bufs]
    reshape, decode, out = calls[0]
    lens_l = lay.lens.tolist()
    kv_bytes = kv_bytes_of(s, lens_l)
    alg = decode_alg_bytes(s, lens_l)
    extra = {}
    if shared:
        # Each request reads the shared prefix blocks again (mostly from L2);
        # the roofline counts every distinct stored byte once.
        uniq = unique_kv_bytes(s, lay)
        alg = alg - kv_bytes + uniq
        extra = {"kv_bytes_unique": uniq, "cow_copies_per_step": n_cow,
                 "alg_bytes": "roofline counts distinct stored K/V bytes; value counts K/V bytes per request",
                 "decode": "prefix-aware (shared prefix read once per group)" if cascade else "plain"}

    for _ in range(max(3, a.warmup)):
        for r_, d_, _ in calls:
            r_()
            d_()
    torch.cuda.synchronize()
    st = P.device_error(dev)
    if st != P.PKV_OK:
        raise SystemExit(f"device check failed during warm-up: {P.status_string(st)}")

    # Timed region 1: K whole steps back to back, events only at its ends (an
    # event between two kernels would keep the second from starting while the
    # first drains). Timed region 2: K decode calls back to back, for the
    # decode call's own duration (the roofline's denominator).
    K = a.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    time.sleep(0.3 if clocks.proc else 0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(K):
        reshape()
        decode()
    stop.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    d0.record()
    for i in range(K):
        decode()
    d1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(stop)
    dec_ms = d0.elapsed_time(d1) / K
    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], dist, f"cuda:{dev}")
    st = P.device_error(dev)
    if st != P.PKV_OK:
        raise SystemExit(f"device check failed: {P.status_string(st)}")
    step_s = elapsed_ms / 1e3 / K
    value = ws * kv_bytes / step_s / 1e9
    # [copy_blocks,] reshape_and_cache, decode, merge [, prefix pass, prefix merge];
    # both timed regions count
    launches_per_step = 3 + (1 if n_cow else 0) + (2 if cascade else 0)
    launches_per_call = 2 + (2 if cascade else 0)

    # ---- end to end through the public API: pinned host in, result out ----
    # Step i: one copy of its packed inputs host->device (buffer i % 2, on a
    # copy stream, once step i - 2 is done with that buffer), the step on the
    # compute stream, one copy of its output device->host (a second copy
    # stream). Step i + 1's inputs cross while step i runs.
    Ke = a.e2e_steps or max(3, min(K, 2000))
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    h_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = bufs[0].nbytes
    d2h = h_out[0].numel() * h_out[0].element_size()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(comp)
    for i in range(Ke):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])
            bufs[b].dev.copy_(bufs[b].host, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])
        calls[b][0]()
        calls[b][1]()
        ev_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            h_out[b].copy_(calls[b][2], non_blocking=True)
            ev_out[b].record(s_out)
    for b in range(2):
        comp.wait_event(ev_out[b])
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    (e2e_ms,) = max_over_ranks([e2e_ms], dist, f"cuda:{dev}")
    e2e_value = ws * kv_bytes / (e2e_ms / 1e3 / Ke) / 1e9
    st = P.device_error(dev)
    if st != P.PKV_OK:
        raise SystemExit(f"device check failed (end-to-end leg): {P.status_string(st)}")

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return
    peak, peak_src = measured_peak_hbm()
    achieved = alg / (dec_ms / 1e3) / 1e9
    cpu = None
    if ws == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(s, _host_inputs(s, lay, t), a.cpu_seconds)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K, "warmup": a.warmup,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3" if fp8 else s.cache_dtype, "data": "synthetic",
        "config": config_of(s, lay, kv_bytes) | {"parallelism": f"replicas x{ws}"} | extra,
        "seqs_per_s": ws * s.num_seqs / step_s,
        "pct_of_hbm_peak": 100.0 * value / ws / peak,
        "roofline": {"kernel": ("paged_attn_decode_cascade (decode, merge, prefix pass, prefix merge)"
                                if cascade else "paged_attn_decode (decode_kernel + decode_merge_kernel)"),
                     "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": profiled_traffic(s), "peak_source": peak_src,
                     "alg_bytes_per_launch": alg, "us_per_launch": dec_ms * 1e3,
                     "timing": "K decode calls back to back between two CUDA events on the launching stream"},
        "cpu_baseline": cpu,
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": Ke, "ms_per_step": e2e_ms / Ke,
                "copies": "per step one host->device copy of the packed inputs (page-locked) and one "
                          "device->host copy of the output; step i+1's inputs copied while step i runs "
                          "(two input buffers, two copy streams)"},
        "gpu_launches": (launches_per_step + launches_per_call) * K,
    }
    print(json.dumps(line))
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

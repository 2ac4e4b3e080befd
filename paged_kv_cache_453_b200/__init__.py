"""Python binding of libpagedkv.so: paged-KV decode attention on B200.

Argument marshalling only. Every device step runs in the library's sm_100a
kernels; torch supplies device memory and the current CUDA stream. There is
no fallback: if the native library is missing or a tensor is not on a CUDA
device, calls raise.

Device calls (names and argument order follow include/pagedkv.h):
    paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens,
                      num_kv_heads, scale, block_size, out)
    paged_attn_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables,
                          context_lens, num_kv_heads, scale, block_size, out)
    paged_attn_decode_ex(..., workspace=<uint8 cuda tensor>, flags=0 | PKV_DECODE_DETERMINISTIC)
    reshape_and_cache(k, v, k_cache, v_cache, slot_mapping)
    reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale)
    copy_blocks(k_cache, v_cache, pairs)
    device_error(device) -> status
Host allocator: BlockAllocator (pkv_alloc_* / pkv_seq_*).
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedkv.so")

PKV_F16, PKV_BF16, PKV_FP8_E4M3, PKV_I32, PKV_I64, PKV_F32 = 0, 1, 2, 3, 4, 5

PKV_OK = 0
PKV_ERR_INVALID_ARG = -1
PKV_ERR_UNSUPPORTED = -2
PKV_ERR_OOM = -3
PKV_ERR_UNKNOWN_SEQ = -4
PKV_ERR_EXISTS = -5
PKV_ERR_DOUBLE_FREE = -6
PKV_ERR_CUDA = -7
PKV_ERR_DEVICE_CHECK = -8
PKV_ERR_WORKSPACE = -9
PKV_ERR_SCRATCH_LIMIT = -10

NOALLOC_SCRATCH_BYTES = 16 << 20  # PKV_NOALLOC_SCRATCH_BYTES of include/pagedkv.h
PKV_DECODE_DETERMINISTIC = 1  # paged_attn_decode_ex flag: static split, identical bits per call

# Every symbol include/pagedkv.h declares.
EXPORTED = (
    "pkv_status_string", "pkv_version",
    "paged_attn_decode", "paged_attn_decode_fp8", "paged_attn_decode_workspace_bytes",
    "paged_attn_decode_ex", "paged_attn_decode_noalloc", "paged_attn_decode_cascade",
    "paged_attn_decode_cascade_fp8", "paged_attn_prefill_fp8", "reshape_and_cache", "reshape_and_cache_fp8", "copy_blocks",
    "pkv_device_error",
    "pkv_alloc_create", "pkv_alloc_destroy", "pkv_seq_allocate", "pkv_seq_append_slot",
    "pkv_seq_fork", "pkv_seq_free", "pkv_seq_num_tokens", "pkv_seq_block_table",
    "pkv_build_block_tables", "pkv_alloc_stats", "pkv_block_refcount", "pkv_prefix_groups",
    "swap_out_blocks", "swap_in_blocks", "pkv_seq_swap_out", "pkv_seq_swap_in",
    "pkv_alloc_utilisation", "pkv_seq_allocate_prefix", "pkv_cache_create", "pkv_cache_destroy",
    "pkv_cache_insert", "pkv_cache_match", "pkv_cache_evict", "pkv_cache_nodes", "paged_attn_prefill",
)


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class pkv_tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded native library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"native library {LIB_PATH} is missing; build it with "
                               "`python -m paged_kv_cache_453_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(pkv_tensor)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        sig = {
            "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "pkv_version": (ctypes.c_int, []),
            "paged_attn_decode": (ctypes.c_int, [P, P, P, P, P, ctypes.c_int, f32, ctypes.c_int, P, vp]),
            "paged_attn_decode_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, ctypes.c_int, f32,
                                                     ctypes.c_int, P, vp]),
            "paged_attn_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 6),
            "paged_attn_decode_ex": (ctypes.c_int, [P, P, P, P, P, P, P, ctypes.c_int, f32,
                                                    ctypes.c_int, P, vp, ctypes.c_size_t, ctypes.c_uint,
                                                    vp]),
            "paged_attn_decode_noalloc": (ctypes.c_int, [P, P, P, P, P, P, P, ctypes.c_int, f32,
                                                         ctypes.c_int, P, vp]),
            "reshape_and_cache": (ctypes.c_int, [P, P, P, P, P, vp]),
            "reshape_and_cache_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, vp]),
            "copy_blocks": (ctypes.c_int, [P, P, P, vp]),
            "pkv_device_error": (ctypes.c_int, [ctypes.c_int]),
            "pkv_alloc_create": (ctypes.c_int, [i32, i32, ctypes.POINTER(i32), ctypes.POINTER(vp)]),
            "pkv_alloc_destroy": (None, [vp]),
            "pkv_seq_allocate": (ctypes.c_int, [vp, i64, i32]),
            "pkv_seq_append_slot": (ctypes.c_int, [vp, i64, ctypes.POINTER(i64), ctypes.POINTER(i32),
                                                   ctypes.POINTER(i32)]),
            "pkv_seq_fork": (ctypes.c_int, [vp, i64, i64]),
            "pkv_seq_free": (ctypes.c_int, [vp, i64]),
            "pkv_seq_num_tokens": (i64, [vp, i64]),
            "pkv_seq_block_table": (ctypes.c_int, [vp, i64, ctypes.POINTER(i32), i32]),
            "pkv_build_block_tables": (ctypes.c_int, [vp, ctypes.POINTER(i64), i32, ctypes.POINTER(i32),
                                                      i32, ctypes.POINTER(i32)]),
            "pkv_alloc_stats": (ctypes.c_int, [vp, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                               ctypes.POINTER(i32), ctypes.POINTER(i64)]),
            "pkv_block_refcount": (ctypes.c_int, [vp, i32]),
            "paged_attn_decode_cascade": (ctypes.c_int, [P, P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                                         ctypes.c_int, ctypes.c_int, f32, ctypes.c_int, P, vp]),
            "paged_attn_decode_cascade_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, P, P, P, ctypes.c_int,
                                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, f32,
                                                             ctypes.c_int, P, vp]),
            "paged_attn_prefill": (ctypes.c_int, [P, P, P, P, P, P, ctypes.c_int, ctypes.c_int, f32, ctypes.c_int,
                                                  P, vp]),
            "paged_attn_prefill_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int, f32,
                                                      ctypes.c_int, P, vp]),
            "pkv_alloc_utilisation": (ctypes.c_int, [vp, ctypes.POINTER(i64), ctypes.POINTER(i32)]),
            "pkv_seq_allocate_prefix": (ctypes.c_int, [vp, i64, ctypes.POINTER(i32), i32, i32]),
            "pkv_cache_create": (ctypes.c_int, [vp, ctypes.POINTER(vp)]),
            "pkv_cache_destroy": (None, [vp]),
            "pkv_cache_insert": (ctypes.c_int, [vp, i64, ctypes.POINTER(i32), i32, ctypes.POINTER(i32)]),
            "pkv_cache_match": (ctypes.c_int, [vp, ctypes.POINTER(i32), i32, ctypes.POINTER(i32), i32,
                                               ctypes.POINTER(i32)]),
            "pkv_cache_evict": (ctypes.c_int, [vp, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]),
            "pkv_cache_nodes": (ctypes.c_int, [vp]),
            "swap_out_blocks": (ctypes.c_int, [P, P, P, vp, ctypes.c_size_t, vp]),
            "swap_in_blocks": (ctypes.c_int, [vp, ctypes.c_size_t, P, P, P, vp]),
            "pkv_seq_swap_out": (ctypes.c_int, [vp, i64, ctypes.POINTER(i32), i32, ctypes.POINTER(i32)]),
            "pkv_seq_swap_in": (ctypes.c_int, [vp, i64, ctypes.POINTER(i32), i32, ctypes.POINTER(i32)]),
            "pkv_prefix_groups": (ctypes.c_int, [ctypes.POINTER(i32), i32, i32, ctypes.POINTER(i32), i32, i32,
                                                 ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                                                 ctypes.POINTER(i32), ctypes.POINTER(i32)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pkv_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != PKV_OK:
        raise PkvError(status, what)


# ---------------------------------------------------------------------------
# torch tensor -> pkv_tensor
# ---------------------------------------------------------------------------

def _code(t, fp8: bool = False) -> int:
    import torch
    if fp8:
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise TypeError(f"fp8 cache must be uint8 or float8_e4m3fn, got {t.dtype}")
        return PKV_FP8_E4M3
    table = {torch.float16: PKV_F16, torch.bfloat16: PKV_BF16, torch.int32: PKV_I32,
             torch.int64: PKV_I64, torch.float32: PKV_F32, torch.float8_e4m3fn: PKV_FP8_E4M3}
    if t.dtype not in table:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return table[t.dtype]


def _desc(t, fp8: bool = False, device: bool = True) -> pkv_tensor:
    if device and not t.is_cuda:
        raise ValueError("device call needs CUDA tensors (no CPU fallback)")
    if t.dim() > 4:
        raise ValueError("at most 4 dims")
    d = pkv_tensor()
    d.data = t.data_ptr() if t.numel() > 0 else (t.data_ptr() or None)
    d.dtype = _code(t, fp8)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream(stream) -> ctypes.c_void_p:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ref(d: pkv_tensor):
    return ctypes.byref(d)


# ---------------------------------------------------------------------------
# Device calls
# ---------------------------------------------------------------------------

def paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads: int,
                      scale: float, block_size: int, out, stream=None) -> None:
    ds = [_desc(x) for x in (q, k_cache, v_cache, block_tables, context_lens, out)]
    _check(lib().paged_attn_decode(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), _ref(ds[4]),
                                   int(num_kv_heads), float(scale), int(block_size), _ref(ds[5]),
                                   _stream(stream)), "paged_attn_decode")


class PrefixGroups:
    """A batch's shared-prefix grouping on the device (from pkv_prefix_groups)."""

    def __init__(self, tables, lens, block_size: int, min_members: int = 2, device=None):
        import torch
        gs, mem, pb = prefix_groups(tables.cpu(), lens.cpu(), block_size, min_members)
        dev = device if device is not None else "cuda"
        self.num_groups = int(gs.numel() - 1)
        sizes = (gs[1:] - gs[:-1]).tolist()
        self.max_group_size = int(max(sizes)) if sizes else 0
        self.max_prefix_blocks = int(pb.max()) if pb.numel() else 0
        self.group_start = gs.to(dev)
        self.members = mem.to(dev) if mem.numel() else torch.zeros(0, dtype=torch.int32, device=dev)
        self.prefix_blocks = pb.to(dev)

    @classmethod
    def on_device(cls, prefix_blocks, group_start, members, num_groups: int, max_group_size: int,
                  max_prefix_blocks: int) -> "PrefixGroups":
        """A grouping whose arrays already live on the device (for instance
        views into a caller's staging buffer)."""
        g = cls.__new__(cls)
        g.prefix_blocks, g.group_start, g.members = prefix_blocks, group_start, members
        g.num_groups, g.max_group_size = int(num_groups), int(max_group_size)
        g.max_prefix_blocks = int(max_prefix_blocks)
        return g


def _cascade_descs(q, k_cache, v_cache, block_tables, context_lens, groups, out, k_scale, v_scale):
    """Descriptors in the argument order of paged_attn_decode_cascade(_fp8)."""
    fp8 = k_scale is not None
    head = [_desc(q), _desc(k_cache, fp8), _desc(v_cache, fp8)]
    if fp8:
        head += [_desc(k_scale), _desc(v_scale)]
    tail = [_desc(x) for x in (block_tables, context_lens, groups.prefix_blocks, groups.group_start,
                               groups.members)]
    return fp8, head + tail, _desc(out)


def paged_attn_decode_cascade(q, k_cache, v_cache, block_tables, context_lens, groups: PrefixGroups,
                              num_kv_heads: int, scale: float, block_size: int, out, stream=None,
                              k_scale=None, v_scale=None) -> None:
    """Prefix-aware decode; with k_scale / v_scale the caches are fp8-e4m3
    (paged_attn_decode_cascade_fp8)."""
    fp8, ds, do = _cascade_descs(q, k_cache, v_cache, block_tables, context_lens, groups, out,
                                 k_scale, v_scale)
    name = "paged_attn_decode_cascade_fp8" if fp8 else "paged_attn_decode_cascade"
    _check(getattr(lib(), name)(*[_ref(d) for d in ds], groups.num_groups, groups.max_group_size,
                                groups.max_prefix_blocks, int(num_kv_heads), float(scale),
                                int(block_size), _ref(do), _stream(stream)), name)


def prepare_decode_cascade(q, k_cache, v_cache, block_tables, context_lens, groups: PrefixGroups,
                           num_kv_heads: int, scale: float, block_size: int, out, stream=None,
                           k_scale=None, v_scale=None) -> "Prepared":
    fp8, ds, do = _cascade_descs(q, k_cache, v_cache, block_tables, context_lens, groups, out,
                                 k_scale, v_scale)
    name = "paged_attn_decode_cascade_fp8" if fp8 else "paged_attn_decode_cascade"
    args = tuple(ctypes.byref(d) for d in ds) + (
        groups.num_groups, groups.max_group_size, groups.max_prefix_blocks, int(num_kv_heads),
        float(scale), int(block_size), ctypes.byref(do))
    return Prepared(name, getattr(lib(), name), args,
                    (ds, do, groups, (q, k_cache, v_cache, block_tables, context_lens, out, k_scale, v_scale)),
                    stream)


def _prefill_descs(q, k_cache, v_cache, block_tables, context_lens, q_start, out, k_scale, v_scale):
    """Descriptors in the argument order of paged_attn_prefill(_fp8)."""
    fp8 = k_scale is not None
    ds = [_desc(q), _desc(k_cache, fp8), _desc(v_cache, fp8)]
    if fp8:
        ds += [_desc(k_scale), _desc(v_scale)]
    ds += [_desc(block_tables), _desc(context_lens), _desc(q_start)]
    return ("paged_attn_prefill_fp8" if fp8 else "paged_attn_prefill"), ds, _desc(out)


def paged_attn_prefill(q, k_cache, v_cache, block_tables, context_lens, q_start, max_q_tokens: int,
                       num_kv_heads: int, scale: float, block_size: int, out, stream=None,
                       k_scale=None, v_scale=None) -> None:
    """Causal attention of several new tokens per sequence (q rows of sequence
    s: q_start[s] .. q_start[s + 1], its last tokens; lens include them); with
    k_scale / v_scale the caches are fp8-e4m3 (paged_attn_prefill_fp8)."""
    name, ds, do = _prefill_descs(q, k_cache, v_cache, block_tables, context_lens, q_start, out,
                                  k_scale, v_scale)
    _check(getattr(lib(), name)(*[_ref(d) for d in ds], int(max_q_tokens), int(num_kv_heads), float(scale),
                                int(block_size), _ref(do), _stream(stream)), name)


def prepare_prefill(q, k_cache, v_cache, block_tables, context_lens, q_start, max_q_tokens: int,
                    num_kv_heads: int, scale: float, block_size: int, out, stream=None,
                    k_scale=None, v_scale=None) -> "Prepared":
    name, ds, do = _prefill_descs(q, k_cache, v_cache, block_tables, context_lens, q_start, out,
                                  k_scale, v_scale)
    args = tuple(ctypes.byref(d) for d in ds) + (int(max_q_tokens), int(num_kv_heads), float(scale),
                                                 int(block_size), ctypes.byref(do))
    return Prepared(name, getattr(lib(), name), args,
                    (ds, do, (q, k_cache, v_cache, block_tables, context_lens, q_start, out, k_scale, v_scale)),
                    stream)


def swap_record_bytes(k_cache) -> int:
    """Bytes of one host record of a block (its K tile then its V tile)."""
    return 2 * k_cache[0].numel() * k_cache.element_size()


def swap_out_blocks(k_cache, v_cache, blocks, host, stream=None) -> None:
    """Copy blocks[i] of both pools into record i of `host` (page-locked)."""
    fp8 = k_cache.dtype in _FP8_TYPES()
    ds = [_desc(k_cache, fp8), _desc(v_cache, fp8), _desc(blocks)]
    _check(lib().swap_out_blocks(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), ctypes.c_void_p(host.data_ptr()),
                                 host.numel() * host.element_size(), _stream(stream)), "swap_out_blocks")


def swap_in_blocks(host, blocks, k_cache, v_cache, stream=None) -> None:
    """Copy record i of `host` (page-locked) into block blocks[i] of both pools."""
    fp8 = k_cache.dtype in _FP8_TYPES()
    ds = [_desc(blocks), _desc(k_cache, fp8), _desc(v_cache, fp8)]
    _check(lib().swap_in_blocks(ctypes.c_void_p(host.data_ptr()), host.numel() * host.element_size(), _ref(ds[0]),
                                _ref(ds[1]), _ref(ds[2]), _stream(stream)), "swap_in_blocks")


def _FP8_TYPES():
    import torch
    return (torch.uint8, torch.float8_e4m3fn)


def paged_attn_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                          num_kv_heads: int, scale: float, block_size: int, out, stream=None) -> None:
    ds = [_desc(q), _desc(k_cache, True), _desc(v_cache, True), _desc(k_scale), _desc(v_scale),
          _desc(block_tables), _desc(context_lens), _desc(out)]
    _check(lib().paged_attn_decode_fp8(*[_ref(d) for d in ds[:7]], int(num_kv_heads), float(scale),
                                       int(block_size), _ref(ds[7]), _stream(stream)),
           "paged_attn_decode_fp8")


def workspace_bytes(num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                    cache_dtype: int, device: int = 0) -> int:
    return int(lib().paged_attn_decode_workspace_bytes(num_q_heads, num_kv_heads, head_dim,
                                                        block_size, cache_dtype, device))


def paged_attn_decode_ex(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads: int,
                         scale: float, block_size: int, out, workspace, k_scale=None, v_scale=None,
                         stream=None, flags: int = 0) -> None:
    fp8 = k_scale is not None
    ks = _desc(k_scale) if fp8 else None
    vs = _desc(v_scale) if fp8 else None
    ds = [_desc(q), _desc(k_cache, fp8), _desc(v_cache, fp8), _desc(block_tables),
          _desc(context_lens), _desc(out)]
    _check(lib().paged_attn_decode_ex(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]),
                                      _ref(ks) if fp8 else None, _ref(vs) if fp8 else None,
                                      _ref(ds[3]), _ref(ds[4]), int(num_kv_heads), float(scale),
                                      int(block_size), _ref(ds[5]),
                                      ctypes.c_void_p(workspace.data_ptr()),
                                      workspace.numel() * workspace.element_size(), int(flags),
                                      _stream(stream)), "paged_attn_decode_ex")


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads: int,
                              scale: float, block_size: int, out, k_scale=None, v_scale=None,
                              stream=None) -> None:
    """Decode for callers that cannot allocate device memory at call time:
    the split-KV scratch is a static device array of the library (see
    paged_attn_decode_noalloc in include/pagedkv.h). Calls on one device
    share that array, so calls that overlap on the GPU race."""
    fp8 = k_scale is not None
    ks = _desc(k_scale) if fp8 else None
    vs = _desc(v_scale) if fp8 else None
    ds = [_desc(q), _desc(k_cache, fp8), _desc(v_cache, fp8), _desc(block_tables),
          _desc(context_lens), _desc(out)]
    _check(lib().paged_attn_decode_noalloc(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]),
                                           _ref(ks) if fp8 else None, _ref(vs) if fp8 else None,
                                           _ref(ds[3]), _ref(ds[4]), int(num_kv_heads), float(scale),
                                           int(block_size), _ref(ds[5]), _stream(stream)),
           "paged_attn_decode_noalloc")


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, stream=None) -> None:
    ds = [_desc(x) for x in (k, v, k_cache, v_cache, slot_mapping)]
    _check(lib().reshape_and_cache(*[_ref(d) for d in ds], _stream(stream)), "reshape_and_cache")


def reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale, stream=None) -> None:
    ds = [_desc(k), _desc(v), _desc(k_cache, True), _desc(v_cache, True), _desc(slot_mapping),
          _desc(k_scale), _desc(v_scale)]
    _check(lib().reshape_and_cache_fp8(*[_ref(d) for d in ds], _stream(stream)),
           "reshape_and_cache_fp8")


def copy_blocks(k_cache, v_cache, pairs, stream=None) -> None:
    import torch
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    ds = [_desc(k_cache, fp8), _desc(v_cache, fp8), _desc(pairs)]
    _check(lib().copy_blocks(*[_ref(d) for d in ds], _stream(stream)), "copy_blocks")


def device_error(device: int = 0) -> int:
    """PKV_OK, or PKV_ERR_DEVICE_CHECK if a kernel flagged a bad index since
    the last call (synchronises the device and clears the flag)."""
    return int(lib().pkv_device_error(int(device)))


# ---------------------------------------------------------------------------
# Host block allocator
# ---------------------------------------------------------------------------

class PrefixCache:
    """Radix tree of cached full blocks over a BlockAllocator (C++)."""

    def __init__(self, alloc: "BlockAllocator"):
        self._alloc = alloc  # keeps the allocator alive while the cache exists
        self._h = ctypes.c_void_p()
        _check(lib().pkv_cache_create(alloc._h, ctypes.byref(self._h)), "pkv_cache_create")

    def close(self) -> None:
        if self._h:
            lib().pkv_cache_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _toks(tokens):
        return (ctypes.c_int32 * max(1, len(tokens)))(*[int(x) for x in tokens])

    def insert(self, seq: int, tokens: Sequence[int]) -> int:
        added = ctypes.c_int32()
        _check(lib().pkv_cache_insert(self._h, int(seq), self._toks(tokens), len(tokens), ctypes.byref(added)),
               "pkv_cache_insert")
        return added.value

    def match(self, tokens: Sequence[int]) -> List[int]:
        cap = max(1, len(tokens))
        buf, m = (ctypes.c_int32 * cap)(), ctypes.c_int32()
        _check(lib().pkv_cache_match(self._h, self._toks(tokens), len(tokens), buf, cap, ctypes.byref(m)),
               "pkv_cache_match")
        return list(buf[:m.value])

    def evict(self, n: int) -> List[int]:
        buf, k = (ctypes.c_int32 * max(1, n))(), ctypes.c_int32()
        _check(lib().pkv_cache_evict(self._h, int(n), buf, ctypes.byref(k)), "pkv_cache_evict")
        return list(buf[:k.value])

    @property
    def nodes(self) -> int:
        return int(lib().pkv_cache_nodes(self._h))


def prefix_groups(tables, lens, block_size: int, min_members: int = 2):
    """Shared-prefix groups of a decode batch (pkv_prefix_groups).

    tables: int32 [S, W] CPU tensor, lens: int32 [S] CPU tensor. Returns
    (group_start int32 [G + 1], members int32 [M], prefix_blocks int32 [S]) as
    CPU tensors."""
    import torch
    t = tables.to(torch.int32).contiguous()
    ln = lens.to(torch.int32).contiguous()
    S, W = int(t.shape[0]), int(t.shape[1])
    gs = torch.empty(S + 1, dtype=torch.int32)
    mem = torch.empty(max(S, 1), dtype=torch.int32)
    pb = torch.empty(max(S, 1), dtype=torch.int32)
    G, M = ctypes.c_int32(), ctypes.c_int32()
    i32 = ctypes.POINTER(ctypes.c_int32)
    _check(lib().pkv_prefix_groups(ctypes.cast(t.data_ptr(), i32), S, max(W, 1), ctypes.cast(ln.data_ptr(), i32),
                                   int(block_size), int(min_members), ctypes.cast(gs.data_ptr(), i32),
                                   ctypes.cast(mem.data_ptr(), i32), ctypes.cast(pb.data_ptr(), i32),
                                   ctypes.byref(G), ctypes.byref(M)), "pkv_prefix_groups")
    return gs[:G.value + 1].clone(), mem[:M.value].clone(), pb[:S].clone()


class BlockAllocator:
    """The C++ block allocator (FIFO free list, refcounts, fork, copy-on-write)."""

    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None):
        self._h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            order = (ctypes.c_int32 * len(free_order))(*[int(b) for b in free_order])
        _check(lib().pkv_alloc_create(int(num_blocks), int(block_size), order, ctypes.byref(self._h)),
               "pkv_alloc_create")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self) -> None:
        if self._h:
            lib().pkv_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, seq: int, num_tokens: int) -> None:
        _check(lib().pkv_seq_allocate(self._h, int(seq), int(num_tokens)), "pkv_seq_allocate")

    def append_slot(self, seq: int) -> Tuple[int, int, int]:
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pkv_seq_append_slot(self._h, int(seq), ctypes.byref(slot), ctypes.byref(src),
                                         ctypes.byref(dst)), "pkv_seq_append_slot")
        return slot.value, src.value, dst.value

    def append_tokens(self, seq: int, count: int) -> List[Tuple[int, int, int]]:
        return [self.append_slot(seq) for _ in range(count)]

    def fork(self, src: int, dst: int) -> None:
        _check(lib().pkv_seq_fork(self._h, int(src), int(dst)), "pkv_seq_fork")

    def free(self, seq: int) -> None:
        _check(lib().pkv_seq_free(self._h, int(seq)), "pkv_seq_free")

    def allocate_prefix(self, seq: int, blocks: Sequence[int], num_tokens: int) -> None:
        arr = (ctypes.c_int32 * max(1, len(blocks)))(*[int(b) for b in blocks])
        _check(lib().pkv_seq_allocate_prefix(self._h, int(seq), arr, len(blocks), int(num_tokens)),
               "pkv_seq_allocate_prefix")

    def utilisation(self):
        """Pool figures: blocks stored vs blocks without sharing, and fill."""
        tb, ns = ctypes.c_int64(), ctypes.c_int32()
        _check(lib().pkv_alloc_utilisation(self._h, ctypes.byref(tb), ctypes.byref(ns)), "pkv_alloc_utilisation")
        st = self.stats()
        used, tokens = st["used"], st["tokens"]
        return {"blocks_stored": used, "blocks_without_sharing": int(tb.value), "sequences": int(ns.value),
                "tokens": tokens, "saved": (1.0 - used / tb.value) if tb.value else 0.0,
                "utilisation": (tokens / (used * self.block_size)) if used else 1.0,
                "waste_slots": used * self.block_size - tokens,
                "waste_bound": (self.block_size - 1) * int(ns.value)}

    def swap_out(self, seq: int) -> List[int]:
        """The sequence's blocks (to copy out first); it becomes swapped out."""
        cap = max(1, self.num_blocks)
        buf, n = (ctypes.c_int32 * cap)(), ctypes.c_int32()
        _check(lib().pkv_seq_swap_out(self._h, int(seq), buf, cap, ctypes.byref(n)), "pkv_seq_swap_out")
        return list(buf[:n.value])

    def swap_in(self, seq: int) -> List[int]:
        """Fresh blocks for a swapped-out sequence (to copy back into)."""
        cap = max(1, self.num_blocks)
        buf, n = (ctypes.c_int32 * cap)(), ctypes.c_int32()
        _check(lib().pkv_seq_swap_in(self._h, int(seq), buf, cap, ctypes.byref(n)), "pkv_seq_swap_in")
        return list(buf[:n.value])

    def num_tokens(self, seq: int) -> int:
        n = lib().pkv_seq_num_tokens(self._h, int(seq))
        if n < 0:
            raise PkvError(int(n), "pkv_seq_num_tokens")
        return int(n)

    def table(self, seq: int) -> List[int]:
        n = lib().pkv_seq_block_table(self._h, int(seq), None, 0)
        if n < 0:
            raise PkvError(n, "pkv_seq_block_table")
        buf = (ctypes.c_int32 * max(n, 1))()
        lib().pkv_seq_block_table(self._h, int(seq), buf, n)
        return list(buf[:n])

    def build_block_tables(self, seqs: Sequence[int], max_blocks: int):
        """(table int32 [n, max_blocks] padded with -1, lens int32 [n]) as CPU tensors."""
        import torch
        n = len(seqs)
        table = torch.empty((n, max_blocks), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        ids = (ctypes.c_int64 * max(n, 1))(*[int(s) for s in seqs])
        _check(lib().pkv_build_block_tables(
            self._h, ids, n, ctypes.cast(table.data_ptr(), ctypes.POINTER(ctypes.c_int32)), max_blocks,
            ctypes.cast(lens.data_ptr(), ctypes.POINTER(ctypes.c_int32))), "pkv_build_block_tables")
        return table, lens

    def stats(self):
        f, u, s, t = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int64()
        _check(lib().pkv_alloc_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(s),
                                     ctypes.byref(t)), "pkv_alloc_stats")
        return {"free": f.value, "used": u.value, "shared": s.value, "tokens": t.value}

    def num_free(self) -> int:
        return self.stats()["free"]

    def refcount(self, block: int) -> int:
        r = lib().pkv_block_refcount(self._h, int(block))
        if r < 0:
            raise PkvError(r, "pkv_block_refcount")
        return r

    def run(self, ops) -> None:
        for op in ops:
            if op[0] == "allocate":
                self.allocate(op[1], op[2])
            elif op[0] == "fork":
                self.fork(op[1], op[2])
            elif op[0] == "free":
                self.free(op[1])
            elif op[0] == "append":
                self.append_tokens(op[1], op[2])
            else:
                raise ValueError(op)


# ---------------------------------------------------------------------------
# Prepared calls: descriptors built once, each launch is one C call.
# ---------------------------------------------------------------------------

class Prepared:
    """A device call with its descriptors built once (argument marshalling
    only); calling it enqueues the kernels on `stream` (default: torch's
    current stream at preparation time). It keeps the tensors it was built
    from alive, so their device memory cannot be reused under it."""

    def __init__(self, name: str, fn, args, keep, stream=None):
        self._name, self._fn, self._args, self._keep = name, fn, args, keep
        self._stream = _stream(stream)

    def __call__(self) -> None:
        st = self._fn(*self._args, self._stream)
        if st != PKV_OK:
            raise PkvError(st, self._name)


def prepare_decode(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads: int, scale: float,
                   block_size: int, out, k_scale=None, v_scale=None, workspace=None,
                   stream=None, flags: int = 0) -> Prepared:
    fp8 = k_scale is not None
    ds = [_desc(q), _desc(k_cache, fp8), _desc(v_cache, fp8), _desc(block_tables), _desc(context_lens),
          _desc(out)]
    tensors = (q, k_cache, v_cache, block_tables, context_lens, out, k_scale, v_scale)
    L = lib()
    if workspace is not None or fp8:
        ks = _desc(k_scale) if fp8 else None
        vs = _desc(v_scale) if fp8 else None
        if workspace is None:
            args = (ctypes.byref(ds[0]), ctypes.byref(ds[1]), ctypes.byref(ds[2]), ctypes.byref(ks),
                    ctypes.byref(vs), ctypes.byref(ds[3]), ctypes.byref(ds[4]), int(num_kv_heads),
                    float(scale), int(block_size), ctypes.byref(ds[5]))
            return Prepared("paged_attn_decode_fp8", L.paged_attn_decode_fp8, args, (ds, ks, vs, tensors), stream)
        args = (ctypes.byref(ds[0]), ctypes.byref(ds[1]), ctypes.byref(ds[2]),
                ctypes.byref(ks) if fp8 else None, ctypes.byref(vs) if fp8 else None,
                ctypes.byref(ds[3]), ctypes.byref(ds[4]), int(num_kv_heads), float(scale),
                int(block_size), ctypes.byref(ds[5]), ctypes.c_void_p(workspace.data_ptr()),
                workspace.numel() * workspace.element_size(), int(flags))
        return Prepared("paged_attn_decode_ex", L.paged_attn_decode_ex, args, (ds, ks, vs, workspace, tensors),
                        stream)
    args = (ctypes.byref(ds[0]), ctypes.byref(ds[1]), ctypes.byref(ds[2]), ctypes.byref(ds[3]),
            ctypes.byref(ds[4]), int(num_kv_heads), float(scale), int(block_size), ctypes.byref(ds[5]))
    return Prepared("paged_attn_decode", L.paged_attn_decode, args, (ds, tensors), stream)


def prepare_reshape(k, v, k_cache, v_cache, slot_mapping, k_scale=None, v_scale=None,
                    stream=None) -> Prepared:
    fp8 = k_scale is not None
    ds = [_desc(k), _desc(v), _desc(k_cache, fp8), _desc(v_cache, fp8), _desc(slot_mapping)]
    L = lib()
    if fp8:
        ds += [_desc(k_scale), _desc(v_scale)]
        return Prepared("reshape_and_cache_fp8", L.reshape_and_cache_fp8,
                        tuple(ctypes.byref(d) for d in ds),
                        (ds, (k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale)), stream)
    return Prepared("reshape_and_cache", L.reshape_and_cache, tuple(ctypes.byref(d) for d in ds),
                    (ds, (k, v, k_cache, v_cache, slot_mapping)), stream)


def prepare_copy_blocks(k_cache, v_cache, pairs, stream=None) -> Prepared:
    import torch
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    ds = [_desc(k_cache, fp8), _desc(v_cache, fp8), _desc(pairs)]
    return Prepared("copy_blocks", lib().copy_blocks, tuple(ctypes.byref(d) for d in ds),
                    (ds, (k_cache, v_cache, pairs)), stream)

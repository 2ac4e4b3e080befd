"""The C-ABI library loads and exports every symbol include/pagedkv.h declares.

No compute call here: this runs without a GPU.
"""
import os
import re
import subprocess

import pytest

import paged_kv_cache_453_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "for")))


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_453_b200.build import build
    build()


def test_header_parses_to_expected_set():
    decl = declared_functions()
    assert set(decl) == set(P.EXPORTED), set(decl) ^ set(P.EXPORTED)


def test_every_declared_symbol_is_exported():
    L = P.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", P.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    dyn = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in dyn]
    assert not missing, missing


def test_status_strings_and_version():
    assert P.status_string(0) == "ok"
    assert P.status_string(P.PKV_ERR_DEVICE_CHECK) == "device-side check failed"
    assert P.lib().pkv_version() >= 100


def test_host_validation_rejects_bad_arguments_without_touching_the_device():
    # NULL descriptors are refused on the host before any CUDA call.
    L = P.lib()
    assert L.paged_attn_decode(None, None, None, None, None, 8, 0.1, 16, None, None) == P.PKV_ERR_INVALID_ARG
    assert L.reshape_and_cache(None, None, None, None, None, None) == P.PKV_ERR_INVALID_ARG
    assert L.copy_blocks(None, None, None, None) == P.PKV_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        P.paged_attn_decode(q, q, q, q, q, 1, 0.1, 16, q)

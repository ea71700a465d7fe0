"""CPU checks of the C-ABI library: it builds for sm_100a, loads without a GPU,
exports every function include/moe.h declares, and its config struct matches
the header field by field.  No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_layer_61_b200 as moe
from mixture_experts_layer_61_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def test_exports_every_declared_function(lib):
    names = moe.header_functions()
    assert "moe_layer_forward" in names and "dense_ffn" in names and "moe_route" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    assert set(names) <= exported


def test_config_struct_matches_header():
    with open(moe.HEADER) as f:
        text = f.read()
    body = re.search(r"typedef struct \{(.*?)\} moe_config_t;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"int\s+(\w+);", body)
    assert fields == [n for n, _ in moe.MoeConfig._fields_]


def test_status_strings_and_pure_host_queries(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.moe_status_string(code)
    cfg = moe.config(2048, 4096, 8, 2, 14336, tile_B=16)
    # P_max = A + min(E, A) * (B - 1)
    assert lib.moe_padded_rows_max(ctypes.byref(cfg)) == 4096 + 8 * 15
    bad = moe.config(4, 4096, 8, 9, 14336)
    assert lib.moe_padded_rows_max(ctypes.byref(bad)) == -1


def test_library_is_sm100a_only():
    # the build targets sm_100a only: the object carries no other SASS/PTX target
    with open(os.path.join(ROOT, "mixture_experts_layer_61_b200", "build.py")) as f:
        src = f.read()
    assert "arch=compute_100a,code=sm_100a" in src
    assert "sm_90" not in src and "compute_90" not in src

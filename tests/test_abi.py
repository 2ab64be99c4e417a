"""The C-ABI library builds, loads without a GPU and exports every entry point
that include/*.h declares; the Python binding mirrors those names; the product
package never reaches into the oracle."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(pa_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def libpath():
    from paged_kv_cache_388_b200 import build
    return build.build()


def test_header_declares_the_contract():
    names = declared_symbols()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_copy_blocks", "pa_decode_workspace_size",
              "pa_get_device_error", "pa_status_string"):
        assert n in names, n


def test_library_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    for n in declared_symbols():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert declared_symbols() <= exported


def test_host_only_entry_points(libpath):
    lib = ctypes.CDLL(libpath)
    lib.pa_status_string.restype = ctypes.c_char_p
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(-3) == b"PA_ERR_WORKSPACE"
    assert lib.pa_abi_version() >> 16 == 1


def test_binding_mirrors_header_names(libpath):
    from paged_kv_cache_388_b200 import _lib
    for n in declared_symbols():
        if n in ("pa_status_string",):
            continue
        assert hasattr(_lib, n), f"binding lacks {n}"


def test_product_never_imports_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_388_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if not path.endswith((".py", ".cu", ".cuh", ".h")):
            continue
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), path
        assert "pa_oracle" not in text, path


def test_oracle_never_imports_product():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.*")):
        if not path.endswith((".py", ".c")):
            continue
        text = open(path, encoding="utf-8").read()
        assert "paged_kv_cache_388_b200" not in text, path
        assert "pa_device" not in text and "include/pa.h" not in text, path

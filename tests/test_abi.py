"""CPU checks of the C ABI: the library builds for sm_100a, loads, and exports
every function that include/*.h declares.  No compute call is made (there is
no GPU here)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        names |= set(re.findall(r"\b(soup_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def libpath():
    from layer_streamed_qlora_b200 import build
    return build.build()


def test_header_declares_entry_points():
    names = _declared()
    for n in ("soup_nf4_quantize", "soup_nf4_dequant", "soup_lora_linear_fwd", "soup_lora_linear_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if l.strip()}
    missing = [n for n in _declared() if n not in syms]
    assert not missing, missing


def test_library_loads_and_binds(libpath):
    from layer_streamed_qlora_b200 import _lib
    L = _lib.lib()
    for n in _declared():
        assert hasattr(L, n)
    # pure host queries work without a GPU
    assert _lib.soup_lora_linear_bwd_workspace(64, 8, 512) > 0
    assert L.soup_last_error() is not None


def test_library_is_sm100a_only(libpath):
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", libpath], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    arches = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert arches == {"100a"}, arches


def test_adamw_refuses_bad_arguments_on_the_host(libpath):
    """soup_adamw_step's argument checks run on the host before any CUDA
    call: the step index, the hyperparameter ranges and the alignment of
    every buffer.  The pointers below are never dereferenced."""
    from layer_streamed_qlora_b200 import _lib
    f = _lib.lib().soup_adamw_step
    P = ctypes.c_void_p
    ok = [P(0x10000), P(0x20000), P(0x30000), P(0x40000), P(0x50000)]  # theta, bf16, grad, m, v

    def call(ptrs=ok, n=1024, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, t=1):
        return f(*ptrs, n, lr, b1, b2, eps, wd, 1.0, t, 1, None, None)

    INVALID, SHAPE, ALIGN = 1, 2, 3
    assert call(t=0) == INVALID
    assert call(b1=1.0) == INVALID and call(b2=-0.1) == INVALID
    assert call(eps=0.0) == INVALID and call(lr=-1e-3) == INVALID and call(wd=-0.1) == INVALID
    assert call(n=-1) == SHAPE
    assert call(n=0) == 0  # nothing to do, nothing launched
    assert call(ptrs=[ok[0], ok[1], P(0x30004), ok[3], ok[4]]) == ALIGN  # grad not 16-byte aligned
    assert call(ptrs=[ok[0], P(0x20004), ok[2], ok[3], ok[4]]) == ALIGN  # bf16 copy not 8-byte aligned
    assert call(ptrs=[None] + ok[1:]) == INVALID
    assert b"soup_adamw_step" in _lib.lib().soup_last_error()


def test_header_is_plain_c(tmp_path):
    """include/soup.h declares a C ABI: a C99 translation unit that includes
    it and takes the address of every declared function compiles with gcc."""
    names = _declared()
    src = tmp_path / "abi.c"
    body = "\n".join(f"  (void)&{n};" for n in names)
    src.write_text(f'#include "soup.h"\nint main(void) {{\n{body}\n  return 0;\n}}\n')
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.join(ROOT, "include"),
                        str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

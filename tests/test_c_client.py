"""The boundary from plain C: include/shampoo.h compiles as C99 and C++11,
and a C program links against the shared library and calls its host-side
entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from shampoo_second_order_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.join(ROOT, "tests", "c_client")
BUILD = os.path.join(HERE, "_build")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"
    return r.stdout


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++11")])
def test_header_is_plain_c(lang, std):
    cc = "gcc" if lang == "c" else "g++"
    _run([cc, "-fsyntax-only", "-x", lang, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror",
          os.path.join(ROOT, "include", "shampoo.h")])


def test_c_program_links_and_calls_the_library():
    if not os.path.exists(L.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, "client")
    libdir = os.path.dirname(L.LIB_PATH)
    _run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
          os.path.join(HERE, "client.c"), "-L", libdir, "-lshampoo_b200", f"-Wl,-rpath,{libdir}", "-o", exe])
    out = _run([exe])
    assert out.startswith("owners ")

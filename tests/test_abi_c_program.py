"""The header is a C header: a plain C99 program compiles against
include/ssm_causal.h, links with libssm_causal.so and runs its calls on the
host (every call is one the host-side checks reject, so no GPU is needed).
Beside it, the header's prototypes are parsed and compared, argument by
argument, with the ctypes signatures of the Python binding, so the header, the
library and the binding cannot drift apart unnoticed."""

import ctypes
import os
import re
import shutil
import subprocess

import pytest

from selective_state_space_causal_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_causal.h")
PROGRAM = os.path.join(ROOT, "tests", "c", "abi_from_c.c")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_compiles_links_and_runs(tmp_path):
    exe = str(tmp_path / "abi_from_c")
    libdir = os.path.dirname(_lib.LIBRARY)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), PROGRAM, "-o", exe,
           "-L", libdir, "-l:" + os.path.basename(_lib.LIBRARY), "-Wl,-rpath," + libdir]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")


def _prototypes():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"^([A-Za-z_][\w \*]*?)\b(ssm_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        args = [] if params in ("", "void") else [" ".join(a.split()) for a in params.split(",")]
        protos[name] = (ret, args)
    return protos


def _kind_of_c(decl: str) -> str:
    """Calling-convention class of a C parameter or return type."""
    if "*" in decl or "ssm_stream_t" in decl:
        return "ptr"
    words = decl.replace("const", "").split()
    if "int64_t" in words:
        return "i64"
    if "size_t" in words or "unsigned long long" in " ".join(words):
        return "u64"  # both are unsigned 64-bit on the supported (LP64) hosts
    if words[0] in ("int", "ssm_dtype"):
        return "i32"
    raise AssertionError(f"unclassified C type: {decl}")


def _kind_of_ctypes(t) -> str:
    if t is None:
        return "none"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and t.__name__.startswith("LP_"):
        return "ptr"
    # ctypes aliases integer types of the same width, so compare width and sign
    size, signed = ctypes.sizeof(t), t(-1).value < 0
    if (size, signed) == (8, True):
        return "i64"
    if (size, signed) == (8, False):
        return "u64"
    if (size, signed) == (4, True):
        return "i32"
    raise AssertionError(f"unclassified ctypes type: {t}")


def test_binding_signatures_match_the_header():
    protos = _prototypes()
    bound = {name: (res, args) for name, res, args in _lib.SIGNATURES}
    assert set(protos) == set(bound)
    for name, (ret, params) in protos.items():
        res, args = bound[name]
        assert len(params) == len(args), f"{name}: {len(params)} parameters, bound {len(args)}"
        for i, (p, a) in enumerate(zip(params, args)):
            assert _kind_of_c(p) == _kind_of_ctypes(a), f"{name} argument {i}: {p} vs {a}"
        assert _kind_of_c(ret + " x") == _kind_of_ctypes(res), f"{name} result: {ret} vs {res}"

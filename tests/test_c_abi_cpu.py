"""The C ABI from plain C (no GPU): tests/c_abi/host_checks.c is compiled with
gcc against include/msa.h alone and linked with libmsa.so.  It checks calls
the host rejects before any device work, and prints the layout of the
descriptor structs, which must match the Python binding's ctypes mirrors."""
import ctypes
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.dirname(msa.LIB_PATH)


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    msa_build.build()
    exe = str(tmp_path_factory.mktemp("c_abi") / "host_checks")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "host_checks.c"),
                    "-L", PKG, "-lmsa", "-Wl,-rpath," + PKG, "-o", exe], check=True)
    return exe


def test_c_program_host_checks_and_layout(program):
    r = subprocess.run([program], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    lines = {l.split()[0]: [int(x) for x in l.split()[1:]] for l in r.stdout.splitlines()
             if l.startswith("msa_")}
    assert r.stdout.strip().endswith("ok")
    for struct, name in ((msa.msa_cache, "msa_cache"), (msa.msa_seqs, "msa_seqs"),
                         (msa.msa_prefix_groups, "msa_prefix_groups")):
        size, *offsets = lines[name]
        assert size == ctypes.sizeof(struct), name
        assert offsets == [getattr(struct, f).offset for f, _ in struct._fields_], name

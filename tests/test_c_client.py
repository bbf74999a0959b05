"""The C ABI from plain C: include/bsattn.h compiles as strict C99 and as C++, and a C
program linked against libbsattn.so gets the same workspace sizes as the Python binding and
the same host-side rejections.  No GPU: the program only calls what needs no device."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
CLIENT = os.path.join(ROOT, "tests", "c_client", "abi_client.c")


@pytest.fixture(scope="module")
def B():
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    b.lib()
    return b


def test_header_is_strict_c99_and_cxx(tmp_path):
    src = tmp_path / "only_header.c"
    src.write_text('#include "bsattn.h"\nint main(void) { return (int)BSA_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    "-fsyntax-only", str(src)], check=True)
    cxx = tmp_path / "only_header.cpp"
    cxx.write_text('#include "bsattn.h"\nint main() { return static_cast<int>(BSA_OK); }\n')
    subprocess.run(["g++", "-std=c++11", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    "-fsyntax-only", str(cxx)], check=True)


def test_c_program_links_and_agrees_with_the_binding(B, tmp_path):
    lib_dir = os.path.dirname(B.bsattn.LIB_PATH)
    exe = tmp_path / "abi_client"
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    CLIENT, "-o", str(exe), "-L", lib_dir, "-lbsattn",
                    "-Wl,-rpath," + lib_dir], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    lines = run.stdout.splitlines()
    assert lines[-1] == "fails 0"
    sizes = {}
    for ln in lines:
        if ln.startswith("shape"):
            name, op, n = ln.split()
            sizes[(int(name[5:]), int(op[2:]))] = int(n)
    shapes = [
        B.Shape(batch=1, heads=40, head_dim=128, T=21, H=45, W=80, Tp=24, Hp=48, Wp=80,
                q_block=64, kv_block=64),
        B.Shape(batch=2, heads=3, head_dim=64, T=6, H=10, W=11, Tp=8, Hp=12, Wp=12,
                q_block=128, kv_block=64),
    ]
    ops = [B.OP_BLOCK_MASS, B.OP_TOPP_SELECT, B.OP_FWD, B.OP_PATTERN, B.OP_POOLED_MASS]
    assert len(sizes) == 10
    for i, s in enumerate(shapes):
        for op in ops:
            assert sizes[(i, op)] == B.workspace_bytes(s, op) > 0, (i, op)

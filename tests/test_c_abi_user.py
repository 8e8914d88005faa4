"""The C ABI from plain C: tests/c/abi_user.c compiles as C99 against
include/bitssm.h and links against libbitssm.so; its host-only calls run
(no device is touched)."""

import os
import subprocess

from tests.test_abi_exports import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_caller_compiles_links_and_runs_host_calls(tmp_path):
    ensure_built()
    libdir = os.path.join(ROOT, "ternary_weight_selective_b200")
    exe = str(tmp_path / "abi_user")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_user.c"),
                    "-L", libdir, "-l:libbitssm.so", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("abi 2, workspace")

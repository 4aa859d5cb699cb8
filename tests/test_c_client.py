"""The C ABI from a plain C program: tests/c_client/bm_client.c is compiled with
the host C compiler against include/pagedkv.h, linked to the in-tree library,
and run (host-side block manager and pair-check calls only, so no GPU is needed);
the header must compile as strict C11 with warnings as errors."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_client_drives_the_block_manager(tmp_path):
    from paged_kv_cache_324_b200 import binding, build
    build.build()
    lib_dir = os.path.dirname(binding._LIB_PATH)
    exe = str(tmp_path / "bm_client")
    subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_client", "bm_client.c"), "-o", exe, "-L", lib_dir, "-lpagedkv",
                    "-Wl,-rpath," + lib_dir], check=True)
    env = dict(os.environ)
    env["LD_LIBRARY_PATH"] = ":".join([lib_dir, "/usr/local/cuda/lib64", env.get("LD_LIBRARY_PATH", "")])
    res = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=60)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == "ok"

"""libonebit from plain C: tests/c_abi_client.c is compiled as strict C99
against include/onebit.h, linked with libonebit.so and run (host-only
calls, no GPU); its results must equal the Python binding's."""
import os
import shutil
import subprocess

import pytest

from error_compensated_bit_adam_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client_links_and_agrees_with_the_binding(tmp_path):
    B.lib()  # built
    libdir = os.path.dirname(B.LIBRARY)
    exe = tmp_path / "client"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_client.c"),
                           "-L", libdir, "-lonebit", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out
    fields = out.stdout.split()
    numel = [100003, 31, 0]
    offsets, n_pad = B.ob_layout(numel)
    cb, ce, wb, we = B.ob_server_shard_range(numel, 8, 4, 1)
    want = [offsets[1], n_pad, *B.ob_chunk_range(numel[0], 8, 3), B.ob_workspace_bytes(numel, 8),
            cb, ce, wb, we]
    assert [int(f) for f in fields[:9]] == want
    assert fields[9] == "OB_ERR_PHASE"

"""The C ABI from plain C: tests/c_client.c, compiled with gcc against
include/bb_attn.h alone and linked with libbbattn.so, runs the host-only
calls; its random tables are compared with the oracle's bit for bit."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from block_sparse_long_bwd_b200 import binding as bb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client(tmp_path):
    lib = bb.LIB_PATH
    assert os.path.exists(lib)
    exe = tmp_path / "c_client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_client.c"), "-o", str(exe),
                    lib, "-Wl,-rpath," + os.path.dirname(lib)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.splitlines()
    assert lines[-1] == "ok"
    tables, cur = {}, None
    for line in lines[:-1]:
        if line.startswith("table "):
            _, name, H, nb, rr = line.split()
            cur = tables[name] = {"shape": (int(H), int(nb), int(rr)),
                                  "rows": []}
        else:
            cur["rows"].append([int(x) for x in line.split()])
    for name, kw in (("plain", {}), ("layer", dict(max_blocks=64,
                                                   last_block=16))):
        H, nb, rr = tables[name]["shape"]
        got = np.array(tables[name]["rows"], dtype=np.int32).reshape(H, nb, rr)
        assert np.array_equal(got, oracle.rand_table(7, H, nb, rr, **kw)), name

"""The C ABI from plain C: tests/abi_c_check.c is compiled with gcc as strict
C11 against include/paged.h and linked with the in-tree libpaged.so, then run
on the host (no device call). Its printed results are checked against
hashlib, the oracle's allocator model and hand-computed slots."""
import hashlib
import os
import shutil
import struct
import subprocess

import pytest

import paged_kv_cache_448_b200 as pk
from oracle.block_manager import BlockManager
from paged_kv_cache_448_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler on this machine")
    lib_dir = os.path.dirname(_native.LIB_PATH)
    _native.lib()  # fails loudly when the library is not built
    exe = str(tmp_path_factory.mktemp("abi_c") / "abi_c_check")
    cmd = [gcc, "-std=c11", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c_check.c"),
           "-L", lib_dir, "-lpaged", f"-Wl,-rpath,{lib_dir}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60)
    out = {}
    for line in run.stdout.splitlines():
        key, _, rest = line.partition(" ")
        out[key] = rest
    return out


def test_hashes_from_c(c_output):
    assert c_output["sha256_abc"] == hashlib.sha256(b"abc").hexdigest()
    tokens = [1000 + 7 * i for i in range(34)]
    parent = bytes(32)
    for j in range(2):
        block = struct.pack("<16i", *tokens[16 * j:16 * j + 16])
        parent = hashlib.sha256(parent + block).digest()
        assert c_output[f"block_hash_{j}"] == parent.hex()


def test_allocator_from_c(c_output):
    bm = BlockManager(8, [5, 2, 7, 0, 1, 6, 3, 4])
    ids = bm.allocate(3)
    assert c_output["allocated"] == " ".join(map(str, ids))
    bm.share(ids[0])
    bm.free(ids)
    assert int(c_output["refcount_first"]) == bm.refcount[ids[0]] == 1
    assert int(c_output["num_free"]) == bm.num_free()
    assert c_output["free_list"].split() == [str(b) for b in bm.free_blocks]
    assert int(c_output["oom"]) == _native.PA_ERR_OOM


def test_slots_and_sizes_from_c(c_output):
    # table rows {4, 9, -1} and {3, 8, 11}, block size 16
    assert c_output["slots"].split() == [str(4 * 16 + 0), str(9 * 16 + 1), str(11 * 16 + 8),
                                         "-1"]
    assert int(c_output["prefill_ws"]) == pk.chunked_prefill_workspace_size(
        16, 16 * 512, 32, 32, 128, 512, 4096)
    status, msg = c_output["bad_decode"].split()
    assert int(status) == _native.PA_ERR_INVALID_ARG and msg == "message"

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


def test_header_links_from_cpp(tmp_path):
    """The same client compiled as C++17: the header's extern "C" block gives
    C linkage, so the library's symbols resolve from C++ too."""
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler on this machine")
    lib_dir = os.path.dirname(_native.LIB_PATH)
    _native.lib()
    exe = str(tmp_path / "abi_cpp_check")
    subprocess.run([gxx, "-x", "c++", "-std=c++17", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_c_check.c"),
                    "-L", lib_dir, "-lpaged", f"-Wl,-rpath,{lib_dir}", "-o", exe],
                   check=True, capture_output=True, text=True)
    run = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60)
    assert f"sha256_abc {hashlib.sha256(b'abc').hexdigest()}" in run.stdout


def test_slots_and_sizes_from_c(c_output):
    # table rows {4, 9, -1} and {3, 8, 11}, block size 16
    assert c_output["slots"].split() == [str(4 * 16 + 0), str(9 * 16 + 1), str(11 * 16 + 8),
                                         "-1"]
    assert int(c_output["prefill_ws"]) == pk.chunked_prefill_workspace_size(
        16, 16 * 512, 32, 32, 128, 512, 4096)
    status, msg = c_output["bad_decode"].split()
    assert int(status) == _native.PA_ERR_INVALID_ARG and msg == "message"


@pytest.mark.gpu
def test_decode_step_from_c(tmp_path):
    """tests/abi_c_decode.c runs reshape_and_cache and decode through the C
    ABI with only the CUDA runtime (no PyTorch): its tables equal the oracle
    allocator's, its scattered caches equal the oracle's bit for bit, and its
    output is within the bf16 tolerance of the oracle's decode."""
    import numpy as np

    import oracle
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler on this machine")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    lib_dir = os.path.dirname(_native.LIB_PATH)
    _native.lib()
    exe = str(tmp_path / "abi_c_decode")
    subprocess.run([gcc, "-std=c11", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    os.path.join(ROOT, "tests", "abi_c_decode.c"),
                    "-L", lib_dir, "-lpaged", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}",
                    "-o", exe], check=True, capture_output=True, text=True)
    run = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    S, H, HKV, D, BS, NB, MAXB = 3, 8, 2, 128, 16, 32, 19

    def load(name, dtype, shape):
        return np.fromfile(tmp_path / name, dtype=dtype).reshape(shape)

    ctx = load("context_lens.bin", np.int32, (S,))
    table = load("block_tables.bin", np.int32, (S, MAXB))
    slots = load("slots.bin", np.int32, (S,))
    bm = BlockManager(NB, [(i * 7 + 3) % NB for i in range(NB)])
    ref_table = np.full((S, MAXB), -1, np.int32)
    for s in range(S):
        ids = bm.allocate(-(-int(ctx[s]) // BS))
        ref_table[s, :len(ids)] = ids
    assert np.array_equal(table, ref_table)
    assert np.array_equal(slots, oracle.slot_mapping(ref_table, ctx - 1, BS))
    kc = load("key_cache_in.bin", np.uint16, (NB, BS, HKV, D)).copy()
    vc = load("value_cache_in.bin", np.uint16, (NB, BS, HKV, D)).copy()
    oracle.reshape_and_cache(load("new_key.bin", np.uint16, (S, HKV, D)),
                             load("new_value.bin", np.uint16, (S, HKV, D)), kc, vc, slots,
                             block_size=BS, kv_dtype="bf16", cache_dtype="bf16")
    assert np.array_equal(load("key_cache_out.bin", np.uint16, (NB, BS, HKV, D)), kc)
    assert np.array_equal(load("value_cache_out.bin", np.uint16, (NB, BS, HKV, D)), vc)
    ref = oracle.decode(load("query.bin", np.uint16, (S, H, D)), kc, vc, ref_table, ctx,
                        scale=np.float32(0.08838834764831845), q_dtype="bf16",
                        cache_dtype="bf16")
    # bf16 output codes -> values: the code is the upper half of an fp32
    got = (load("out.bin", np.uint16, (S, H, D)).astype(np.uint32) << 16).view(np.float32)
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= 2e-3 + 1e-2 * np.abs(ref)), float(err.max())

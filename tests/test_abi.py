"""CPU tests of the C ABI: the library loads, exports every symbol the header
declares, and its host logic (partition math, argument checks) is right. No
compute call reaches a GPU here."""

import ctypes
import os
import re

import pytest

from oracle.partition import balanced_ranges as oracle_ranges
from oracle.partition import head_chunk_ranges as oracle_chunks

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import build
    build.build()
    from ulysses_sequence_attention_sp_b200 import usp as mod
    return mod


def _header_symbols():
    text = open(os.path.join(ROOT, "include", "usp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(usp_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(usp):
    lib = ctypes.CDLL(usp.library_path())
    declared = _header_symbols()
    assert len(declared) >= 18
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(usp.EXPORTED) == declared


def test_library_version(usp):
    assert usp.version() >= 100


def test_partition_matches_oracle(usp):
    for total, parts in [(10, 3), (37, 4), (6, 4), (75600, 7), (24, 7), (576, 4), (1, 1), (32, 32), (1000, 31)]:
        assert usp.balanced_ranges(total, parts) == oracle_ranges(total, parts)
        assert usp.sp_seq_split(total, parts) == [b - a for a, b in oracle_ranges(total, parts)]
    for total, parts in [(2, 3), (5, 0), (0, 1), (3, -2)]:
        with pytest.raises(usp.UspError) as e:
            usp.sp_seq_split(total, parts)
        assert e.value.code == usp.USP_ERR_INVALID_ARG


def test_head_chunks_match_oracle(usp):
    for g in range(1, 20):
        for n in range(1, 25):
            assert usp.head_chunk_ranges(g, n) == oracle_chunks(g, n)
    for g, n in [(0, 1), (3, 0), (3, -1)]:
        with pytest.raises(usp.UspError):
            usp.head_chunk_ranges(g, n)


@pytest.mark.parametrize("args,code", [
    (dict(batch=1, seq_len=8, heads=4, head_dim=16, world=0), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=4, head_dim=16, world=33), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=3, heads=4, head_dim=16, world=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=3, head_dim=16, world=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=0, seq_len=8, heads=4, head_dim=16, world=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=4, head_dim=0, world=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=300, head_dim=16, world=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=4, head_dim=16, world=4, prefix=2), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=4, head_dim=16, world=4, dtype=9), "USP_ERR_DTYPE"),
    # grouped-query attention: kv heads must divide q heads, split over every rank
    (dict(batch=1, seq_len=8, heads=6, head_dim=16, world=2, kv_heads=4), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=8, head_dim=16, world=4, kv_heads=2), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=8, heads=8, head_dim=16, world=2, kv_heads=0), "USP_ERR_INVALID_ARG"),
    # q 4,4,4 over kv 2,1,1: rank 1's query heads 4..7 need kv heads 2 and 3
    (dict(batch=1, seq_len=9, heads=12, head_dim=16, world=3, kv_heads=4), "USP_ERR_SHAPE"),
    # Ulysses + Ring hybrid: ring_size must divide world, world <= 32, heads >= ulysses ranks
    (dict(batch=1, seq_len=64, heads=8, head_dim=16, world=8, ring_size=3), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=64, heads=32, head_dim=16, world=64, ring_size=2), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=64, heads=2, head_dim=16, world=8, ring_size=2), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=5, heads=4, head_dim=16, world=8, ring_size=2), "USP_ERR_INVALID_ARG"),
    (dict(batch=1, seq_len=64, heads=4, head_dim=16, world=4, ring_size=0), "USP_ERR_INVALID_ARG"),
    # fewer kv heads than ranks
    (dict(batch=1, seq_len=9, heads=6, head_dim=16, world=4, kv_heads=2), "USP_ERR_INVALID_ARG"),
])
def test_plan_rejects_bad_arguments_before_any_device_work(usp, args, code):
    with pytest.raises(usp.UspError) as e:
        usp.Plan(**args)
    assert e.value.code == getattr(usp, code)


def test_plan_without_device_or_valid(usp):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible; covered by the GPU tests")
    with pytest.raises(usp.UspError) as e:
        usp.Plan(1, 37, 6, 16, 4, "fp32")
    assert e.value.code == usp.USP_ERR_NO_DEVICE


def test_null_pointers_rejected(usp):
    lib = ctypes.CDLL(usp.library_path())
    lib.usp_scatter_sequence.restype = ctypes.c_int
    lib.usp_ulysses_attention.restype = ctypes.c_int
    lib.usp_plan_query.restype = ctypes.c_int
    # NULL plan is rejected before anything else
    assert lib.usp_scatter_sequence(None, None, None, ctypes.c_int64(0), ctypes.c_int64(0), None) == usp.USP_ERR_INVALID_ARG
    assert lib.usp_plan_query(None, None, None, None, None) == usp.USP_ERR_INVALID_ARG
    lib.usp_last_error_message.restype = ctypes.c_char_p
    assert b"plan is NULL" in lib.usp_last_error_message()
    lib.usp_debug_wait_timeout.restype = ctypes.c_int
    assert lib.usp_debug_wait_timeout(ctypes.c_uint32(0), None) == usp.USP_ERR_INVALID_ARG


def test_header_compiles_and_links_from_c(usp, tmp_path):
    """include/usp.h is plain C11: the C caller used by the GPU test compiles
    with -Wall -Werror and links against the library (nothing is run here)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    libdir = os.path.dirname(usp.library_path())
    out = tmp_path / "c_abi_block"
    subprocess.run(["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), "-o", str(out), os.path.join(ROOT, "tests", "c_abi_block.c"),
                    "-L", libdir, "-lusp", "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{libdir}"],
                   check=True)
    usage = subprocess.run([str(out)], capture_output=True, text=True)
    assert usage.returncode == 2 and "usage" in usage.stderr


def test_noalloc_scratch_size_matches_header(usp):
    """The binding's copy of the allocation-free scratch size is the header's."""
    import re
    with open(os.path.join(ROOT, "include", "usp.h")) as f:
        m = re.search(r"#define USP_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", f.read())
    assert m, "USP_NOALLOC_SCRATCH_BYTES not found in include/usp.h"
    assert usp.NOALLOC_SCRATCH_BYTES == int(m[1]) * int(m[2]) * int(m[3])

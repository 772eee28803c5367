"""The C ABI from C: tests/c_abi_block.c, compiled with gcc against
include/usp.h and libusp.so, runs scatter_sequence -> the Ulysses block ->
gather_sequence with no Python in the path. Its output is compared with the
float64 definition of attention on the full tensors (the block on P virtual
ranks computes exactly full-sequence attention per head)."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle.attention import attention_bshd
from tests.gpu_util import assert_close
from ulysses_sequence_attention_sp_b200 import build as usp_build
from ulysses_sequence_attention_sp_b200.synth import make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.fail("gcc is needed to build the C caller")
    lib = usp_build.build()
    out = str(tmp_path_factory.mktemp("c_abi") / "c_abi_block")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), "-o", out, os.path.join(HERE, "c_abi_block.c"),
           "-L", libdir, "-lusp", "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True)
    return out


CASES = [  # workload, num_chunks
    (Workload("c1", 1, 333, 0, 6, 64, 3, "fp32", 1.0, 71, (2,)), 2),
    (Workload("c2", 2, 517, 0, 8, 128, 4, "bf16", 1.0, 72, (3,)), 3),
    (Workload("c3", 1, 1000, 0, 5, 128, 5, "bf16", 1.0, 73, (1,)), 1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_block_through_the_c_abi(exe, tmp_path, case):
    w, n = case
    q, k, v = make_qkv(w)
    src, dst = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(src, "wb") as f:
        for x in (q, k, v):
            f.write(np.ascontiguousarray(x).tobytes())
    run = subprocess.run([exe, str(src), str(dst), str(n), str(w.world), str(w.batch), str(w.tokens), str(w.heads),
                          str(w.head_dim), w.dtype], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert run.stdout.startswith("ok"), run.stdout
    storage = np.fromfile(dst, dtype=q.dtype).reshape(q.shape)
    got = storage_to_f64(storage, w.dtype)
    ref = attention_bshd(*(storage_to_f64(x, w.dtype) for x in (q, k, v)))
    assert_close(got, ref, w.dtype, f"{w.name} via C")

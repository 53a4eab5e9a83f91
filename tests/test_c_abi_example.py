"""The C ABI from C: tests/c_abi/psa_from_c.c compiles as C99 against
include/psa.h and links to libpsa.so (CPU); on a GPU it runs the whole path
and writes the same bytes as the Python binding (GPU)."""

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "psa_from_c.c")
CUDA = "/usr/local/cuda"


def _build(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(psa.LIB_PATH):
        pytest.skip("libpsa.so not built")
    exe = str(tmp_path / "psa_from_c")
    libdir = os.path.dirname(psa.LIB_PATH)
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", SRC, "-o", exe, "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), "-L", libdir, "-lpsa", "-Wl,-rpath," + libdir,
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_example_compiles_and_links(tmp_path):
    _build(tmp_path)


@pytest.mark.gpu
def test_c_example_matches_python_binding(tmp_path):
    exe = _build(tmp_path)
    B, H, N, d, density = 1, 2, 24 * 64, 128, 0.25
    q, k, v = make_qkv(B, H, N, d, "clustered", seed=26)
    raw = torch.cat([x.reshape(-1) for x in (q, k, v)]).view(torch.int16).numpy()
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    raw.tofile(fin)
    r = subprocess.run([exe, str(B), str(H), str(N), str(d), str(density), str(fin), str(fout)],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.fromfile(fout, dtype=np.int16)
    out, _ = psa.psa_forward(q.cuda(), k.cuda(), v.cuda(), mode="topk", density=density)
    want = out.cpu().reshape(-1).view(torch.int16).numpy()
    assert np.array_equal(got, want)

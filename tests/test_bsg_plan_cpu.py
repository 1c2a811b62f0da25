"""The closed-form block + strided + global tile plan, checked on the CPU.

The plan (sparse_mask_scaled_b200/csrc/bsg_plan.cuh) is plain integer
arithmetic shared by the host and the GPU kernel. A small driver built from it
with the host compiler lists, for one (b, h), how often every entry (i, j) is
computed by the regular query blocks and the residue-permuted blocks. Against
the oracle's brute-force mask ("Sparse Attention" notes page, pattern list:
block, strided and global tokens) every entry of the mask must be computed
exactly once and nothing else ever, and the rows flagged as having permuted
entries must be exactly those that get some. Parameter corners: with and
without each part, block sizes from 1 to 128, global counts up to 128, and
sequence lengths with fewer or more than 128 positions per residue.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("bsg") / "bsg_plan_probe")
    subprocess.check_call([cxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "sparse_mask_scaled_b200", "csrc"),
                           os.path.join(ROOT, "tests", "bsg_plan_probe.cpp"), "-o", exe])
    return exe


CASES = [
    (16384 // 8, 64, 128, 32), (384, 64, 128, 32), (256, 1, 128, 1), (1024, 32, 128, 0), (1024, 0, 128, 16),
    (1024, 128, 0, 8), (1280, 16, 128, 128), (640, 128, 128, 128), (512, 2, 128, 100), (896, 8, 0, 0),
]


@pytest.mark.parametrize("n,block,stride,ng", CASES)
@pytest.mark.parametrize("chunk", [8, 3])
def test_plan_covers_every_entry_once(probe, n, block, stride, ng, chunk):
    r = subprocess.run([probe, str(n), str(block), str(stride), str(ng), str(chunk)], capture_output=True)
    assert r.returncode == 0, f"probe exit {r.returncode}"
    raw = np.frombuffer(r.stdout, np.uint8)
    assert raw.size == n * n + 2 * n
    cnt = raw[: n * n].reshape(n, n)
    perm_rows, has = raw[n * n: n * n + n], raw[n * n + n:]
    rp, ci = oracle.mask_csr("bsg", n, 1, block=block, stride=stride, n_global=ng)
    want = np.zeros((n, n), np.uint8)
    for i in range(n):
        want[i, ci[rp[i]:rp[i + 1]]] = 1
    bad = np.argwhere(cnt != want)
    assert bad.size == 0, f"{len(bad)} entries wrong, first (i, j) = {tuple(bad[0])}: {cnt[tuple(bad[0])]}"
    assert np.array_equal(perm_rows, has)


@pytest.mark.parametrize("n,block,stride,ng", [(1000, 64, 128, 32), (1024, 48, 128, 32), (1024, 64, 64, 32),
                                               (1024, 64, 128, 129), (1024, 0, 128, 0)])
def test_parameters_outside_the_closed_form_are_refused(probe, n, block, stride, ng):
    r = subprocess.run([probe, str(n), str(block), str(stride), str(ng), "8"], capture_output=True)
    assert r.returncode == 2

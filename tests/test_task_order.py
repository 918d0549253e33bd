"""The persistent kernels' task queues end on any number of resident CTAs.

chol_persist_kernel and sweep_persist_kernel take tasks from one counter in
queue order, and tasks wait (bounded) on counters that other tasks publish.
Every wait ends if each task's waits are met by tasks earlier in the queue.
The two host programs replay the queues with the kernels' own task decoders
(included from the CUDA sources, built as PTX only and never launched).
They check the waits against what earlier tasks published, the order in
which each tile receives its updates, and the final counts.  The factorisation
is checked over every width it takes (n = 384 .. 8064), the sweep over row
blocks x column blocks x group widths.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else shutil.which("nvcc")


@pytest.fixture(scope="module")
def replays(tmp_path_factory):
    nvcc = _nvcc()
    if not nvcc:
        pytest.skip("nvcc is not available")
    out = tmp_path_factory.mktemp("replay")
    procs = {}
    for name in ("replay_factorisation", "replay_sweep"):
        exe = str(out / name)
        cmd = [nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=compute_100a",
               "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
               os.path.join(HERE, name + ".cu"), "-o", exe]
        procs[name] = (exe, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                             text=True))
    exes = {}
    for name, (exe, p) in procs.items():
        log, _ = p.communicate(timeout=600)
        assert p.returncode == 0, log[-2000:]
        exes[name] = exe
    return exes


@pytest.mark.parametrize("name,shapes", [("replay_factorisation", 61), ("replay_sweep", 1860)])
def test_every_wait_is_met_by_earlier_tasks(replays, name, shapes):
    r = subprocess.run([replays[name]], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == f"ok {shapes}"

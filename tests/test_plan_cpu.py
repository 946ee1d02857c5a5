"""The split-KV planner's host-callable arithmetic (worker_of_tile,
worker_begin, for_each_piece in csrc/simt.cuh), compiled from the library's
own header into a host program and run on the CPU (tests/plan_check.cu): tile
coverage, partial-slot numbering, and the next-piece rule of the few-head
attention kernel's Q prefetch, over random batches and worker counts."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_planner_pieces_cover_every_tile_once(tmp_path):
    exe = tmp_path / "plan_check"
    cmd = ["nvcc", "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I" + os.path.join(ROOT, "mla_latent_kv_47_b200", "csrc"), "-I" + os.path.join(ROOT, "include"),
           "-o", str(exe), os.path.join(ROOT, "tests", "plan_check.cu")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr

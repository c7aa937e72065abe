"""Host side of bench.py on the CPU: the multi-rank timing (world-size-2 gloo
processes on 127.0.0.1) and the reference arm's contract line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    # each rank's own device time; the job's time is the slowest rank's
    t = bench.max_over_ranks(0.5 + rank, world, torch.device("cpu"))
    out[rank] = t
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: 1.5, 1: 1.5}


def test_max_over_ranks_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, 1, torch.device("cpu")) == 0.25


def _bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    r = _bench({}, "--impl", "reference", "--steps", "1", "--warmup", "0", "--reference-budget-s", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "scaling", "vs_baseline", "dtype",
                "data", "config"):
        assert key in d, key


@pytest.mark.parametrize("rank", ["1"])
def test_reference_arm_other_ranks_exit_quietly(rank):
    r = _bench({"RANK": rank, "WORLD_SIZE": "2"}, "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_kernel_hash_ignores_comments_only():
    """The recorded decode traffic is used only while the decode kernels'
    code hashes to the recorded value: comment edits keep the hash, code
    edits change it, and no string literal in those files holds a comment
    marker (which would make the comment stripping cut code)."""
    import re
    import shutil

    sys.path.insert(0, ROOT)
    import bench
    from block_quantized_expert_mxfp4_b200 import build as b

    assert bench._code_only("int a; // note\n/* block\n comment */ int b;\n\n") == "int a;\n int b;"
    names = bench.DECODE_KERNEL_FILES
    for n in names:
        for lit in re.findall(r'"(?:[^"\\\n]|\\.)*"', open(os.path.join(b.CSRC, n)).read()):
            assert "//" not in lit and "/*" not in lit, (n, lit)
    tmp = os.path.join(ROOT, "tests", "_build", "hash_check")
    shutil.rmtree(tmp, ignore_errors=True)
    os.makedirs(tmp)
    for n in names:
        shutil.copy(os.path.join(b.CSRC, n), tmp)
    h0 = bench.kernel_source_hash()
    orig = b.CSRC
    try:
        b.CSRC = tmp
        assert bench.kernel_source_hash() == h0
        p = os.path.join(tmp, names[0])
        src = open(p).read()
        open(p, "w").write(src.replace("namespace qk {", "namespace qk {\n// a comment added\n", 1))
        assert bench.kernel_source_hash() == h0
        open(p, "w").write(src.replace("namespace qk {", "namespace qk {\nconstexpr int kUnused = 1;\n", 1))
        assert bench.kernel_source_hash() != h0
    finally:
        b.CSRC = orig
        shutil.rmtree(tmp, ignore_errors=True)

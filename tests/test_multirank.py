"""CPU tests of the benchmark's multi-rank plumbing (gloo, world size 2) and of its reference
leg.  Decode work shards by sequence with no data-path collective, so N ranks run N replicas;
the job's time is the slowest rank's, its throughput the sum of the ranks' bytes over that."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        worst = bench.rank_max(local_ms, world, "cpu")
        gbs = bench.job_throughput(2e9, world, worst)
        dist.barrier()
        out[rank] = (worst, gbs)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_throughput():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    worst, gbs = res[0]
    assert worst == 15.0
    assert gbs == pytest.approx(2 * 2e9 / 15e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench.rank_max(3.5, 1) == 3.5
    assert bench.job_throughput(1e9, 1, 1000.0) == pytest.approx(1.0)


@pytest.mark.slow
def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["unit"] == "GB/s" and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["metric"] == bench.METRIC


def test_kernel_hash_covers_every_decode_source():
    """The roofline's DRAM traffic is looked up by a hash of the decode kernel sources; every
    source of the partial and merge kernels must be part of it, so that a changed kernel never
    reuses a stale capture."""
    import glob
    csrc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "mixed_format_paged_mkv_b200", "csrc")
    decode = {os.path.basename(f) for f in glob.glob(os.path.join(csrc, "decode*"))}
    import inspect
    src = inspect.getsource(bench.kernel_hash)
    missing = [f for f in sorted(decode | {"device_util.cuh", "mkv_internal.h"}) if f not in src]
    assert not missing, missing

"""Multi-process (world size 2, gloo on CPU) tests of the data-parallel
plumbing bench.py uses under torchrun: each rank runs its own batch, the job's
throughput is all ranks' work over the slowest rank's time, every rank takes
the same collective steps, and the reference arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from paged_kv_attention_38_b200 import workloads as W
    # each rank plans its own independent batch
    p = W.gqa_prefill(shard=rank)
    work = bench.attention_flops(p)
    ms = [2.0, 5.0][rank]
    rate, ms_max = bench.job_throughput(work, ms, world, device="cpu")
    lens = p.qo_lens.tolist()
    dist.barrier()
    q.put((rank, work, rate, ms_max, lens))
    dist.destroy_process_group()


def test_job_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    (r0, w0, rate0, ms0, lens0), (r1, w1, rate1, ms1, lens1) = out
    assert lens0 != lens1, "ranks must run different batches"
    assert ms0 == ms1 == 5.0, "time is the slowest rank's"
    expect = (w0 + w1) / 5e-3
    assert abs(rate0 - expect) / expect < 1e-12 and rate0 == rate1


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""

"""Host logic of the multi-GPU benchmark path on CPU ranks (gloo, world 2):
max-over-ranks timing, the weak-scaling job value, and the reference arm
running on rank 0 only. No GPU and no data-path collective are involved."""
import io
import os
import socket
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 40.0][rank]
        ms = bench.max_over_ranks(dist, local_ms, device="cpu")
        value = bench.job_value(world, 1e12, ms)
        buf = io.StringIO()

        class Args:
            steps, warmup, gpus, workload = 1, 0, world, "swa"
            oracle_table, no_graph, layers, batch, seq = False, False, None, None, None
        os.environ["MIMO_REF_STEP_SECONDS"] = "0.2"
        with contextlib.redirect_stdout(buf):
            bench.run_reference(Args())
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms} {value} {len(buf.getvalue().strip())}\n")
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_reference_on_rank0(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = open(tmp_path / "rank0.txt").read().split()
    r1 = open(tmp_path / "rank1.txt").read().split()
    assert float(r0[0]) == 40.0 and float(r1[0]) == 40.0       # slowest rank sets the step time
    assert float(r0[1]) == pytest.approx(2 * 1e12 / 0.040 / 1e12)  # both ranks' units / max time
    assert int(r0[2]) > 0 and int(r1[2]) == 0                  # only rank 0 prints the reference line

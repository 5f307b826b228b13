"""The multi-rank path of bench.py on the CPU: two gloo ranks (spawned processes, rendezvous
on 127.0.0.1) agree on the maximum of their per-rank times, the rank environment is read as
torchrun sets it, and under several ranks only rank 0 runs the reference arm. No GPU."""
import importlib.util
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    bench = _load_bench()
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        env = bench.rank_env()
        mx = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        # the reference arm: ranks other than 0 return at once and print nothing
        printed = io.StringIO()
        rc = None
        if rank != 0:
            with redirect_stdout(printed):
                rc = bench.run_reference(None)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"env": env, "max": mx, "rc": rc, "printed": printed.getvalue()}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["env"] == [r, r, world]
        assert d["max"] == 15.0                      # the slowest rank's time, on every rank
    assert res[1]["rc"] == 0 and res[1]["printed"] == ""


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    bench = _load_bench()
    assert bench.rank_env() == (0, 0, 1)
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5

"""The N > 1 host logic of bench.py (replicas only: no collective on the data path),
run as two gloo ranks on the CPU: distinct per-rank inputs, max-over-ranks timing, the
whole-job rate, and the reference arm running on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    import dit_synth as S
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    w, r, _ = bench.dist_setup()
    cfg = bench.CFG
    x = S.make_inputs(cfg, seed=bench.replica_seed(cfg, r))["x"]
    slow = [3.0, 5.0][r]                                  # per-rank "time" of the timed region
    tmax = bench.max_over_ranks(slow, w)
    rate = bench.aggregate_rate(100.0, w, 10, tmax)

    class A:                                              # the reference arm's arguments
        steps, warmup, gpus = 1, 0, w
    buf = io.StringIO()
    if r != 0:
        with redirect_stdout(buf):
            rc = bench.run_reference(A)                   # non-zero ranks leave without work
    else:
        rc = 0
    dist.barrier()
    dist.destroy_process_group()
    np.save(os.path.join(outdir, f"x{r}.npy"), x)
    with open(os.path.join(outdir, f"r{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "tmax": tmax, "rate": rate, "ref_rc": rc, "ref_out": buf.getvalue()}, f)


def test_two_gloo_ranks_replicas(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert [q["world"] for q in res] == [2, 2] and [q["rank"] for q in res] == [0, 1]
    assert all(q["tmax"] == 5.0 for q in res)             # every rank sees the slowest rank's time
    assert all(abs(q["rate"] - 100.0 * 2 * 10 / 5.0) < 1e-9 for q in res)
    assert res[1]["ref_rc"] == 0 and res[1]["ref_out"] == ""
    x0, x1 = np.load(tmp_path / "x0.npy"), np.load(tmp_path / "x1.npy")
    assert x0.shape == x1.shape and not np.array_equal(x0, x1)   # each replica has its own latents

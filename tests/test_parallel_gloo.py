"""The multi-rank path on CPU with gloo, world size 2: every rank draws its own
token batch with the same weights, runs the layer (here the fp64 oracle, as
there is no GPU in this test), and the job's time is the maximum over ranks;
the reference arm does its work on rank 0 only."""
import json
import os
import socket
import subprocess
import sys
import time

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_mixture_experts_renorm_b200 import parallel as par
    from sparse_mixture_experts_renorm_b200.workloads import WORKLOADS, make_inputs, make_tokens

    par.init("gloo", 60.0)
    w, r, _ = par.env_ranks()
    wl = WORKLOADS["tiny_f32"]
    inp = make_inputs(wl, "cpu", 0)
    x = make_tokens(wl, wl.T, "cpu", seed=par.batch_seed(r))
    par.barrier()
    t0 = time.perf_counter()
    res = oracle.forward(x, inp.w_router, None, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    dt = time.perf_counter() - t0 + 0.05 * r  # ranks finish at different times
    mx = par.max_over_ranks(dt)
    par.barrier()
    with open(os.path.join(outdir, f"r{r}.json"), "w") as f:
        json.dump({"dt": dt, "max": mx, "x00": float(x[0, 0]), "wsum": float(inp.w_gate.double().sum()),
                   "counts": int(res.counts.sum()), "tokens": par.job_tokens(wl.T, w, 3)}, f)
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_time(tmp_path):
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    a, b = (json.load(open(tmp_path / f"r{i}.json")) for i in range(2))
    assert a["max"] == b["max"] == max(a["dt"], b["dt"])
    assert a["x00"] != b["x00"], "each rank draws its own batch"
    assert a["wsum"] == b["wsum"], "every rank holds the same weights"
    assert a["counts"] == b["counts"] == 64 * 2
    assert a["tokens"] == 2 * 64 * 3


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    from sparse_mixture_experts_renorm_b200 import parallel as par

    assert par.max_over_ranks(3.5) == 3.5
    par.barrier()
    assert par.job_tokens(4096, 1, 10) == 40960


def test_reference_arm_works_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""

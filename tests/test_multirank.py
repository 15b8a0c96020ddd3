"""The benchmark's multi-rank host logic on CPU (gloo, world size 2): process
group set-up from the launcher's environment, the barrier, the max-over-ranks
timing reduction, independent inputs per rank (weak scaling, no data-path
collective), and the reference arm running on rank 0 only."""
import os
import socket
import subprocess
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import qsa_inputs as Q
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    assert torch.distributed.get_backend() == "gloo"
    bench.barrier(w)
    # each rank reports a different time; every rank receives the slowest
    ms = bench.max_over_ranks(10.0 + 7.5 * rank, w)
    # per-rank inputs: the same workload recipe, an independent sequence
    P = Q.PrefillProblem(T=64, seed=bench.rank_seed(0, r), n_plant=2)
    D = Q.DecodeProblem(B=2, L=32, steps=1, seed=bench.rank_seed(0, r), n_plant=2)
    digest = torch.tensor([float(P.q_idx(0, 8).astype(np.float64).sum()),
                           float(D.cache_kidx(0, 0, 8).astype(np.float64).sum())], dtype=torch.float64)
    all_d = [torch.zeros_like(digest) for _ in range(w)]
    torch.distributed.all_gather(all_d, digest)
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([ms] + [float(x) for d in all_d for x in d]))


def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [np.load(tmp_path / f"r{r}.npy") for r in range(world)]
    for r in range(world):
        assert res[r][0] == 17.5, "max over ranks"
        assert np.array_equal(res[r], res[0]), "every rank sees the same reduced values"
    d0, d1 = res[0][1:3], res[0][3:5]
    assert not np.array_equal(d0, d1), "ranks must draw independent sequences"


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0
    assert p.stdout.strip() == ""

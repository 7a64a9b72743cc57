"""bench.py's multi-rank plumbing over two gloo ranks on CPU: the step time every rank
reports is the maximum over ranks, and each rank draws its own seed (weak scaling)."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.0 + rank * 2.5, world, "cpu")
        bench.barrier(world)
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([got, bench.rank_seed(1002, rank)]))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank_seeds(tmp_path):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.spawn(_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r0, r1 = np.load(tmp_path / "r0.npy"), np.load(tmp_path / "r1.npy")
    assert r0[0] == r1[0] == 3.5          # the slowest rank's time, on every rank
    assert r0[1] != r1[1]                 # independent batches per rank
    assert bench.max_over_ranks(2.0, 1, "cpu") == 2.0


def test_kernel_hash_ignores_comments_not_code():
    """The traffic figures are keyed to the kernels' code: comment and layout edits keep the
    hash, a code edit changes it, and comment markers inside literals are code."""
    import bench

    base = 'int f(int x) { return x + 1; } // one\n/* two */ const char *s = "a // b /* c */";\n'
    same = '/* lead */\nint f(int x)   {\n  return x + 1;  // changed comment\n}\nconst char *s = "a // b /* c */";'
    other = 'int f(int x) { return x + 2; }\nconst char *s = "a // b /* c */";'
    lit = 'int f(int x) { return x + 1; }\nconst char *s = "a // b";'

    def norm(src):
        return " ".join(bench.strip_comments(src).split())

    assert norm(base) == norm(same)
    assert norm(base) != norm(other)
    assert norm(base) != norm(lit)
    assert "'/'" in bench.strip_comments("char c = '/'; // x")


def test_backward_cpu_baseline_runs_on_a_small_sample():
    """bench.py's CPU baseline for the backward leg (the oracle timed on a bounded sample)."""
    import numpy as np
    import torch

    import bench
    from chunked_linear_attention_chunk_b200 import synth

    x = synth.make_inputs(1, 96, 2, 16, 16, "bf16", seed=5, s0_std=0.1)
    dO = torch.from_numpy(np.random.default_rng(5).normal(size=(1, 96, 2, 16)).astype(np.float32)).to(torch.bfloat16)
    r = bench.cpu_baseline_bwd(x, dO, 64)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    assert "first 64 of 96 tokens" in r["sample"]

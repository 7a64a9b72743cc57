"""The sequence-parallel orchestration over two gloo ranks on CPU: each rank holds half of
one sequence; the exchange of affine maps and the prefix combine must give every rank the
outputs of its half and the final state of one run over the whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from chunked_linear_attention_chunk_b200 import synth
from chunked_linear_attention_chunk_b200.sp import sp_chunk_fwd
from sp_oracle_ops import NAMES, OracleSegmentOps

B, T, H, D = 1, 90, 2, 16
CUT = [0, 37, 90]  # rank r holds tokens CUT[r] .. CUT[r+1]


def _inputs():
    return synth.make_inputs(B, T, H, D, D, "f32", seed=1300, s0_std=0.2)


def _rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _inputs()
        seg = [x[n][:, CUT[rank]:CUT[rank + 1]] for n in NAMES]
        o, S_T = sp_chunk_fwd(*seg, S0=x["S0"].double(), ops=OracleSegmentOps())
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"s{rank}.npy"), S_T.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_match_one_sequence(tmp_path):
    mp.spawn(_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    x = _inputs()
    o_ref, S_ref = oracle.recurrence(*(x[n].numpy() for n in NAMES), -5.0, S0=x["S0"].numpy().astype(np.float64))
    for r in range(2):
        o = np.load(tmp_path / f"o{r}.npy")
        assert np.allclose(o, o_ref[:, CUT[r]:CUT[r + 1]], rtol=1e-9, atol=1e-12), r
        assert np.allclose(np.load(tmp_path / f"s{r}.npy"), S_ref, rtol=1e-9, atol=1e-12), r

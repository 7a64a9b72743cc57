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


def _rank_bwd(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from chunked_linear_attention_chunk_b200.sp import sp_chunk_bwd
        x = _inputs()
        dO, dST = _grads()
        seg = [x[n][:, CUT[rank]:CUT[rank + 1]] for n in NAMES]
        g = sp_chunk_bwd(*seg, dO[:, CUT[rank]:CUT[rank + 1]], S0=x["S0"].double(), dS_T=dST,
                         ops=OracleSegmentOps())
        for n, t in g.items():
            if t is not None:
                np.save(os.path.join(out_dir, f"{n}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def _grads():
    rng = np.random.default_rng(1301)
    dO = torch.from_numpy(rng.normal(size=(B, T, H, D)).astype(np.float32))
    dST = torch.from_numpy(rng.normal(size=(B, H, D, D)))
    return dO, dST


def test_two_ranks_backward_match_one_sequence(tmp_path):
    """The sequence-parallel backward: each rank's token gradients equal the slice of one
    backward over the whole sequence, and every rank returns the whole sequence's dS0."""
    mp.spawn(_rank_bwd, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    x = _inputs()
    dO, dST = _grads()
    ref = oracle.backward(*(x[n].numpy() for n in NAMES), dO.numpy(), -5.0, S0=x["S0"].numpy().astype(np.float64),
                          dST=dST.numpy())
    for r in range(2):
        for n in ("dq", "dk", "dv", "da", "dbeta"):
            got = np.load(tmp_path / f"{n}{r}.npy")
            assert np.allclose(got, ref[n][:, CUT[r]:CUT[r + 1]], rtol=1e-8, atol=1e-11), (r, n)
        assert np.allclose(np.load(tmp_path / f"dS0{r}.npy"), ref["dS0"], rtol=1e-8, atol=1e-11), r


def test_one_rank_backward_is_the_plain_backward():
    from chunked_linear_attention_chunk_b200.sp import sp_chunk_bwd
    x = _inputs()
    dO, dST = _grads()
    g = sp_chunk_bwd(*(x[n] for n in NAMES), dO, S0=x["S0"].double(), dS_T=dST, ops=OracleSegmentOps())
    ref = oracle.backward(*(x[n].numpy() for n in NAMES), dO.numpy(), -5.0, S0=x["S0"].numpy().astype(np.float64),
                          dST=dST.numpy())
    for n in ref:
        assert np.allclose(g[n].numpy(), ref[n], rtol=1e-9, atol=1e-12), n


CUT3 = [0, 50, 50, 90]  # three ranks, the middle one with an empty segment


def _rank_bwd3(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from chunked_linear_attention_chunk_b200.sp import sp_chunk_bwd
        x = _inputs()
        dO, dST = _grads()
        seg = [x[n][:, CUT3[rank]:CUT3[rank + 1]] for n in NAMES]
        g = sp_chunk_bwd(*seg, dO[:, CUT3[rank]:CUT3[rank + 1]], S0=x["S0"].double(), dS_T=dST,
                         ops=OracleSegmentOps())
        for n, t in g.items():
            if t is not None:
                np.save(os.path.join(out_dir, f"{n}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def test_three_ranks_backward_with_an_empty_segment(tmp_path):
    mp.spawn(_rank_bwd3, args=(3, _free_port(), str(tmp_path)), nprocs=3, join=True)
    x = _inputs()
    dO, dST = _grads()
    ref = oracle.backward(*(x[n].numpy() for n in NAMES), dO.numpy(), -5.0, S0=x["S0"].numpy().astype(np.float64),
                          dST=dST.numpy())
    for r in range(3):
        for n in ("dq", "dk", "dv", "da", "dbeta"):
            got = np.load(tmp_path / f"{n}{r}.npy")
            assert got.shape[1] == CUT3[r + 1] - CUT3[r]
            assert np.allclose(got, ref[n][:, CUT3[r]:CUT3[r + 1]], rtol=1e-8, atol=1e-11), (r, n)
        assert np.allclose(np.load(tmp_path / f"dS0{r}.npy"), ref["dS0"], rtol=1e-8, atol=1e-11), r

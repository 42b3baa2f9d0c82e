"""Multi-rank host logic on CPU (gloo, world size 2): head and sequence
sharding cover every (sequence, head) chain exactly once, and per-rank results
assembled from the shards equal one run over everything (checked with the
oracle, which is the same whoever computes a chain), and the slowest-rank
timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_103_b200 import inputs
from gated_delta_rule_103_b200.sharding import (balance_sequences, head_range, max_over_ranks,
                                                 slice_heads)


def test_head_range_partitions():
    for H in (1, 2, 7, 32, 33):
        for world in (1, 2, 3, 8):
            got = [head_range(H, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            for (a0, a1), (b0, b1) in zip(got, got[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1


def test_balance_sequences():
    lengths = inputs.varlen_lengths(16, 1024, 32768, seed=1004)
    for world in (1, 2, 4, 8):
        parts = balance_sequences(lengths, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(lengths)))
        loads = [sum(lengths[i] for i in p) for p in parts]
        # greedy longest-first: spread at most one sequence's length
        assert max(loads) - min(loads) <= max(lengths)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = inputs.prefill_inputs(1, 70, 5, dk=8, dv=6, dtype=torch.float32, seed=3,
                                  init_std=0.1)
        h0, h1 = head_range(x["H"], world, rank)
        y = slice_heads(x, h0, h1)
        out, fs = oracle.kda_forward(y["q"], y["k"], y["v"], y["log_alpha"], y["beta"],
                                     initial_state=y["initial_state"], scale=x["scale"])
        # the backward pass shards the same way: the adjoints of a rank's heads
        d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), 1, x["H"], 8, 6,
                                              dtype=torch.float32, seed=4)
        grads = oracle.kda_backward(y["q"], y["k"], y["v"], y["log_alpha"], y["beta"],
                                    d_out[:, :, h0:h1], initial_state=y["initial_state"],
                                    d_final_state=dfs[:, h0:h1], scale=x["scale"])
        # gather the per-rank shards (test-only assembly; the operator needs none)
        gathered = [None] * world
        dist.all_gather_object(gathered, (h0, h1, out, fs, grads))
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            results["shards"] = gathered
            results["max"] = t
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharding_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    x = inputs.prefill_inputs(1, 70, 5, dk=8, dv=6, dtype=torch.float32, seed=3, init_std=0.1)
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"])
    shards = results["shards"]
    out = np.concatenate([s[2] for s in sorted(shards, key=lambda s: s[0])], axis=2)
    fs = np.concatenate([s[3] for s in sorted(shards, key=lambda s: s[0])], axis=1)
    np.testing.assert_array_equal(out, o_ref)
    np.testing.assert_array_equal(fs, f_ref)
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), 1, x["H"], 8, 6,
                                          dtype=torch.float32, seed=4)
    g_ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_out,
                                initial_state=x["initial_state"], d_final_state=dfs,
                                scale=x["scale"])
    head_axis = (2, 2, 2, 2, 2, 1)   # dq dk dv dlog_alpha dbeta d_initial_state
    ordered = sorted(shards, key=lambda s: s[0])
    for i, (ax, ref) in enumerate(zip(head_axis, g_ref)):
        got = np.concatenate([s[4][i] for s in ordered], axis=ax)
        np.testing.assert_array_equal(got, ref)
    assert results["max"] == 2.0


# ---------------------------------------------------------------- sequence parallelism
def test_token_range_partitions():
    from gated_delta_rule_103_b200.sharding import token_range
    for T in (1, 63, 64, 65, 1000, 4096):
        for world in (1, 2, 3, 8):
            got = [token_range(T, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == T
            for (a0, a1), (b0, b1) in zip(got, got[1:]):
                assert a1 == b0
            # every boundary but the sequence's end falls on a whole chunk
            assert all(a % 64 == 0 or a == T for a, _ in got)


def _oracle_ops():
    """The compute steps of a sequence-parallel prefill done by the oracle in
    fp64 (the transition: the recurrence from the identity with v = 0)."""
    from gated_delta_rule_103_b200.sharding import RangeOps

    def fwd(q, k, v, g, b, s0):
        o, f = oracle.kda_forward(q, k, v, g, b, initial_state=s0, scale=0.3)
        return torch.from_numpy(o), torch.from_numpy(f)

    def trans(q, k, g, b):
        B, T, H, dk = k.shape
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, m = oracle.kda_forward(q, k, np.zeros((B, T, H, dk)), g, b, initial_state=eye, scale=0.3)
        return torch.from_numpy(m)

    def affine(m, b, s):
        return torch.einsum("nhij,nhjk->nhik", m, s) + b

    return RangeOps(fwd, trans, affine)


def _seq_worker(rank, world, port, results):
    from gated_delta_rule_103_b200.sharding import (sequence_parallel_chunk_fwd, token_range,
                                                     torch_all_gather)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = inputs.prefill_inputs(2, 300, 3, dk=6, dv=6, dtype=torch.float64, seed=21,
                                  init_std=0.5, u_lo=-7.0, u_hi=-4.0)
        t0, t1 = token_range(x["T"], world, rank)
        sl = {n: x[n][:, t0:t1].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
        out, fs = sequence_parallel_chunk_fwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"],
                                              sl["beta"], x["initial_state"], rank, world,
                                              torch_all_gather(), _oracle_ops())
        gathered = [None] * world
        dist.all_gather_object(gathered, (t0, out.numpy(), fs.numpy()))
        if rank == 0:
            results["parts"] = gathered
    finally:
        dist.destroy_process_group()


def test_three_rank_sequence_parallel_gloo():
    """A sequence batch split by tokens over three gloo ranks: the assembled
    outputs and the last rank's exit state equal one oracle run over all
    tokens (fp64; the slow gate keeps the transitions far from zero)."""
    world = 3
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_seq_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    x = inputs.prefill_inputs(2, 300, 3, dk=6, dv=6, dtype=torch.float64, seed=21, init_std=0.5,
                              u_lo=-7.0, u_hi=-4.0)
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=0.3)
    parts = sorted(results["parts"], key=lambda p: p[0])
    out = np.concatenate([p[1] for p in parts], axis=1)
    np.testing.assert_allclose(out, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(parts[-1][2], f_ref, rtol=1e-10, atol=1e-12)
    # the transitions matter: the last range run from a zero state is far off
    from gated_delta_rule_103_b200.sharding import token_range
    t0, _ = token_range(x["T"], world, world - 1)
    _, f_zero = oracle.kda_forward(*(x[n][:, t0:] for n in ("q", "k", "v", "log_alpha", "beta")),
                                   scale=0.3)
    assert np.linalg.norm(f_zero - f_ref) > 1e-2 * np.linalg.norm(f_ref)

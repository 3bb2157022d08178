"""Data-parallel host logic on CPU: two gloo ranks, each with its own token
shard, combine their outlier column maxima through ColmaxExchange; the
result (and the momentum state built from it) must equal the unsharded
batch's bit for bit (Quaff notes, 目标动量缩放: the statistic is a max over
the step's tokens, exact and order-free)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from quantized_linear_layers_token_b200 import synth
from quantized_linear_layers_token_b200.dp import ColmaxExchange


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shards, n_outliers, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = ColmaxExchange(n_outliers)
        for j, (Xs, O) in enumerate(shards[rank]):
            if len(O) and len(Xs):
                col = np.abs(Xs[:, O].astype(np.float32)).max(axis=0)
                x.view(j).copy_(torch.from_numpy(col))
        x.allreduce()
        q.put((rank, x.buf.numpy().copy()))
    finally:
        dist.destroy_process_group()


def _layers():
    """Three layers of the small and decode recipes (one with no outliers)."""
    out = []
    wl = synth.WORKLOADS["llama7b_w4_decode"]
    for si, M in [(0, 13), (6, 5)]:
        L = synth.layer(wl, si, M=M)
        out.append((L["X"], np.asarray(L["O"], np.int32), L["W"]))
    Ls = synth.layer(synth.WORKLOADS["small"], 0, M=16)
    out.append((Ls["X"], np.zeros(0, np.int32), Ls["W"]))
    return out


def test_colmax_exchange_two_ranks(oracle):
    layers = _layers()
    world = 2
    # uneven shards: rank 0 gets the first row only, rank 1 the rest
    shards = [[(X[:1], O) for X, O, _ in layers], [(X[1:], O) for X, O, _ in layers]]
    n_out = [len(O) for _, O, _ in layers]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shards, n_out, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, buf = q.get(timeout=120)
        got[r] = buf
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    np.testing.assert_array_equal(got[0], got[1])
    ex = ColmaxExchange(n_out)
    for j, (X, O, W) in enumerate(layers):
        red = got[0][ex.offsets[j]:ex.offsets[j] + len(O)]
        full = np.abs(X[:, O].astype(np.float32)).max(axis=0) if len(O) else np.zeros(0, np.float32)
        np.testing.assert_array_equal(red, full)
        if not len(O):
            continue
        # the recurrence applied to the exchanged maxima equals the update
        # over the whole batch (a one-row input carrying the maxima)
        Xb = np.ascontiguousarray(X).view(np.uint16)
        Wb = np.ascontiguousarray(W).view(np.uint16)
        wmax = oracle.outlier_wmax(Wb, O)
        s0 = np.full(len(O), 1.25, np.float32)
        s_full = oracle.momentum_update(Xb, O, wmax, 0.9, s0)
        row = np.zeros((1, X.shape[1]), np.float16)
        row[0, O] = red.astype(np.float16)  # maxima of fp16 values are fp16 values
        s_dp = oracle.momentum_update(row.view(np.uint16), O, wmax, 0.9, s0)
        np.testing.assert_array_equal(s_dp, s_full)


def test_exchange_layout_and_single_process_noop():
    ex = ColmaxExchange([3, 0, 5])
    assert ex.offsets == [0, 3, 3] and ex.total == 8
    ex.view(2).fill_(2.0)
    ex.view(0).fill_(1.0)
    ex.allreduce()  # no process group: nothing to combine
    assert ex.buf.tolist() == [1.0] * 3 + [2.0] * 5
    assert ex.view(1).numel() == 0
    with pytest.raises(ValueError):
        ColmaxExchange([-1])

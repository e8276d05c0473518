"""Multi-rank host logic on CPU: two gloo ranks (127.0.0.1), no GPU.

The path shards with no collective on the data path: by batch (every rank its
own sequences) or by KV heads (every rank its slice of the one batch, as
tensor-parallel attention).  These tests run the oracle on each rank's shard
and check that the shards, put together, are exactly the single-process
result, and that the timing reduction takes the slowest rank.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from hierarchical_long_context_b200 import synth
from tests import lodtest as lt

WORKLOAD = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hkv=4, Hq=16, T=2048)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _decode_oracle(w):
    """Oracle decode of every (sequence, query head) of workload w at t = T - 1:
    out [B, Hq, d] float64, selected groups [B, Hq, top_groups]."""
    K, V = synth.kv_cache(w, threads=2)
    q = synth.decode_queries(w).float().numpy()
    cfg = lt.oracle_cfg(w)
    out = np.empty((w.B, w.Hq, w.d))
    sel = np.empty((w.B, w.Hq, w.top_groups), np.int32)
    for b in range(w.B):
        for h in range(w.Hkv):
            Kh, Vh = K[b, h].float().numpy(), V[b, h].float().numpy()
            # the k-means initialisation's model-wide sequence-head index
            unit = b * (w.hkv_model or w.Hkv) + w.kvh0 + h
            ix = oracle.build_sequence(cfg, unit, Kh, Vh, w.T // 256)
            for j in range(w.g):
                hq = h * w.g + j
                o, _, sg, _, _ = oracle.attend_row(cfg, q[b, hq], w.T - 1, Kh, Vh, ix)
                out[b, hq], sel[b, hq] = o, sg
    return out, sel


def _rank(rank, world, port, mode, q):
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        w = synth.shard(WORKLOAD, mode, rank, world)
        out, sel = _decode_oracle(w)
        outs = [None] * world
        dist.all_gather_object(outs, (w.kvh0, w.Hkv, w.seed, out, sel))
        slowest = bench.dist_max(float(rank + 1) * 0.25, world, device="cpu")
        if rank == 0:
            q.put((outs, slowest))
    finally:
        dist.destroy_process_group()


def _run(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = q.get(timeout=300)
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


def test_head_shards_reassemble_the_single_process_decode():
    outs, slowest = _run("heads")
    assert slowest == 0.5
    # the two ranks hold disjoint, consecutive KV-head slices covering all heads
    assert [(o[0], o[1]) for o in outs] == [(0, 2), (2, 2)]
    out = np.concatenate([o[3] for o in outs], axis=1)
    sel = np.concatenate([o[4] for o in outs], axis=1)
    ref_out, ref_sel = _decode_oracle(WORKLOAD)
    np.testing.assert_array_equal(out, ref_out)
    np.testing.assert_array_equal(sel, ref_sel)


def test_batch_shards_are_independent_replicas():
    outs, slowest = _run("batch")
    assert slowest == 0.5
    assert [o[2] for o in outs] == [WORKLOAD.seed, WORKLOAD.seed + 1]
    assert all(o[1] == WORKLOAD.Hkv for o in outs)
    assert not np.array_equal(outs[0][3], outs[1][3])
    ref_out, _ = _decode_oracle(WORKLOAD)
    np.testing.assert_array_equal(outs[0][3], ref_out)

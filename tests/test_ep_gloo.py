"""The expert-parallel split on CPU: two gloo ranks, each computing its own
experts' part of a layer with the fp64 oracle (one expert at a time), summed
by an all-reduce; the sum must be the whole layer's expert output m, and the
ranks' expert blocks must cover every expert once."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from int4_routed_expert_02_b200 import synth
from int4_routed_expert_02_b200.ep import expert_range, shared_owner


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_part(OL, xe, idx, w, e_lo, e_hi, with_shared):
    T, H = xe.shape
    m = np.zeros((T, H))
    for t in range(T):
        for s in range(idx.shape[1]):
            e = int(idx[t, s])
            if e_lo <= e < e_hi:
                m[t] += w[t, s] * oracle.expert(OL, e, xe[t])
        if with_shared:
            m[t] += oracle.expert(OL, -1, xe[t])
    return m


def _worker(rank, world, port, layer, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = synth.CONFIGS[0]
        w = synth.gen_layer(cfg, 0, layer)
        OL = oracle.OracleLayer.from_config(w, cfg)
        h = synth.gen_hidden(cfg, 0, 77, cfg.T)
        _, idx, wt, xn = oracle.router(OL, h)
        xe = oracle.bf16_to_f64(oracle.f64_to_bf16(xn))
        e_lo, e_hi = expert_range(cfg.E, world, rank)
        part = torch.from_numpy(_rank_part(OL, xe, idx, wt, e_lo, e_hi, shared_owner(layer, world) == rank))
        dist.all_reduce(part)
        if rank == 0:
            full = oracle.expert_ffn(OL, xe, idx, wt)
            q.put((part.numpy(), full, [expert_range(cfg.E, world, r) for r in range(world)]))
    finally:
        dist.destroy_process_group()


def _run(world, layer):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, layer, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return got


def test_two_ranks_sum_to_the_whole_layer():
    for layer in (0, 1):   # the shared expert belongs to rank 0, then to rank 1
        m, full, ranges = _run(2, layer)
        rms = float(np.sqrt(np.mean(full * full)))
        assert np.max(np.abs(m - full)) <= 1e-12 * rms
        covered = sorted(e for lo, hi in ranges for e in range(lo, hi))
        assert covered == list(range(synth.CONFIGS[0].E))


def test_expert_ranges_partition_every_expert_count():
    for E in (8, 16, 128, 257, 512):
        for world in (1, 2, 3, 4, 8):
            rs = [expert_range(E, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == E
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [hi - lo for lo, hi in rs]
            assert max(sizes) - min(sizes) <= 1
    assert [shared_owner(l, 4) for l in range(6)] == [0, 1, 2, 3, 0, 1]

"""The data-parallel path on CPU: two gloo ranks, each with a shard of whole
sequences, reproduce the single-process hash indices and, after the
all-reduce, the weight gradients of the whole batch (oracle arithmetic)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from engram_conditional_memory_hash_b200 import dp, inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = oracle.default()
        o.set_threads(1)
        w = inputs.Workload("dp", 80, B=5, S=16, H=64, backward=True, ids="uniform",
                            id_high=50, prime_base=4099, D=32)
        h = inputs.hash_inputs(w, with_tables=False)
        gi = inputs.gate_inputs(w)
        a, b = dp.shard_sequences(w.B, world, rank)
        idx = o.engram_hash(h["tokens"][a:b], h["multipliers"], h["ngram_n"], h["table_sizes"],
                            pad_id=h["pad_id"])
        rows = slice(a * w.S, b * w.S)
        res = o.engram_gate_bwd(gi["g"][rows], gi["x"][rows], gi["k"][rows], gi["v"][rows],
                                gi["wh"], gi["we"], per_token=False)
        dw = torch.from_numpy(np.stack([res["dwh"], res["dwe"]]))
        dp.allreduce_weight_grads(dw)
        q.put((rank, a, b, idx, dw.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_match_single_process(oracle_lib):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    w = inputs.Workload("dp", 80, B=5, S=16, H=64, backward=True, ids="uniform", id_high=50,
                        prime_base=4099, D=32)
    h = inputs.hash_inputs(w, with_tables=False)
    gi = inputs.gate_inputs(w)
    full_idx = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"],
                                      h["table_sizes"], pad_id=h["pad_id"])
    np.testing.assert_array_equal(np.concatenate([g[3] for g in got]), full_idx)
    full = oracle_lib.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"],
                                      per_token=False)
    for g in got:
        np.testing.assert_allclose(g[4][0], full["dwh"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g[4][1], full["dwe"], rtol=1e-12, atol=1e-12)


def test_shard_bounds_cover_every_sequence_once():
    for n in range(0, 12):
        for world in range(1, 5):
            spans = [dp.shard_sequences(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1

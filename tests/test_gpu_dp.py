"""The data-parallel path through the CUDA library: two ranks (processes) on
cuda:0, joined by a gloo process group, each run the benchmark's step
(EngramStep: engram_hash_gather, engram_gate_fwd, engram_gate_bwd_fused and
the all-reduce of the [2, H] weight gradient, dp.allreduce_weight_grads) on
its shard of whole sequences of one batch.  Together they must reproduce the
oracle on the whole batch: every hash index and gathered row bit for bit,
every per-token gate output within the parity tolerances, and on every rank
the all-reduced dwh, dwe of all tokens.

The ranks share one GPU only for this test; their kernels never wait on each
other (the exchange is gloo's, through host memory)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from engram_conditional_memory_hash_b200 import inputs

pytestmark = pytest.mark.gpu

WORLD = 2
W = inputs.Workload("dp_gpu", 95, B=5, S=256, H=4096, backward=True, ids="zipf", vocab=129280,
                    prime_base=4099, D=32)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _worker(rank, port, q):
    import torch.distributed as dist

    from engram_conditional_memory_hash_b200 import dp, step
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=120))
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        h = inputs.hash_inputs(W)
        gi = inputs.gate_inputs(W)
        a, b = dp.shard_sequences(W.B, WORLD, rank)
        rows = slice(a * W.S, b * W.S)

        def bf(arr):
            return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(
                torch.bfloat16).to(dev)

        st = step.EngramStep(b - a, W.S, W.H, dev, bf(h["tables"]).view(-1, W.D), bf(gi["wh"]),
                             bf(gi["we"]), h["multipliers"], h["ngram_n"], h["table_sizes"],
                             pad_id=h["pad_id"], eps=W.eps)
        buf = st.buffers()
        buf.tokens.copy_(torch.from_numpy(h["tokens"][a:b]))
        for n in ("x", "k", "v", "g"):
            getattr(buf, n).copy_(bf(gi[n][rows]))
        stream = torch.cuda.current_stream(dev)
        st.run(buf, stream)
        torch.cuda.synchronize(dev)
        q.put((rank, a, b, buf.idx.cpu().numpy(), _bits(buf.rows), _bits(buf.out),
               buf.gate.cpu().numpy(), _bits(buf.dx), _bits(buf.dk), _bits(buf.dv),
               buf.dw.cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_on_the_library_match_the_oracle(oracle_lib):
    from parity import assert_bf16_close, assert_dw_close, assert_gate_close, ill_conditioned
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=600) for _ in range(WORLD))
    finally:
        for p in procs:
            p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)

    h = inputs.hash_inputs(W)
    gi = inputs.gate_inputs(W)
    T, H = W.T, W.H
    assert [g[1] for g in got] == [0, got[0][2]] and got[-1][2] == W.B

    want_idx = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"],
                                      h["table_sizes"], pad_id=h["pad_id"])
    np.testing.assert_array_equal(np.concatenate([g[3] for g in got]), want_idx)
    want_rows = oracle_lib.engram_gather(want_idx, h["table_sizes"], h["tables"], W.D)
    np.testing.assert_array_equal(np.concatenate([g[4] for g in got]).reshape(want_rows.shape),
                                  want_rows)

    def cat(i):
        return torch.from_numpy(np.concatenate([g[i] for g in got]).view(np.int16)).view(
            torch.bfloat16).reshape(T, H)

    ref_out, ref_gate = oracle_lib.engram_gate_fwd(gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    ref = oracle_lib.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    ill = ill_conditioned(ref["s"])
    assert_bf16_close("out", cat(5), ref_out)
    assert_gate_close(torch.from_numpy(np.concatenate([g[6] for g in got])), ref_gate)
    assert_bf16_close("dx", cat(7), ref["dx"], rows_relaxed=ill)
    assert_bf16_close("dk", cat(8), ref["dk"], rows_relaxed=ill)
    assert_bf16_close("dv", cat(9), ref["dv"])
    for g in got:     # every rank holds the all-reduced gradient of the whole batch
        assert_dw_close("dwh", torch.from_numpy(g[10][0]), ref["dwh"])
        assert_dw_close("dwe", torch.from_numpy(g[10][1]), ref["dwe"])
    np.testing.assert_array_equal(got[0][10], got[1][10])

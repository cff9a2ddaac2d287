"""The full path at the benchmark's workload and launch configuration: 4 x 16384
tokens with Zipf(1.1) ids, hash + gather over 16 tables of ~1M rows x 64, gate
forward + backward at H = 7168 and the weight-gradient reduction.

Every hash index is compared bit for bit; gathered rows and per-token gate
outputs on a sample of tokens (including the tokens with the smallest |s|);
dwh and dwe over all 65536 tokens, the oracle's sums being formed over token
blocks and added (the weight gradient is linear in the tokens, a property the
oracle pins)."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import (assert_bf16_close, assert_dw_close, assert_gate_close, bf16_bits,
                    ill_conditioned, to_dev_bf16)

pytestmark = pytest.mark.gpu


def test_full_path_workload(oracle_lib):
    w = inputs.WORKLOADS["full_path"]
    h = inputs.hash_inputs(w)
    gi = inputs.gate_inputs(w)
    T, H = w.T, w.H

    tok = torch.from_numpy(h["tokens"]).cuda()
    tables = to_dev_bf16(h["tables"])
    t = {n: to_dev_bf16(a) for n, a in gi.items()}
    idx, rows = eng.engram_hash_gather(tok, h["multipliers"], h["ngram_n"], h["table_sizes"],
                                       tables, pad_id=h["pad_id"])
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"], eps=w.eps)
    G = eng.engram_gate_bwd_num_partials(T, H)
    dx, dk, dv, part = eng.engram_gate_bwd(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"],
                                           eps=w.eps, G=G)
    dwh, dwe = eng.engram_grad_w_reduce(part, t["wh"], t["we"])
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0

    # hash: every index; rows of a token sample
    want_idx = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"],
                                      h["table_sizes"], pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    r = np.random.default_rng(7)
    sample = np.sort(r.choice(T, size=2048, replace=False))
    flat_idx = want_idx.reshape(T, 2, 8)
    want_rows = oracle_lib.engram_gather(flat_idx[sample], h["table_sizes"], h["tables"], w.D)
    got_rows = bf16_bits(rows.view(T, 2, 8, w.D)[torch.from_numpy(sample).cuda()])
    np.testing.assert_array_equal(got_rows, want_rows)
    del tables, rows

    # weight gradients over all tokens, oracle summed block by block
    dw_ref = {"dwh": np.zeros(H), "dwe": np.zeros(H)}
    s_all = np.empty(T)
    blk = 4096
    for a in range(0, T, blk):
        sl = slice(a, a + blk)
        res = oracle_lib.engram_gate_bwd(gi["g"][sl], gi["x"][sl], gi["k"][sl], gi["v"][sl],
                                         gi["wh"], gi["we"], eps=w.eps, per_token=False)
        dw_ref["dwh"] += res["dwh"]
        dw_ref["dwe"] += res["dwe"]
        s_all[sl] = res["s"]
    assert_dw_close("dwh", dwh, dw_ref["dwh"])
    assert_dw_close("dwe", dwe, dw_ref["dwe"])

    # per-token outputs on a sample that includes the most ill-conditioned tokens
    worst = np.argsort(np.abs(s_all))[:16]
    rows_s = np.unique(np.concatenate([r.choice(T, size=496, replace=False), worst, [0, T - 1]]))
    sub = {n: (a[rows_s] if a.ndim == 2 else a) for n, a in gi.items()}
    ref_out, ref_gate = oracle_lib.engram_gate_fwd(sub["x"], sub["k"], sub["v"], sub["wh"],
                                                   sub["we"], eps=w.eps)
    ref = oracle_lib.engram_gate_bwd(sub["g"], sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"],
                                     eps=w.eps, weights=False)
    sel = torch.from_numpy(rows_s).cuda()
    ill = ill_conditioned(ref["s"])
    assert_bf16_close("out", out[sel], ref_out)
    assert_gate_close(gate[sel], ref_gate)
    assert_bf16_close("dx", dx[sel], ref["dx"], rows_relaxed=ill)
    assert_bf16_close("dk", dk[sel], ref["dk"], rows_relaxed=ill)
    assert_bf16_close("dv", dv[sel], ref["dv"])

"""The full path at the benchmark's workload and launch configuration: 4 x 16384
tokens with Zipf(1.1) ids, hash + gather over 16 tables of ~1M rows x 64, gate
forward + backward at H = 7168 and the weight-gradient reduction.

The calls are the benchmark's: engram_hash_gather, engram_gate_fwd and
engram_gate_bwd_fused (the backward with the weight-gradient reduction in its
tail).  Every hash index and every gathered row is compared bit for bit;
every element of every per-token gate output, and dwh and dwe over all 65536
tokens, against the oracle computed block by block of tokens (the weight
gradient is linear in the tokens, a property the oracle pins)."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import assert_dw_close, bf16_bits, check_gate_blockwise, to_dev_bf16

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
    dx, dk, dv, dwh, dwe = eng.engram_gate_bwd_fused(t["g"], t["x"], t["k"], t["v"], t["wh"],
                                                     t["we"], eps=w.eps, G=G)
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0

    # hash: every index and every gathered row, bit for bit
    want_idx = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"],
                                      h["table_sizes"], pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    want_rows = oracle_lib.engram_gather(want_idx.reshape(T, 2, 8), h["table_sizes"],
                                         h["tables"], w.D)
    np.testing.assert_array_equal(bf16_bits(rows.view(T, 2, 8, w.D)), want_rows)
    del tables, rows, want_rows

    # every per-token output, and the weight gradients over all tokens
    res = dict(out=out, gate=gate, dx=dx, dk=dk, dv=dv)
    dw_ref, _ = check_gate_blockwise(oracle_lib, gi, res, w.eps)
    assert_dw_close("dwh", dwh, dw_ref["dwh"])
    assert_dw_close("dwe", dwe, dw_ref["dwe"])

"""GPU parity of engram_hash_gather against the oracle: indices and rows must be
bit-exact (the n-gram hash of the page "DeepSeek 开源 TileKernels",
zhichai.net/topic/177618722, section "5. Engram — 条件记忆门控")."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import bf16_bits, to_dev_bf16

pytestmark = pytest.mark.gpu


def _run(h, tokens=None, want_rows=True, tables_dev=None):
    tok = torch.from_numpy(h["tokens"] if tokens is None else tokens).cuda()
    if want_rows and tables_dev is None:
        tables_dev = to_dev_bf16(h["tables"])
    idx, rows = eng.engram_hash_gather(tok, h["multipliers"], h["ngram_n"], h["table_sizes"],
                                       tables_dev, pad_id=h["pad_id"], want_rows=want_rows)
    torch.cuda.synchronize()
    return idx, rows


def test_tiny_bit_exact(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    idx, rows = _run(h)
    want = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], h["table_sizes"],
                                  pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    want_rows = oracle_lib.engram_gather(want, h["table_sizes"], h["tables"], w.D)
    np.testing.assert_array_equal(bf16_bits(rows).reshape(want_rows.shape), want_rows)


def test_handworked_on_gpu(oracle_lib):
    import oracle_pins
    g = oracle_pins._golden()
    tok = torch.tensor(g["tokens"], dtype=torch.int64).cuda()
    idx, _ = eng.engram_hash_gather(tok, np.array(g["multipliers"], dtype=np.uint64), g["ngram_n"],
                                    np.array(g["table_sizes"], dtype=np.int64), None,
                                    pad_id=g["pad_id"], want_rows=False)
    idx = idx.cpu().numpy()
    for case in g["cases"]:
        assert idx[0, case["s"], case["layer"]].tolist() == case["idx"]


@pytest.mark.parametrize("D", [8, 40, 64, 128, 256])
def test_row_widths_and_ragged_shapes(oracle_lib, D):
    r = np.random.default_rng(D)
    L, J, n_max = 3, 11, 4
    B, S = 3, 37                        # T*L = 333 groups: not a multiple of the 32-group block
    tokens = r.integers(0, 5000, size=(B, S), dtype=np.int64)
    mult = r.integers(0, 2**64, size=(L, n_max), dtype=np.uint64, endpoint=False) | np.uint64(1)
    nn = np.array([1, 2, 4], dtype=np.int32)
    sizes = inputs.consecutive_primes(101, L * J).reshape(L, J)
    tables = inputs.normal_bf16(7, 0, (int(sizes.sum()), D))
    h = dict(tokens=tokens, multipliers=mult, ngram_n=nn, table_sizes=sizes, tables=tables,
             pad_id=12345)
    idx, rows = _run(h)
    want = oracle_lib.engram_hash(tokens, mult, nn, sizes, pad_id=12345)
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    want_rows = oracle_lib.engram_gather(want, sizes, tables, D)
    np.testing.assert_array_equal(bf16_bits(rows).reshape(want_rows.shape), want_rows)


def _random_case(r, L, J, D, B, S, n_max=3, vocab=5000, prime_base=1009):
    tokens = r.integers(0, vocab, size=(B, S), dtype=np.int64)
    mult = r.integers(0, 2**64, size=(L, n_max), dtype=np.uint64, endpoint=False) | np.uint64(1)
    nn = r.integers(1, n_max + 1, size=L).astype(np.int32)
    sizes = inputs.consecutive_primes(prime_base, L * J).reshape(L, J)
    tables = inputs.normal_bf16(int(r.integers(1 << 30)), 0, (int(sizes.sum()), D))
    return dict(tokens=tokens, multipliers=mult, ngram_n=nn, table_sizes=sizes, tables=tables,
                pad_id=-3)


# (L, J, D): from one table of 8-value rows to 32 tables, rows of 16 to 512
# bytes (one to four 16-byte chunks per lane), n-grams up to order 8
@pytest.mark.parametrize("L,J,D", [(1, 1, 8), (2, 8, 64), (3, 5, 136), (2, 8, 256), (4, 8, 8),
                                   (1, 16, 256), (4, 8, 256), (3, 11, 64)])
def test_gather_paths_bit_exact(oracle_lib, L, J, D):
    r = np.random.default_rng(L * 1000 + J * 10 + D)
    h = _random_case(r, L, J, D, B=3, S=37, n_max=8)    # n-grams up to the longest history
    idx, rows = _run(h)
    want = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], h["table_sizes"],
                                  pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    want_rows = oracle_lib.engram_gather(want, h["table_sizes"], h["tables"], D)
    np.testing.assert_array_equal(bf16_bits(rows).reshape(want_rows.shape), want_rows)


@pytest.mark.parametrize("B,S,L,J,D", [(5, 4001, 2, 8, 64), (5, 4001, 2, 8, 136), (4, 30011, 1, 2, 8)])
def test_many_tokens_per_warp(oracle_lib, B, S, L, J, D):
    # tens of thousands of tokens, up to 120K: many waves of CTAs, sequences
    # that span several CTAs' token ranges
    r = np.random.default_rng(D + S)
    h = _random_case(r, L, J, D, B=B, S=S)
    idx, rows = _run(h)
    want = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], h["table_sizes"],
                                  pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    want_rows = oracle_lib.engram_gather(want, h["table_sizes"], h["tables"], D)
    np.testing.assert_array_equal(bf16_bits(rows).reshape(want_rows.shape), want_rows)
    assert eng.engram_read_device_error() == 0


def test_large_table_sizes_and_full_range_ids(oracle_lib):
    # unsigned remainders for table sizes up to 2^62 and ids across all of int64
    import oracle_pins
    r = np.random.default_rng(99)
    L, J, n_max = 4, 16, 8
    B, S = 5, 23
    tokens = r.integers(-(2**63), 2**63 - 1, size=(B, S), dtype=np.int64)
    mult = r.integers(0, 2**64, size=(L, n_max), dtype=np.uint64, endpoint=False) | np.uint64(1)
    nn = np.array([1, 3, 5, 8], dtype=np.int32)
    sizes = r.integers(1, 2**62, size=(L, J), dtype=np.int64)
    sizes[0, :4] = [1, 2, 3, 2**62]
    sizes[1, :3] = [2**32 - 5, 2**32, 2**32 + 15]
    pad = -7
    tok = torch.from_numpy(tokens).cuda()
    idx, _ = eng.engram_hash_gather(tok, mult, nn, sizes, None, pad_id=pad, want_rows=False)
    got = idx.cpu().numpy()
    np.testing.assert_array_equal(got, oracle_lib.engram_hash(tokens, mult, nn, sizes, pad_id=pad))
    np.testing.assert_array_equal(got, oracle_pins.bigint_hash(tokens, mult, nn, sizes, pad))


def test_short_sequences_and_empty(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    tabs = to_dev_bf16(h["tables"])
    for B, S in ((1, 1), (3, 2), (2, 3)):
        toks = h["tokens"][:B, :S].copy()
        idx, rows = _run(h, tokens=toks, tables_dev=tabs)
        want = oracle_lib.engram_hash(toks, h["multipliers"], h["ngram_n"], h["table_sizes"],
                                      pad_id=h["pad_id"])
        np.testing.assert_array_equal(idx.cpu().numpy(), want)
        want_rows = oracle_lib.engram_gather(want, h["table_sizes"], h["tables"], w.D)
        np.testing.assert_array_equal(bf16_bits(rows).reshape(want_rows.shape), want_rows)
    idx, rows = _run(h, tokens=np.zeros((0, 5), dtype=np.int64), tables_dev=tabs)
    assert idx.numel() == 0 and rows.numel() == 0


def test_rows_only_matches_idx_and_rows():
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    tok = torch.from_numpy(h["tokens"]).cuda()
    tabs = to_dev_bf16(h["tables"])
    idx, rows = eng.engram_hash_gather(tok, h["multipliers"], h["ngram_n"], h["table_sizes"], tabs,
                                       pad_id=h["pad_id"])
    _, rows2 = eng.engram_hash_gather(tok, h["multipliers"], h["ngram_n"], h["table_sizes"], tabs,
                                      pad_id=h["pad_id"], want_idx=False)
    torch.cuda.synchronize()
    assert torch.equal(rows.view(torch.int16), rows2.view(torch.int16))


def test_misaligned_rows_rejected():
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    tok = torch.from_numpy(h["tokens"]).cuda()
    tabs = to_dev_bf16(h["tables"])
    T = h["tokens"].size
    buf = torch.empty(T * 16 * w.D + 8, dtype=torch.bfloat16, device="cuda")
    bad = buf[4:4 + T * 16 * w.D].view(*h["tokens"].shape, 2, 8, w.D)   # 8-byte offset
    with pytest.raises(eng.EngramError):
        eng.engram_hash_gather(tok, h["multipliers"], h["ngram_n"], h["table_sizes"], tabs,
                               pad_id=h["pad_id"], rows_out=bad)


def test_full_size_zipf(oracle_lib):
    """The hash+gather workload at full size (16 x 2048 Zipf(1.1) ids, 16 tables
    of ~1M rows x 64): every index bit-exact, and every gathered row checked
    byte for byte against the table on the device."""
    w = inputs.WORKLOADS["hash_gather"]
    h = inputs.hash_inputs(w)
    tabs = to_dev_bf16(h["tables"])
    idx, rows = _run(h, tables_dev=tabs)
    want = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], h["table_sizes"],
                                  pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    # rows: gather the oracle's rows for a sample on the host, all rows on the device
    r = np.random.default_rng(0)
    sample = r.choice(w.T, size=2048, replace=False)
    flat_want = want.reshape(w.T, 2, 8)[sample]
    want_rows = oracle_lib.engram_gather(flat_want, h["table_sizes"], h["tables"], w.D)
    got_rows = bf16_bits(rows.view(w.T, 2, 8, w.D)[torch.from_numpy(sample).cuda()])
    np.testing.assert_array_equal(got_rows, want_rows)
    first = np.concatenate([[0], np.cumsum(h["table_sizes"].ravel())[:-1]]).reshape(1, 2, 8)
    glob = torch.from_numpy((want.reshape(w.T, 2, 8) + first).reshape(-1)).cuda()
    ref_rows = tabs.view(torch.int16)[glob].view(w.T, 2, 8, w.D)
    assert torch.equal(ref_rows, rows.view(torch.int16).view(w.T, 2, 8, w.D))

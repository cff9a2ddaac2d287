"""GPU parity of engram_gather_bwd (the transpose of the Engram table-row gather of
the page "DeepSeek 开源 TileKernels", zhichai.net/topic/177618722, section
"5. Engram — 条件记忆门控") against the oracle's gather backward.

Tolerance, derived from the arithmetic.  The kernels sum the n bf16 gradients
of a row in fp64 and add that sum to the row's fp32 value in fp64 with one
rounding to fp32; the oracle sums the same values in fp64 in token order.  Each
fp64 sum of n terms is within (n - 1) 2^-53 sum|terms| of the exact sum, and
the final rounding to fp32 adds at most 2^-24 |result|, so per element
    |gpu - (init + ref)| <= 2^-24 |init + ref| + 2 n 2^-52 (|init| + sum|terms|).
Rows that no entry reads must come back bit-identical.
"""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import to_dev_bf16

pytestmark = pytest.mark.gpu


def _widen(bits):
    return inputs.bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def _expect(o, idx, sizes, d_rows_bits, init, row_lo=0, row_hi=None):
    """(init + oracle sum, tolerance) over the global rows [row_lo, row_hi)."""
    ref = o.engram_gather_bwd(idx, sizes, d_rows_bits, row_lo, row_hi)
    absref = o.engram_gather_bwd(idx, sizes, np.abs(_widen(d_rows_bits)), row_lo, row_hi)
    ones = np.ones(idx.shape + (1,), dtype=np.float64)
    count = o.engram_gather_bwd(idx, sizes, ones, row_lo, row_hi)[:, :1]
    want = init + ref
    tol = 2.0 ** -24 * np.abs(want) + 2.0 * count * 2.0 ** -52 * (np.abs(init) + absref)
    return want, tol, count[:, 0] > 0


def _check(got, want, tol, touched, init):
    got = got.detach().cpu().double().numpy()
    err = np.abs(got - want)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{int(bad.sum())} of {err.size} elements out of tolerance; worst at "
                             f"{i}: got {got[i]!r}, want {want[i]!r}, tol {tol[i]!r}")
    # untouched rows are not written at all
    np.testing.assert_array_equal(got[~touched].astype(np.float32), init[~touched].astype(np.float32))


def _run(idx_dev, sizes, d_rows_bits, init):
    d_tables = torch.from_numpy(init.astype(np.float32)).cuda()
    eng.engram_gather_bwd(idx_dev, sizes, to_dev_bf16(d_rows_bits), d_tables)
    assert eng.engram_read_device_error() == 0
    return d_tables


def test_tiny_workload(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w, with_tables=False)
    idx, _ = eng.engram_hash_gather(torch.from_numpy(h["tokens"]).cuda(), h["multipliers"],
                                    h["ngram_n"], h["table_sizes"], None, pad_id=h["pad_id"],
                                    want_rows=False)
    idx_np = idx.cpu().numpy()
    d_rows = inputs.gather_grad_inputs(w)
    R = int(h["table_sizes"].sum())
    init = np.random.default_rng(5).standard_normal((R, w.D)).astype(np.float32).astype(np.float64)
    got = _run(idx, h["table_sizes"], d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, h["table_sizes"], d_rows, init)
    _check(got, want, tol, touched, init)


@pytest.mark.parametrize("D", [8, 24, 64, 136, 256])
def test_ragged_shapes_and_duplicates(oracle_lib, D):
    # 3 layers x 5 tables of 17..59 rows and 777 tokens: every row is read many
    # times, segments cross chunk boundaries, and T*L*J = 11655 fills neither a
    # sort tile nor a chunk evenly
    r = np.random.default_rng(D)
    L, J, T = 3, 5, 777
    sizes = r.integers(17, 60, size=(L, J), dtype=np.int64)
    idx_np = (r.random((T, L, J)) ** 3 * sizes[None]).astype(np.int64)   # skewed to low rows
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    init = np.zeros((R, D))
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    _check(got, want, tol, touched, init)


@pytest.mark.parametrize("T", [1, 31, 5000])
def test_one_hot_row_per_table(oracle_lib, T):
    # every token reads the same row of each table: one segment of T entries per
    # table, spanning up to ~78 chunks of 64 (more than one 32-chunk window)
    r = np.random.default_rng(T)
    L, J, D = 2, 8, 64
    sizes = inputs.consecutive_primes(4099, L * J).reshape(L, J)
    idx_np = np.broadcast_to(r.integers(0, 4099, size=(1, L, J)), (T, L, J)).astype(np.int64).copy()
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    init = np.zeros((R, D))
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    _check(got, want, tol, touched, init)


def test_most_tables(oracle_lib):
    # the largest table count the library takes (4 layers x 16 tables), every
    # table a different size, so each entry's table offset and bound come from
    # its own slot of the per-table parameters
    r = np.random.default_rng(64)
    L, J, T, D = 4, 16, 389, 32
    sizes = inputs.consecutive_primes(211, L * J).reshape(L, J)
    idx_np = (r.random((T, L, J)) ** 2 * sizes[None]).astype(np.int64)
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    init = r.standard_normal((R, D)).astype(np.float32).astype(np.float64)
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    _check(got, want, tol, touched, init)


def test_no_repeated_rows(oracle_lib):
    # every entry reads its own row: all of them take the in-place update and
    # the list of repeated rows' entries is empty (its kernels see M = 0)
    L, J, T, D = 2, 8, 1500, 64
    sizes = np.full((L, J), 4 * T + 1, dtype=np.int64)
    t = np.arange(T, dtype=np.int64)[:, None, None]
    q = np.arange(L * J, dtype=np.int64).reshape(1, L, J)
    idx_np = (3 * t + q) % sizes[None]          # distinct within each table
    r = np.random.default_rng(15)
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    init = r.standard_normal((R, D)).astype(np.float32).astype(np.float64)
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    assert int(touched.sum()) == T * L * J
    _check(got, want, tol, touched, init)


def test_deterministic_and_accumulating(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    r = np.random.default_rng(3)
    sizes = np.full((2, 8), 97, dtype=np.int64)
    T = 3000
    idx_np = r.integers(0, 97, size=(T, 2, 8), dtype=np.int64)
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, 2, 8, w.D)).astype(np.float32))
    idx = torch.from_numpy(idx_np).cuda()
    a = _run(idx, sizes, d_rows, np.zeros((int(sizes.sum()), w.D)))
    b = _run(idx, sizes, d_rows, np.zeros((int(sizes.sum()), w.D)))
    assert torch.equal(a.view(torch.int32), b.view(torch.int32)), "not bitwise reproducible"
    # two calls accumulate: a + (a's gradient again)
    eng.engram_gather_bwd(idx, sizes, to_dev_bf16(d_rows), a)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, b.cpu().double().numpy())
    _check(a, want, tol, touched, b.cpu().double().numpy())


def test_out_of_range_index_is_skipped_and_reported(oracle_lib):
    r = np.random.default_rng(11)
    L, J, T, D = 2, 4, 200, 32
    sizes = np.full((L, J), 50, dtype=np.int64)
    idx_np = r.integers(0, 50, size=(T, L, J), dtype=np.int64)
    bad = np.zeros(idx_np.shape, dtype=bool)
    bad[3, 0, 1] = bad[77, 1, 3] = bad[199, 1, 0] = True
    idx_bad = idx_np.copy()
    idx_bad[3, 0, 1], idx_bad[77, 1, 3], idx_bad[199, 1, 0] = -1, 50, 2**40
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    assert eng.engram_read_device_error() == 0
    d_tables = torch.zeros((R, D), dtype=torch.float32, device="cuda")
    eng.engram_gather_bwd(torch.from_numpy(idx_bad).cuda(), sizes, to_dev_bf16(d_rows), d_tables)
    assert eng.engram_read_device_error() == eng.DEVICE_ERR_INDEX_RANGE
    # the valid entries are summed as if the invalid ones were absent
    d_ok = d_rows.copy()
    d_ok[bad] = 0
    want, tol, _ = _expect(oracle_lib, np.where(bad, 0, idx_np), sizes, d_ok, np.zeros((R, D)))
    err = np.abs(d_tables.cpu().double().numpy() - want)
    assert np.all(err <= tol)


def test_empty_and_argument_errors():
    sizes = np.full((2, 8), 101, dtype=np.int64)
    d_tables = torch.ones((int(sizes.sum()), 16), dtype=torch.float32, device="cuda")
    idx = torch.zeros((0, 2, 8), dtype=torch.int64, device="cuda")
    d_rows = torch.zeros((0, 2, 8, 16), dtype=torch.bfloat16, device="cuda")
    eng.engram_gather_bwd(idx, sizes, d_rows, d_tables)
    torch.cuda.synchronize()
    assert bool((d_tables == 1).all())
    idx = torch.zeros((4, 2, 8), dtype=torch.int64, device="cuda")
    d_rows = torch.zeros((4, 2, 8, 16), dtype=torch.bfloat16, device="cuda")
    small = torch.empty((16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(eng.EngramError):
        eng.engram_gather_bwd(idx, sizes, d_rows, d_tables, workspace=small)


@pytest.mark.parametrize("sizes", [[300], [100, 100], [128, 128], [128, 129], [150, 150, 100],
                                   [40000, 30000]])
def test_sort_levels(oracle_lib, sizes):
    # total rows R = 300 (a single table), 200, 256 (keys of 8 bits: one radix
    # pass), 257 (9 bits: a second pass on one bit), 400, 70000 (17 bits: three
    # passes); every row read several times
    r = np.random.default_rng(len(sizes) + sum(sizes))
    sizes = np.array(sizes, dtype=np.int64).reshape(1, -1)
    T, D = 3000, 16
    idx_np = (r.random((T,) + sizes.shape) ** 3 * sizes[None]).astype(np.int64)
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T,) + sizes.shape + (D,)).astype(np.float32))
    R = int(sizes.sum())
    init = r.standard_normal((R, D)).astype(np.float32).astype(np.float64)
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    _check(got, want, tol, touched, init)


def test_every_token_the_same():
    # the degenerate input: every token reads the same row of each of 16 tables
    # of ~1M rows, so 16 rows hold all 20000 entries each: one digit value per
    # radix pass takes nearly every entry, and each row's run spans 313 chunks
    # (the result: each of those rows gets the column sums of its table's
    # gradients)
    r = np.random.default_rng(9)
    L, J, T, D = 2, 8, 20000, 8
    sizes = inputs.consecutive_primes(1000003, L * J).reshape(L, J)
    pick = r.integers(0, 1000003, size=(1, L, J))
    idx_np = np.broadcast_to(pick, (T, L, J)).astype(np.int64).copy()
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    d_tables = torch.zeros((R, D), dtype=torch.float32, device="cuda")
    eng.engram_gather_bwd(torch.from_numpy(idx_np).cuda(), sizes, to_dev_bf16(d_rows), d_tables)
    assert eng.engram_read_device_error() == 0
    first = np.concatenate([[0], np.cumsum(sizes.ravel())[:-1]])
    rows = first + pick.ravel()
    g = _widen(d_rows).reshape(T, L * J, D)
    want = g.sum(axis=0)
    absum = np.abs(g).sum(axis=0)
    got = d_tables[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    assert np.all(np.abs(got - want) <= 2.0 ** -24 * np.abs(want) + 2 * T * 2.0 ** -52 * absum)
    assert int((d_tables != 0).any(dim=1).sum()) == L * J


def test_four_radix_passes(oracle_lib):
    # 16 tables of ~4.19M rows (67M rows in all, more than 2^24): row keys need
    # four 8-bit radix passes; a Zipf-like skew makes many rows repeat.  D = 8
    # keeps the fp32 table gradient at 2.1 GB.  Checked on row windows around
    # the hottest rows and at random, plus the touched-row property.
    r = np.random.default_rng(44)
    L, J, T, D = 2, 8, 4096, 8
    sizes = inputs.consecutive_primes(4194301, L * J).reshape(L, J)
    R = int(sizes.sum())
    assert R > 2 ** 24 * 3
    idx_np = np.minimum((r.pareto(0.8, size=(T, L, J)) * 50).astype(np.int64), sizes[None] - 1)
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    d_tables = torch.zeros((R, D), dtype=torch.float32, device="cuda")
    eng.engram_gather_bwd(torch.from_numpy(idx_np).cuda(), sizes, to_dev_bf16(d_rows), d_tables)
    assert eng.engram_read_device_error() == 0
    first = np.concatenate([[0], np.cumsum(sizes.ravel())[:-1]])
    rows = (idx_np.reshape(-1, L * J) + first[None]).ravel()
    uniq, counts = np.unique(rows, return_counts=True)
    assert counts.max() > 50
    hot = uniq[np.argsort(counts)[-3:]]
    for lo in [0, R - 64] + [int(x) - 2 for x in hot] + [int(x) for x in r.integers(0, R - 64, 3)]:
        lo = max(0, lo)
        hi = min(R, lo + 64)
        want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, np.zeros((hi - lo, D)), lo, hi)
        _check(d_tables[lo:hi], want, tol, touched, np.zeros((hi - lo, D)))
    nonzero = (d_tables != 0).any(dim=1).nonzero().flatten().cpu().numpy()
    np.testing.assert_array_equal(nonzero, uniq)


def test_full_path_size_sampled(oracle_lib):
    # the full-path workload as the benchmark runs it: 65536 Zipf tokens, 16
    # tables of ~1M rows x 64; d_tables (4.1 GB fp32) checked on windows of rows
    # around the hottest rows, at random and at both ends, plus two properties
    # over all rows: column sums equal those of d_rows, and exactly the rows
    # that some entry reads are nonzero
    w = inputs.WORKLOADS["full_path"]
    h = inputs.hash_inputs(w, with_tables=False)
    sizes = h["table_sizes"]
    idx_np = oracle_lib.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], sizes,
                                    pad_id=h["pad_id"])
    idx, _ = eng.engram_hash_gather(torch.from_numpy(h["tokens"]).cuda(), h["multipliers"],
                                    h["ngram_n"], sizes, None, pad_id=h["pad_id"], want_rows=False)
    assert np.array_equal(idx.cpu().numpy(), idx_np)
    d_rows = inputs.gather_grad_inputs(w)
    R = int(sizes.sum())
    d_tables = torch.zeros((R, w.D), dtype=torch.float32, device="cuda")
    eng.engram_gather_bwd(idx, sizes, to_dev_bf16(d_rows), d_tables)
    assert eng.engram_read_device_error() == 0

    first = np.concatenate([[0], np.cumsum(sizes.ravel())[:-1]])
    rows = (idx_np.reshape(-1, 16) + first[None]).ravel()
    uniq, counts = np.unique(rows, return_counts=True)
    hot = uniq[np.argsort(counts)[-4:]]
    r = np.random.default_rng(0)
    starts = [0, R - 64] + [int(x) - 2 for x in hot] + [int(x) for x in r.integers(0, R - 64, 4)]
    for lo in starts:
        lo = max(0, lo)
        hi = min(R, lo + 64)
        want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, np.zeros((hi - lo, w.D)),
                                     lo, hi)
        _check(d_tables[lo:hi], want, tol, touched, np.zeros((hi - lo, w.D)))
    assert counts.max() > 500          # the Zipf head really produced long segments

    nonzero = (d_tables != 0).any(dim=1).nonzero().flatten().cpu().numpy()
    np.testing.assert_array_equal(nonzero, uniq)
    colsum = torch.zeros(w.D, dtype=torch.float64, device="cuda")
    for c in range(0, R, 1 << 22):
        colsum += d_tables[c:c + (1 << 22)].double().sum(0)
    want_sum = _widen(d_rows).reshape(-1, w.D).sum(0)
    absum = np.abs(_widen(d_rows)).reshape(-1, w.D).sum(0)
    # each row value carries one fp32 rounding (2^-24 relative)
    assert np.all(np.abs(colsum.cpu().numpy() - want_sum) <= 2.0 ** -23 * absum)


def _side_stream_cases(n):
    """n independent (idx, table sizes, d_rows) problems with many repeated rows,
    so that every call has work on the library's side stream."""
    cases = []
    for k in range(n):
        r = np.random.default_rng(100 + k)
        sizes = np.full((2, 4), 300 + 50 * k, dtype=np.int64)
        T = 20000 + 3000 * k
        idx = r.integers(0, int(sizes[0, 0]), size=(T, 2, 4), dtype=np.int64)
        d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, 2, 4, 32)).astype(np.float32))
        cases.append((torch.from_numpy(idx).cuda(), sizes, to_dev_bf16(d_rows)))
    return cases


def _serial(cases, repeats):
    out = []
    for idx, sizes, d_rows in cases:
        t = torch.zeros((int(sizes.sum()), 32), dtype=torch.float32, device="cuda")
        for _ in range(repeats):
            eng.engram_gather_bwd(idx, sizes, d_rows, t)
        out.append(t)
    torch.cuda.synchronize()
    return out


def _workspaces(cases):
    return [torch.empty(eng.engram_gather_bwd_workspace_size(idx.shape[0], 2, 4, 32, int(sizes.sum())),
                        dtype=torch.uint8, device="cuda") for idx, sizes, _ in cases]


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_side_stream_calls_on_two_streams():
    # calls on two caller streams, interleaved: the library's side stream is
    # shared, each call joins back into its own stream; results as if serial
    cases = _side_stream_cases(2)
    want = _serial(cases, 3)
    ws = _workspaces(cases)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    got = [torch.zeros_like(w) for w in want]
    torch.cuda.synchronize()
    for _ in range(3):
        for (idx, sizes, d_rows), t, w, s in zip(cases, got, ws, streams):
            eng.engram_gather_bwd(idx, sizes, d_rows, t, workspace=w, stream=s)
    # what follows on each caller stream sees the finished result
    sums = []
    for t, s in zip(got, streams):
        with torch.cuda.stream(s):
            sums.append(t.double().sum())
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0
    for g, w, sm in zip(got, want, sums):
        assert _bits_equal(g, w)
        assert sm.item() == w.double().sum().item()


def test_side_stream_calls_from_two_threads():
    import threading

    cases = _side_stream_cases(2)
    want = _serial(cases, 4)
    ws = _workspaces(cases)
    got = [torch.zeros_like(w) for w in want]
    torch.cuda.synchronize()
    errors = []

    def worker(k):
        try:
            s = torch.cuda.Stream()
            idx, sizes, d_rows = cases[k]
            for _ in range(4):
                eng.engram_gather_bwd(idx, sizes, d_rows, got[k], workspace=ws[k], stream=s)
            s.synchronize()
        except Exception as exc:       # reported on the main thread
            errors.append(exc)

    th = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for g, w in zip(got, want):
        assert _bits_equal(g, w)


def test_side_stream_in_cuda_graph():
    # the fork and join are captured like any other stream work; the first
    # call on the device (which creates the side stream) happens before capture
    cases = _side_stream_cases(1)
    idx, sizes, d_rows = cases[0]
    want = _serial(cases, 2)[0]
    ws = _workspaces(cases)[0]
    t = torch.zeros_like(want)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        eng.engram_gather_bwd(idx, sizes, d_rows, t, workspace=ws)
    torch.cuda.synchronize()
    assert not t.any()                 # captured, not run
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0
    assert _bits_equal(t, want)
    del g


@pytest.mark.parametrize("repeated", [1024, 1025, 2048, 4097, 64 * 37])
def test_list_lengths_at_tile_edges(oracle_lib, repeated):
    # exactly `repeated` entries fall on rows read more than once (pairs, plus
    # one triple when the count is odd), the other entries on rows read once:
    # the sorted list then fills whole radix tiles of 1024 entries, or spills
    # one entry into the next tile, or whole segment chunks of 64 entries
    r = np.random.default_rng(repeated)
    L, J, D = 1, 4, 16
    sizes = np.full((L, J), 200003, dtype=np.int64)
    T = 6000
    n = T * L * J
    tab = np.tile(np.arange(J), T)                 # entry e belongs to table e % J
    rows = np.empty(n, dtype=np.int64)
    # distinct rows per table for every entry first
    for j in range(J):
        sel = np.flatnonzero(tab == j)
        rows[sel] = r.choice(200003, size=sel.size, replace=False)
    # then make `repeated` entries share rows: pairs of entries of the same
    # table read the same row (a triple if the count is odd)
    pick = r.choice(np.flatnonzero(tab == 0), size=repeated, replace=False)
    k = 0
    while k < repeated:
        take = 3 if repeated - k == 3 else 2
        rows[pick[k:k + take]] = rows[pick[k]]
        k += take
    idx_np = rows.reshape(T, L, J)
    first = np.concatenate([[0], np.cumsum(sizes.ravel())[:-1]])
    keys = (idx_np.reshape(-1, L * J) + first[None]).ravel()
    _, inv, cnt = np.unique(keys, return_inverse=True, return_counts=True)
    assert int((cnt[inv] > 1).sum()) == repeated
    d_rows = inputs.f32_to_bf16_bits(r.standard_normal((T, L, J, D)).astype(np.float32))
    R = int(sizes.sum())
    init = np.zeros((R, D))
    got = _run(torch.from_numpy(idx_np).cuda(), sizes, d_rows, init)
    want, tol, touched = _expect(oracle_lib, idx_np, sizes, d_rows, init)
    _check(got, want, tol, touched, init)

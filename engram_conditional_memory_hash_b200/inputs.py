"""Seeded synthetic inputs for the Engram hash/gather and gate workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no hash, no modulo by table sizes, no normalisation, no
gate).  The tests, the benchmark and the oracle's callers share it.

Recipe (numpy PCG64, every tensor from its own seed stream so that tensors do
not depend on the order they are drawn in, and large tensors are drawn in
fixed-size chunks, each with its own stream, so that the values do not depend
on the number of host threads):

* bf16 "N(0,1)" tensors: float32 ``standard_normal`` rounded to bf16
  (round to nearest, ties to even); ``wh``/``we`` = bf16(1 + 0.1 * N(0,1)).
* token ids: uniform integers, or Zipf(s) over ranks 1..vocab sampled by
  inverse CDF (P(rank r) proportional to r^-s), id = rank - 1.
* multipliers: uniform 64-bit integers with the low bit set (odd).
* table sizes: ``count`` consecutive primes from ``base`` upward, assigned to
  tables in (layer, table) order.
* tables: bf16 N(0,1), all tables concatenated row-major.
* d_rows (the gradient reaching the gathered rows, for the gather backward):
  bf16 N(0,1) of shape [T, L, J, D].

The workloads (token count T = B*S, hidden size H, tables of D columns):

=============  =====================  ======  ===================================
name           T                      H       hash tables
=============  =====================  ======  ===================================
tiny           2 x 128, ids U[0,1000)  256     16 primes from 4099, D = 32
gate_fwd       4 x 4096                4096    (none)
gate_fwdbwd    8 x 4096                7168    (none)
hash_gather    16 x 2048, Zipf(1.1)    (none)  16 primes from 1,000,003, D = 64
full_path      4 x 16384, Zipf(1.1)    7168    16 primes from 1,000,003, D = 64
=============  =====================  ======  ===================================
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SEED_BASE = 20260422
CHUNK = 1 << 22  # elements per independently seeded chunk

# One seed stream per tensor.
STREAM_X, STREAM_K, STREAM_V, STREAM_G = 0, 1, 2, 3
STREAM_WH, STREAM_WE = 4, 5
STREAM_TOKENS, STREAM_MULT, STREAM_TABLES = 6, 7, 8
STREAM_DROWS = 9


def generator(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 bit patterns (nearest, ties to even)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_bf16(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """bf16 bits of mean + std * N(0,1), drawn in float32, chunk by chunk."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.uint16)

    def fill(c: int) -> None:
        lo = c * CHUNK
        hi = min(n, lo + CHUNK)
        z = generator(seed, stream, c).standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            z *= np.float32(std)
        if mean != 0.0:
            z += np.float32(mean)
        out[lo:hi] = f32_to_bf16_bits(z)

    nchunks = (n + CHUNK - 1) // CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def uniform_ids(seed: int, stream: int, shape, low: int, high: int) -> np.ndarray:
    return generator(seed, stream).integers(low, high, size=shape, dtype=np.int64)


def zipf_ids(seed: int, stream: int, shape, vocab: int, s: float) -> np.ndarray:
    """ids in [0, vocab) with P(id = r - 1) proportional to r^-s (inverse CDF)."""
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** (-s))
    cdf /= cdf[-1]
    u = generator(seed, stream).random(size=shape)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int64)


def odd_multipliers(seed: int, stream: int, L: int, n_max: int) -> np.ndarray:
    m = generator(seed, stream).integers(0, 2**64, size=(L, n_max), dtype=np.uint64, endpoint=False)
    return m | np.uint64(1)


def consecutive_primes(base: int, count: int) -> np.ndarray:
    out = []
    p = max(2, int(base))
    while len(out) < count:
        if all(p % q for q in range(2, int(p ** 0.5) + 1)):
            out.append(p)
        p += 1
    return np.asarray(out, dtype=np.int64)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int              # position in the workload list; seed = SEED_BASE + index
    B: int = 0
    S: int = 0
    H: int = 0              # 0: no gate stage
    backward: bool = False
    ids: str = ""           # "" (no hash stage), "uniform" or "zipf"
    id_high: int = 0        # uniform ids in [0, id_high)
    vocab: int = 0          # zipf vocabulary
    zipf_s: float = 1.1
    L: int = 2
    J: int = 8
    ngram_n: tuple = (2, 3)
    prime_base: int = 0
    D: int = 0
    pad_id: int = -1
    eps: float = 1e-6

    @property
    def T(self) -> int:
        return self.B * self.S

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def has_hash(self) -> bool:
        return bool(self.ids)

    @property
    def has_gate(self) -> bool:
        return self.H > 0


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", 0, B=2, S=128, H=256, backward=True, ids="uniform", id_high=1000,
                 prime_base=4099, D=32),
        Workload("gate_fwd", 1, B=4, S=4096, H=4096, backward=False),
        Workload("gate_fwdbwd", 2, B=8, S=4096, H=7168, backward=True),
        Workload("hash_gather", 3, B=16, S=2048, ids="zipf", vocab=129280,
                 prime_base=1000003, D=64),
        Workload("full_path", 4, B=4, S=16384, H=7168, backward=True, ids="zipf",
                 vocab=129280, prime_base=1000003, D=64),
    ]
}


def gate_inputs(w: Workload, T: int | None = None, H: int | None = None) -> dict:
    """x, k, v, g [T, H] and wh, we [H] as bf16 bits (uint16)."""
    T = w.T if T is None else T
    H = w.H if H is None else H
    return {
        "x": normal_bf16(w.seed, STREAM_X, (T, H)),
        "k": normal_bf16(w.seed, STREAM_K, (T, H)),
        "v": normal_bf16(w.seed, STREAM_V, (T, H)),
        "g": normal_bf16(w.seed, STREAM_G, (T, H)),
        "wh": normal_bf16(w.seed, STREAM_WH, (H,), mean=1.0, std=0.1),
        "we": normal_bf16(w.seed, STREAM_WE, (H,), mean=1.0, std=0.1),
    }


def hash_inputs(w: Workload, B: int | None = None, S: int | None = None,
                with_tables: bool = True) -> dict:
    """tokens [B, S] int64, multipliers [L, n_max] uint64, ngram_n [L] int32,
    table_sizes [L, J] int64 and (optionally) tables [sum(P) * D] bf16 bits."""
    B = w.B if B is None else B
    S = w.S if S is None else S
    if w.ids == "uniform":
        tokens = uniform_ids(w.seed, STREAM_TOKENS, (B, S), 0, w.id_high)
    else:
        tokens = zipf_ids(w.seed, STREAM_TOKENS, (B, S), w.vocab, w.zipf_s)
    n_max = max(w.ngram_n)
    out = {
        "tokens": tokens,
        "multipliers": odd_multipliers(w.seed, STREAM_MULT, w.L, n_max),
        "ngram_n": np.asarray(w.ngram_n, dtype=np.int32),
        "table_sizes": consecutive_primes(w.prime_base, w.L * w.J).reshape(w.L, w.J),
        "pad_id": w.pad_id,
        "D": w.D,
    }
    if with_tables:
        rows = int(out["table_sizes"].sum())
        out["tables"] = normal_bf16(w.seed, STREAM_TABLES, (rows, w.D))
    return out


def gather_grad_inputs(w: Workload, T: int | None = None) -> np.ndarray:
    """d_rows [T, L, J, D] as bf16 bits (uint16): the gradient of the gathered rows."""
    T = w.T if T is None else T
    return normal_bf16(w.seed, STREAM_DROWS, (T, w.L, w.J, w.D))

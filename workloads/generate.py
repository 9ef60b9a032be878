"""Seeded synthetic workloads for the Engram N-gram hash / gather / backward path.

This module is the only code shared by the oracle side (tests, CPU baseline)
and the CUDA side (tests, bench). It draws inputs and holds none of the
method's arithmetic: it produces raw token IDs, sequence bounds, per-head
moduli/offsets (configuration inputs), tables and output gradients.

The five workloads stand in for the engram pages' own runs (right-tail-padded
4,096-token samples, packed THD documents given by cu_seqlens, and the 262,144
native length on the full 320,001,536 x 160 table). No dataset item is used or
reproduced; every value comes from a seeded NumPy PCG64 or torch generator.
"""

from __future__ import annotations

import dataclasses
from functools import lru_cache

import numpy as np

from . import constants as C

DTYPE_CODES = {"f32": 0, "bf16": 1, "f16": 2}
DTYPE_BYTES = {"f32": 4, "bf16": 2, "f16": 2}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    structure: str               # "rows" | "docs_cu" | "docs_eos"
    batch: int                   # rows (structure == "rows"), else 1
    seq_len: int                 # tokens per row, or total tokens for docs
    doc_len: tuple[int, int] | None
    id_dist: str                 # "uniform" | "zipf"
    zipf_s: float
    id_range: int
    eos_id: int
    eos_p: float                 # i.i.d. EOS replacement rate ("rows" only)
    heads: str                   # "seeded" | "page"
    table_rows: int | None       # None: sum of seeded moduli rounded up to 128
    prime_range: tuple[int, int] | None
    dtype: str                   # table / dout dtype: "f32" | "bf16"
    description: str = ""

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len


WORKLOADS = {
    "tiny": Workload(
        "tiny", 0, "rows", 2, 64, None, "uniform", 0.0, 1000, 999, 0.05,
        "seeded", None, (900, 1100), "f32",
        "2 x 64 tokens, IDs U[0,1000), EOS 999 i.i.d. p=0.05, 16 seeded prime "
        "heads ~1,000 rows each, fp32 table"),
    "b4x4096": Workload(
        "b4x4096", 1, "rows", 4, 4096, None, "uniform", 0.0, C.TOKENIZER_VOCAB,
        C.EOS_TOKEN_ID, 1.0 / 512, "seeded", 16_777_216, (943_718, 1_048_576),
        "bf16",
        "4 x 4,096 tokens, IDs U[0,248320), EOS i.i.d. p=1/512, 16,777,216-row "
        "bf16 table split by 16 seeded prime heads"),
    "thd64k": Workload(
        "thd64k", 2, "docs_cu", 1, 65_536, (128, 4096), "zipf", 1.1,
        C.TOKENIZER_VOCAB, C.EOS_TOKEN_ID, 0.0, "seeded", 67_108_864,
        (3_774_873, 4_194_304), "bf16",
        "65,536 packed tokens, documents of U[128,4096] tokens each ending in "
        "EOS and bounded by cu_seqlens, Zipf(1.1) IDs, 67,108,864-row table"),
    "full": Workload(
        "full", 3, "rows", 16, 4096, None, "uniform", 0.0, C.TOKENIZER_VOCAB,
        C.EOS_TOKEN_ID, 1.0 / 512, "page", C.PADDED_ROWS, None, "bf16",
        "16 x 4,096 tokens, IDs U[0,248320), EOS i.i.d. p=1/512, full "
        "320,001,536 x 160 bf16 table with the page's head constants"),
    "long256k": Workload(
        "long256k", 4, "docs_eos", 1, 262_144, (1024, 32768), "zipf", 1.2,
        C.TOKENIZER_VOCAB, C.EOS_TOKEN_ID, 0.0, "page", C.PADDED_ROWS, None,
        "bf16",
        "one 262,144-token row of documents of U[1024,32768] tokens delimited "
        "by EOS only, Zipf(1.2) IDs, full table"),
}


# ---------------------------------------------------------------- head params

def _primes_in(lo: int, hi: int) -> np.ndarray:
    """All primes p with lo <= p < hi (sieve of Eratosthenes)."""
    sieve = np.ones(hi, dtype=bool)
    sieve[:2] = False
    for f in range(2, int(hi ** 0.5) + 1):
        if sieve[f]:
            sieve[f * f::f] = False
    return np.nonzero(sieve[lo:])[0] + lo


@lru_cache(maxsize=None)
def head_params(name: str) -> dict:
    """Configuration of the hash: multipliers, moduli, offsets, rows, EOS, fill.

    Seeded workloads draw 16 distinct primes from their range (sorted, so the
    offsets ascend like the page's) and pack them back to back; the page
    workloads take the page's constants.
    """
    w = WORKLOADS[name]
    if w.heads == "page":
        vocab, offsets, rows = C.page_head_tables()
    else:
        rng = np.random.Generator(np.random.PCG64(1000 + w.seed))
        cands = _primes_in(*w.prime_range)
        picks = np.sort(rng.choice(cands, size=C.HEADS_PER_NGRAM * (C.NGRAM_SIZE - 1),
                                   replace=False))
        vocab = tuple(int(v) for v in picks)
        offsets = C.running_offsets(vocab)
        total = offsets[-1] + vocab[-1]
        rows = w.table_rows if w.table_rows is not None else -(-total // 128) * 128
        assert total <= rows
    return {
        "ngram_size": C.NGRAM_SIZE,
        "heads_per_ngram": C.HEADS_PER_NGRAM,
        "multipliers": tuple(C.LAYER_MULTIPLIERS),
        "vocab_sizes": tuple(vocab),
        "offsets": tuple(offsets),
        "table_rows": int(rows),
        "dim": C.EMBEDDING_DIM,
        "eos_id": int(w.eos_id),
        "fill_id": 0,
    }


# ---------------------------------------------------------------- token IDs

def _zipf_ids(rng, n: int, s: float, vocab: int) -> np.ndarray:
    """Zipf(s) over ranks 1..vocab by inverse CDF; id = rank - 1 (hot = small)."""
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int32)


def _doc_bounds(rng, total: int, lo: int, hi: int) -> np.ndarray:
    """Document boundaries covering [0, total); lengths U[lo, hi], last cut to fit."""
    bounds = [0]
    while bounds[-1] < total:
        bounds.append(min(total, bounds[-1] + int(rng.integers(lo, hi + 1))))
    return np.asarray(bounds, dtype=np.int64)


@lru_cache(maxsize=None)
def token_stream(name: str):
    """(ids int32 [T], cu_seqlens int32 [nseq+1]) for a named workload."""
    w = WORKLOADS[name]
    rng = np.random.Generator(np.random.PCG64(w.seed))
    T = w.tokens
    if w.id_dist == "uniform":
        ids = rng.integers(0, w.id_range, size=T, dtype=np.int64).astype(np.int32)
    else:
        ids = _zipf_ids(rng, T, w.zipf_s, w.id_range)
    if w.structure == "rows":
        if w.eos_p > 0:
            ids[rng.random(T) < w.eos_p] = w.eos_id
        cu = np.arange(0, T + 1, w.seq_len, dtype=np.int32)
    else:
        bounds = _doc_bounds(rng, T, *w.doc_len)
        ids[bounds[1:] - 1] = w.eos_id          # every document ends in EOS
        if w.structure == "docs_cu":
            cu = bounds.astype(np.int32)
        else:
            cu = np.asarray([0, T], dtype=np.int32)
    ids.setflags(write=False)
    cu.setflags(write=False)
    return ids, cu


def random_stream(seed: int, T: int, id_range: int, eos_id: int, eos_p: float,
                  nseq: int = 1, min_len: int = 0):
    """Small ad-hoc stream for tests: ids U[0,id_range) with EOS rate eos_p and
    nseq sequences of random lengths (>= min_len) summing to T."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ids = rng.integers(0, id_range, size=T, dtype=np.int64).astype(np.int32)
    if eos_p > 0:
        ids[rng.random(T) < eos_p] = eos_id
    if nseq <= 1:
        cu = np.asarray([0, T], dtype=np.int32)
    else:
        cuts = np.sort(rng.integers(0, T + 1, size=nseq - 1))
        cu = np.concatenate([[0], cuts, [T]]).astype(np.int32)
    return ids, cu


# ---------------------------------------------------------------- tables, dout

def host_table(name: str, rows: int | None = None, seed_offset: int = 0) -> np.ndarray:
    """N(0, 0.02) table in fp32 on the host (small workloads only)."""
    w = WORKLOADS[name]
    p = head_params(name)
    rows = p["table_rows"] if rows is None else rows
    rng = np.random.Generator(np.random.PCG64(2000 + w.seed + seed_offset))
    return (rng.standard_normal((rows, p["dim"])) * C.INITIALIZER_RANGE).astype(np.float32)


def fill_device_table(table, seed: int, std: float = C.INITIALIZER_RANGE,
                      chunk_rows: int = 1 << 22) -> None:
    """Fill a device table tensor [R, D] with seeded N(0, std) in chunks (torch)."""
    import torch
    g = torch.Generator(device=table.device)
    g.manual_seed(3000 + seed)
    for a in range(0, table.shape[0], chunk_rows):
        table[a:a + chunk_rows].normal_(0.0, std, generator=g)


def host_dout(name: str, n_lookups: int, dim: int, dtype: str, seed_offset: int = 0):
    """N(0,1) output gradient [n_lookups, dim] as a CPU torch tensor of `dtype`."""
    import torch
    w = WORKLOADS[name]
    g = torch.Generator()
    g.manual_seed(4000 + w.seed + seed_offset)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    return torch.randn(n_lookups, dim, generator=g, dtype=torch.float32).to(tdt)


# ------------------------------------------------------------ PLE layer tail

@dataclasses.dataclass(frozen=True)
class PleShape:
    """Shape of the PLE convolution tail: T tokens of C = branches * G channels."""
    name: str
    seed: int
    batch: int          # rows of the [batch, seq_len] token batch (cu_seqlens per row)
    seq_len: int
    branches: int       # hc_count
    group: int          # hidden_size, features normalised together
    kernel: int         # conv_kernel_size
    dilation: int       # short_conv_dilation = ngram_size
    dtype: str
    description: str = ""

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len

    @property
    def channels(self) -> int:
        return self.branches * self.group


PLE_SHAPES = {
    "ple_small": PleShape(
        "ple_small", 10, 3, 700, 4, 256, C.PLE_CONV_KERNEL, C.NGRAM_SIZE, "bf16",
        "3 x 700 tokens, 4 branches of 256 channels, kernel 4, dilation 3"),
    "ple_full": PleShape(
        "ple_full", 11, 16, 4096, C.HC_COUNT, C.HIDDEN_SIZE, C.PLE_CONV_KERNEL, C.NGRAM_SIZE,
        "bf16",
        "16 x 4,096 tokens (the full workload's batch), 4 HyperConnection branches "
        "of 2,560 channels (C = 10,240), kernel 4, dilation 3, bf16"),
}


def ple_inputs(T: int, channels: int, kernel: int, seed: int, dtype: str = "bf16"):
    """Host inputs of the PLE tail: x [T, C] ~ N(0, 1), norm scale [C] ~
    N(0, 0.1^2), conv weight [C, K] ~ N(0, 0.5^2), bias [C] ~ N(0, 0.1^2).

    Returns float32 arrays for "f32", else uint16 bit patterns of the dtype
    (rounded to nearest even by torch)."""
    import torch
    g = torch.Generator().manual_seed(5000 + int(seed))
    x = torch.randn((T, channels), generator=g, dtype=torch.float32)
    nw = 0.1 * torch.randn(channels, generator=g, dtype=torch.float32)
    w = 0.5 * torch.randn((channels, kernel), generator=g, dtype=torch.float32)
    b = 0.1 * torch.randn(channels, generator=g, dtype=torch.float32)

    def cast(t):
        if dtype == "f32":
            return t.numpy()
        tt = torch.bfloat16 if dtype == "bf16" else torch.float16
        return t.to(tt).view(torch.int16).numpy().view(np.uint16)

    return cast(x), cast(nw), cast(w), cast(b)


def row_bounds(batch: int, seq_len: int) -> np.ndarray:
    """cu_seqlens of a [batch, seq_len] batch: 0, S, 2S, ..., batch * S."""
    return (np.arange(batch + 1, dtype=np.int64) * seq_len).astype(np.int32)

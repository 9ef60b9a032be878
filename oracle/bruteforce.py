"""Arbitrary-precision brute-force hash for tiny inputs.

TEST INFRASTRUCTURE ONLY: an independent second statement of the Engram
N-gram hash (Qwen3.8-Flash-Next engram API page, NGramEmbedding), used to pin
the C oracle. It is organised differently from the C oracle on purpose:

* the stream is cut into segments instead of walking back from each token:
  a segment runs from a sequence start, or from the token after an EOS, up to
  and including the next EOS (or the sequence end), since an EOS terminates
  the segment before it;
* each segment is left-padded with ngram_size-1 fill values, so the context of
  every token is a plain window of the padded segment;
* products are exact Python integers reduced to signed 64-bit afterwards, and
  the remainder is Python's floor-mod.
"""

from __future__ import annotations

MASK64 = (1 << 64) - 1


def to_int64(v: int) -> int:
    """Reduce an exact integer to signed 64-bit two's complement."""
    v &= MASK64
    return v - (1 << 64) if v >> 63 else v


def segments(ids, cu, eos):
    """Yield (start, tokens) for every EOS-terminated piece of every sequence."""
    bounds = list(cu) if cu is not None else [0, len(ids)]
    for s in range(len(bounds) - 1):
        b, e = int(bounds[s]), int(bounds[s + 1])
        start = b
        for t in range(b, e):
            if int(ids[t]) == eos:
                yield start, [int(x) for x in ids[start:t + 1]]
                start = t + 1
        if start < e:
            yield start, [int(x) for x in ids[start:e]]


def hash_ids(ids, cu, params) -> list[list[int]]:
    """Row IDs [T][H] for a tiny stream, with exact integer arithmetic."""
    N = params["ngram_size"]
    K = params["heads_per_ngram"]
    mult = params["multipliers"]
    vocab = params["vocab_sizes"]
    off = params["offsets"]
    fill = params["fill_id"]
    eos = params["eos_id"]
    out = [None] * len(ids)
    for start, seg in segments(ids, cu, eos):
        padded = [fill] * (N - 1) + seg
        for i in range(len(seg)):
            window = padded[i:i + N]          # oldest ... current
            ctx = window[::-1]                # ctx[k] = token k places back
            prods = [to_int64(ctx[k] * mult[k]) for k in range(N)]
            row = []
            for n in range(2, N + 1):
                mix = 0
                for k in range(n):
                    mix ^= prods[k]
                for i_h in range(K):
                    h = (n - 2) * K + i_h
                    row.append(off[h] + mix % vocab[h])
            out[start + i] = row
    return out

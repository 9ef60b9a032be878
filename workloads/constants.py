"""Hash-head constants of the Qwen3.8-Flash-Next Engram N-gram Embedding table.

Source: the `qwen3_8_flash_next.engram` API page (NeMo AutoModel docs), module
data `QWEN3_8_FLASH_NEXT_LAYER_MULTIPLIERS`, `QWEN3_8_FLASH_NEXT_NGRAM_HEAD_VOCAB_SIZES`,
`QWEN3_8_FLASH_NEXT_NGRAM_HEAD_OFFSETS` and `QWEN3_8_FLASH_NEXT_NGRAM_PADDED_ROWS`.

The page prints the multipliers and the padded row count in full, but cuts the
two per-head tuples short: 8 of the 16 vocab sizes and 8 offsets plus the first
digits ("160...") of the ninth. This module keeps the printed values apart from
the inferred continuation:

* the 8 printed vocab sizes are exactly the 8 consecutive primes from 2*10**7;
  the remaining 8 heads take the next 8 consecutive primes;
* the printed offsets are exactly the running sums of the printed sizes, so
  every offset is the running sum of the sizes before it;
* the 16 sizes sum to 320,001,446; rounded up to a multiple of 128 (the page's
  128 checkpoint shards) that is 320,001,536, the printed padded row count.

These are configuration inputs of the method (the page calls the offsets
checkpoint-provided). Both the oracle and the CUDA path receive them; neither
computes them.
"""

from __future__ import annotations

# Printed in full on the engram API page (module data).
LAYER_MULTIPLIERS = (23703573157769, 20109073645365, 8052911324071)
PADDED_ROWS = 320001536
EOS_TOKEN_ID = 248044          # NGramEmbedding constructor default
NGRAM_SIZE = 3                 # NGramEmbedding constructor default
HEADS_PER_NGRAM = 8            # NGramEmbedding constructor default
EMBEDDING_DIM = 160            # row width of the [320001536, 160] table
INITIALIZER_RANGE = 0.02       # EngramTableConfig default std
TOKENIZER_VOCAB = 248320       # raw token ID range used by the workloads

# PLE layer (engram page, Qwen3_8_FlashNextPLELayer; model overview page,
# Architecture: four persistent HyperConnection streams of width 2,560).
HC_COUNT = 4                   # HyperConnection branches
HIDDEN_SIZE = 2560             # width of one branch (the norm group)
PLE_CONV_KERNEL = 4            # conv_kernel_size default
PLE_RMS_EPS = 1e-6             # rms_norm_eps default

# Printed prefix of the truncated tuples.
PRINTED_VOCAB_SIZES = (20000003, 20000023, 20000033, 20000047,
                       20000059, 20000063, 20000069, 20000077)
PRINTED_OFFSETS = (0, 20000003, 40000026, 60000059,
                   80000106, 100000165, 120000228, 140000297)
PRINTED_NINTH_OFFSET_PREFIX = "160"

# Inferred continuation (see module docstring): the next 8 consecutive primes.
INFERRED_VOCAB_SIZES = (20000081, 20000093, 20000107, 20000147,
                        20000153, 20000159, 20000161, 20000171)


def is_prime(n: int) -> bool:
    """Deterministic trial division; fine for the ~2e7 moduli used here."""
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def running_offsets(sizes) -> tuple[int, ...]:
    """Offsets of heads packed back to back: offset_h = sum of sizes before h."""
    out, acc = [], 0
    for s in sizes:
        out.append(acc)
        acc += s
    return tuple(out)


def page_head_tables():
    """(vocab_sizes[16], offsets[16], padded_rows) for the released table."""
    vocab = PRINTED_VOCAB_SIZES + INFERRED_VOCAB_SIZES
    offsets = running_offsets(vocab)
    return vocab, offsets, PADDED_ROWS

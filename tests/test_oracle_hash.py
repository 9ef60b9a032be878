"""Pins of the oracle hash (CPU only).

The engram page prints no hashed IDs, so the oracle's hash is pinned by:
  * the constants the page does print (tests/golden/page_constants.txt);
  * a hand-worked example written out below;
  * an independent exact-integer brute force on tiny and adversarial streams;
  * closed forms: multipliers with a single non-zero entry isolate one term;
  * invariants: head ranges, disjoint slices, reset after EOS, the value at a
    segment start, and the whole-stream/slice property of
    `_forward_global_slice` (hashing the full sequence preserves the two
    preceding tokens and EOS resets at a shard boundary).
"""

import numpy as np
import pytest

import oracle
from oracle import bruteforce
from tests.conftest import read_golden
from workloads import constants as C
from workloads import head_params, random_stream, token_stream


def small_params(seed=0, N=3, K=8, eos=999, fill=0, mult=None):
    """Seeded small moduli (distinct primes) packed back to back."""
    rng = np.random.Generator(np.random.PCG64(seed))
    primes = [p for p in range(200, 2000) if C.is_prime(p)]
    H = (N - 1) * K
    vocab = tuple(int(v) for v in rng.choice(primes, size=H, replace=False))
    offsets = C.running_offsets(vocab)
    if mult is None:
        mult = C.LAYER_MULTIPLIERS + (6364136223846793005,)
    return {
        "ngram_size": N, "heads_per_ngram": K,
        "multipliers": tuple(mult[:N]), "vocab_sizes": vocab, "offsets": offsets,
        "table_rows": offsets[-1] + vocab[-1], "dim": 160, "eos_id": eos,
        "fill_id": fill,
    }


# ---------------------------------------------------------------- page constants

def test_page_constants_fixture_matches_workloads():
    g = read_golden("page_constants.txt")
    assert tuple(g["layer_multipliers"]) == C.LAYER_MULTIPLIERS
    assert tuple(g["head_vocab_sizes_printed"]) == C.PRINTED_VOCAB_SIZES
    assert tuple(g["head_offsets_printed"]) == C.PRINTED_OFFSETS
    assert g["padded_rows"] == C.PADDED_ROWS
    assert g["eos_token_id"] == C.EOS_TOKEN_ID
    assert (g["ngram_size"], g["heads_per_ngram"]) == (C.NGRAM_SIZE, C.HEADS_PER_NGRAM)
    assert g["embedding_dim"] == C.EMBEDDING_DIM


def test_printed_sizes_are_consecutive_primes_and_offsets_running_sums():
    g = read_golden("page_constants.txt")
    sizes = g["head_vocab_sizes_printed"]
    consecutive = [p for p in range(20_000_000, 20_000_080) if C.is_prime(p)]
    assert consecutive == list(sizes)
    assert list(C.running_offsets(sizes)) == list(g["head_offsets_printed"])
    # the ninth offset (sum of the 8 printed sizes) begins with the printed "160"
    assert str(sum(sizes)).startswith(str(g["head_offset_9_prefix"]))


def test_inferred_continuation_reaches_padded_rows():
    g = read_golden("page_constants.txt")
    vocab, offsets, rows = C.page_head_tables()
    nxt = [p for p in range(20_000_078, 20_000_200) if C.is_prime(p)][:8]
    assert tuple(nxt) == C.INFERRED_VOCAB_SIZES
    total = offsets[-1] + vocab[-1]
    assert total == 320_001_446
    shards = g["checkpoint_shards"]
    assert -(-total // shards) * shards == g["padded_rows"] == rows
    assert rows - total < shards          # only the rounding gap is unused


def test_products_fit_int64_for_tokenizer_ids():
    # IDs < 248,320 times multipliers < 2**45 never wrap: mixes are >= 0 on the
    # page's workloads; the wrap and positive-remainder rules need larger IDs.
    assert max(C.LAYER_MULTIPLIERS) * (C.TOKENIZER_VOCAB - 1) < 2 ** 63


# ---------------------------------------------------------------- worked example

def test_hand_worked_example():
    # multipliers (3, 5, 7), one head per order (K=1): bigram mod 11 at offset 0,
    # trigram mod 13 at offset 11; EOS = 9; fill = 0. Stream [2, 4, 9, 6]:
    #  t=0 x=(2,0,0): mix2 = 6,            mix3 = 6        -> (6, 11+6)
    #  t=1 x=(4,2,0): mix2 = 12^10 = 6,    mix3 = 6        -> (6, 11+6)
    #  t=2 x=(9,4,2): mix2 = 27^20 = 15,   mix3 = 15^14=1  -> (15%11=4, 11+1)
    #  t=3 after EOS, x=(6,0,0): mix2 = mix3 = 18          -> (18%11=7, 11+18%13=16)
    p = {"ngram_size": 3, "heads_per_ngram": 1, "multipliers": (3, 5, 7),
         "vocab_sizes": (11, 13), "offsets": (0, 11), "table_rows": 24,
         "dim": 160, "eos_id": 9, "fill_id": 0}
    got = oracle.hash_ids(np.array([2, 4, 9, 6], np.int32), None, p)
    assert got.tolist() == [[6, 17], [6, 17], [4, 12], [7, 16]]
    # a sequence boundary at t=1 resets like an EOS does: t=1 now sees (4,0,0)
    got = oracle.hash_ids(np.array([2, 4, 9, 6], np.int32), np.array([0, 1, 4]), p)
    assert got[1].tolist() == [12 % 11, 11 + 12 % 13]
    # negative mix: 2**62 * 3 wraps to -2**62 (mod 2**64) at t=0 with fill 0;
    # floor-mod keeps the remainder in [0, p)
    p2 = dict(p, multipliers=(3 << 60, 5, 7), eos_id=-1)
    got = oracle.hash_ids(np.array([4], np.int32), None, p2)
    mix = -(1 << 62)          # 4 * 3 * 2**60 = 3 * 2**62 -> -2**62
    assert got[0].tolist() == [mix % 11, 11 + mix % 13]
    assert mix % 11 != abs(mix) % 11  # a truncating remainder would differ


# ---------------------------------------------------------------- brute force

ADVERSARIAL = [
    # (ids, cu) -- eos is 999
    ([999], None),
    ([999, 999, 999], None),
    ([5, 999], None),
    ([999, 5, 6, 7], None),
    ([5, 6, 999, 999, 7, 8], None),
    ([1, 2, 3, 4, 5, 999], None),
    ([0, 0, 0, 0], None),                                # fill-equal IDs
    ([2 ** 31 - 1, 2 ** 31 - 2, 2 ** 31 - 3, 7], None),  # products wrap
    ([-1, -2 ** 31, 5, -7], None),                       # negative raw IDs
    ([3, 4, 5, 6, 7], [0, 1, 2, 3, 5]),                  # length-1/2 sequences
    ([3, 4, 5, 6, 7, 8], [0, 0, 3, 3, 6]),               # empty sequences
    ([999, 1, 2, 999, 3], [0, 2, 5]),
    ([], None),
]


@pytest.mark.parametrize("fill", [0, 17])
@pytest.mark.parametrize("case", range(len(ADVERSARIAL)))
def test_bruteforce_adversarial(case, fill):
    ids, cu = ADVERSARIAL[case]
    p = small_params(seed=case, eos=999, fill=fill)
    ids = np.array(ids, dtype=np.int32)
    cu_a = None if cu is None else np.array(cu, dtype=np.int32)
    got = oracle.hash_ids(ids, cu_a, p)
    want = bruteforce.hash_ids(ids, cu_a, p)
    assert got.tolist() == [list(r) for r in want]


@pytest.mark.parametrize("N,K", [(2, 3), (3, 8), (4, 2)])
@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_random(seed, N, K):
    p = small_params(seed=seed, N=N, K=K, eos=7, fill=seed % 2)
    id_range = [20, 1000, 2 ** 31 - 1][seed % 3]
    ids, cu = random_stream(seed, 300, id_range, 7, 0.08, nseq=1 + seed)
    if id_range > 1000:   # also large negative IDs
        ids = ids.copy()
        ids[::5] = -ids[::5]
    got = oracle.hash_ids(ids, cu, p)
    want = bruteforce.hash_ids(ids, cu, p)
    assert got.tolist() == [list(r) for r in want]


def test_bruteforce_covers_negative_mixes():
    p = small_params(seed=3)
    ids = np.array([2 ** 31 - 1, 2 ** 30 + 12345, 2 ** 31 - 77, 99], dtype=np.int32)
    prods = [bruteforce.to_int64(int(x) * p["multipliers"][0]) for x in ids]
    assert any(v < 0 for v in prods)
    assert oracle.hash_ids(ids, None, p).tolist() == bruteforce.hash_ids(ids, None, p)


# ---------------------------------------------------------------- closed forms

def test_single_term_multipliers_isolate_positions():
    ids, cu = random_stream(11, 200, 5000, 4999, 0.05, nseq=3)
    eos = 4999
    base = small_params(seed=5, eos=eos)
    K = base["heads_per_ngram"]
    vocab = np.array(base["vocab_sizes"], dtype=np.int64)
    off = np.array(base["offsets"], dtype=np.int64)
    # context of every token by the segment rule, written out directly
    starts = np.zeros(len(ids), dtype=np.int64)
    seq_start = {int(c) for c in cu[:-1]}
    s = 0
    for t in range(len(ids)):
        if t in seq_start or (t > 0 and ids[t - 1] == eos):
            s = t
        starts[t] = s
    x = np.zeros((len(ids), 3), dtype=np.int64)
    for t in range(len(ids)):
        for k in range(3):
            x[t, k] = ids[t - k] if t - k >= starts[t] else 0
    for k, m in enumerate([12345, 67891, 23456]):
        mult = [0, 0, 0]
        mult[k] = m
        p = dict(base, multipliers=tuple(mult))
        got = oracle.hash_ids(ids, cu, p) - off
        term = x[:, k] * m                                # no wrap for these sizes
        mix2 = term if k < 2 else np.zeros_like(term)     # bigram uses x0, x1 only
        mix3 = term
        np.testing.assert_array_equal(got[:, :K], mix2[:, None] % vocab[None, :K])
        np.testing.assert_array_equal(got[:, K:], mix3[:, None] % vocab[None, K:])


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("name", ["tiny", "b4x4096"])
def test_rows_inside_head_slices(name):
    p = head_params(name)
    ids, cu = token_stream(name)
    idx = oracle.hash_ids(ids, cu, p)
    lo = np.array(p["offsets"])
    hi = lo + np.array(p["vocab_sizes"])
    assert (idx >= lo).all() and (idx < hi).all() and (idx < p["table_rows"]).all()
    assert (hi[:-1] <= lo[1:]).all()                    # disjoint, ascending slices


def test_page_slices_disjoint_and_below_padded_rows():
    vocab, offsets, rows = C.page_head_tables()
    for h in range(15):
        assert offsets[h] + vocab[h] <= offsets[h + 1]
    assert offsets[15] + vocab[15] <= rows


def test_token_after_eos_hashes_like_sequence_start():
    p = head_params("full")
    eos = p["eos_id"]
    rng = np.random.Generator(np.random.PCG64(9))
    for _ in range(20):
        tail = rng.integers(0, 248320, size=5).astype(np.int32)
        head = rng.integers(0, 248320, size=rng.integers(0, 6)).astype(np.int32)
        a = oracle.hash_ids(np.concatenate([head, [eos], tail]).astype(np.int32), None, p)
        b = oracle.hash_ids(tail, None, p)
        np.testing.assert_array_equal(a[-5:], b)


def test_segment_start_closed_form():
    p = head_params("full")
    m0 = p["multipliers"][0]
    ids, cu = token_stream("full")
    idx = oracle.hash_ids(ids[:8192], np.array([0, 4096, 8192], np.int32), p)
    starts = [0, 4096] + [t + 1 for t in range(8191) if ids[t] == p["eos_id"] and t + 1 != 4096]
    for t in starts:
        want = [o + (int(ids[t]) * m0) % v for o, v in zip(p["offsets"], p["vocab_sizes"])]
        assert idx[t].tolist() == want


def test_eos_token_keeps_its_own_left_context():
    p = small_params(seed=1, eos=999)
    a = oracle.hash_ids(np.array([5, 6, 999], np.int32), None, p)
    b = oracle.hash_ids(np.array([999], np.int32), None, p)
    assert a[2].tolist() != b[0].tolist()   # EOS ends the segment it closes


@pytest.mark.parametrize("start,end", [(0, 1), (1, 2), (2, 3), (100, 355), (4095, 4097),
                                       (4096, 8192), (8000, 8192)])
def test_global_slice_equals_slice_of_global_hash(start, end):
    # `_forward_global_slice`: hashing the whole sequence and keeping [start, end)
    # equals hashing [start-2, end) and dropping the 2-token halo, as long as the
    # halo does not reach past a reset (it is cut at sequence starts and EOS).
    p = head_params("full")
    ids, cu = token_stream("full")
    ids, cu = ids[:8192], np.array([0, 4096, 8192], np.int32)
    whole = oracle.hash_ids(ids, cu, p)[start:end]
    lo = max(0, start - 2)
    if lo < 4096 <= start:
        lo = 4096
    sub_cu = np.array([0, end - lo], np.int32)
    if lo < 4096 < end:
        sub_cu = np.array([0, 4096 - lo, end - lo], np.int32)
    part = oracle.hash_ids(ids[lo:end], sub_cu, p)[start - lo:]
    np.testing.assert_array_equal(whole, part)

"""Pins of the oracle's delta + entropy stage over the lattice indices.

The pages say only that consecutive tokens give similar lattice indices, that
the differences are stored and compressed (zingnex.cn "Implementation
details"; dev.to step 6, with zstd); the coder here is rANS (Duda, 2013) with a
static table, so the pins come from its definition and from arithmetic:

* the table rule on counts worked out by hand;
* the coded size against a bound proven from the state update: with the state
  x >= 2^16 before every step and f <= 4096, one step multiplies x by at most
  (M / f)(1 + f / x) <= (M / f)(17 / 16), and every emitted word removes 16
  bits, so 16 * words <= sum_t log2(M / F_{s_t}) + n log2(17/16) + 32;
* a stream of one symbol with F = M never changes the state (closed form);
* round trips, and a numpy restatement of the stream layout (segments,
  coordinate order, differences mod 2^b) and of the per-(unit, head) counts;
* streams worked out by hand from the coder's definition
  (tests/golden/rans_examples.txt).
"""
import math
import os

import numpy as np
import pytest

import oracle as oq

M = 4096


def test_table_rule_worked_examples():
    # counts (1, 0, 3, 996), total 1000: floor(c * 4096 / 1000) = 4, -, 12, 4079
    # (4.096, 12.288, 4079.616); sum 4095, remainder +1 to the largest -> 4080
    assert oq.ans_table([1, 0, 3, 996]).tolist() == [4, 0, 12, 4080]
    # (1, 1, 1, 10^6): floor(4096 / 1000003) = 0 -> 1 each; floor(4096e6 / 1000003)
    # = 4095 (4095.9877); sum 4098, remainder -2 -> 4093
    assert oq.ans_table([1, 1, 1, 1000000]).tolist() == [1, 1, 1, 4093]
    assert oq.ans_table([5] * 8).tolist() == [512] * 8
    assert oq.ans_table([7, 0, 0, 0]).tolist() == [4096, 0, 0, 0]
    # ties for the largest go to the lowest symbol: (3, 3) -> 2048 each, no remainder;
    # (1, 1, 1) -> 1365 each, remainder 1 to symbol 0
    assert oq.ans_table([1, 1, 1, 0]).tolist() == [1366, 1365, 1365, 0]


def test_table_properties_on_random_counts():
    rng = np.random.default_rng(1)
    for _ in range(500):
        A = int(rng.choice([4, 8]))
        c = rng.integers(0, 1000, A) * (rng.random(A) < 0.7)
        if c.sum() == 0:
            c[0] = 1
        if rng.random() < 0.3:
            c[rng.integers(A)] = rng.integers(10**6, 10**9)
        F = oq.ans_table(c).astype(np.int64)
        assert F.sum() == M
        assert np.all((F == 0) == (c == 0))
        ideal = c * M / c.sum()
        assert np.all(np.abs(F - ideal) <= A + 1)


def cost_bits(sym, F):
    return float(np.sum(np.log2(M / F[sym].astype(np.float64))))


@pytest.mark.parametrize("A", [4, 8])
def test_round_trip_and_size_bound(A):
    rng = np.random.default_rng(A)
    for trial in range(40):
        n = int(rng.choice([0, 1, 2, 3, 100, 2048, 20000]))
        p = rng.dirichlet(np.full(A, 0.3 if trial % 2 else 3.0))
        sym = rng.choice(A, size=n, p=p).astype(np.uint8)
        counts = np.bincount(sym, minlength=A)
        if n == 0:
            counts[0] = 1
        F = oq.ans_table(counts)
        w = oq.ans_encode(sym, F)
        back, used = oq.ans_decode(w, F, n)
        assert used == w.size and np.array_equal(back, sym)
        assert 16 * w.size <= cost_bits(sym, F) + n * math.log2(17 / 16) + 32 + 1e-6


def test_rare_symbols_and_worst_case_table():
    # the rarest possible symbol (F = 1) costs 12 bits a step: the bound still holds
    F = np.array([4093, 1, 1, 1], np.uint16)
    sym = np.array([1, 2, 3] * 300 + [0] * 50, np.uint8)
    w = oq.ans_encode(sym, F)
    back, used = oq.ans_decode(w, F, sym.size)
    assert used == w.size and np.array_equal(back, sym)
    assert 16 * w.size <= cost_bits(sym, F) + sym.size * math.log2(17 / 16) + 32
    assert 16 * w.size >= 12 * 900  # 900 symbols at 12 bits each cannot shrink


def test_single_symbol_stream_is_the_initial_state():
    # F_0 = M: x = floor(x / M) M + x mod M = x, and x < 2^32 = F_0 2^20 never
    # emits, so the stream is the initial state 2^16 = (low 0, high 1)
    F = np.array([4096, 0, 0, 0, 0, 0, 0, 0], np.uint16)
    for n in (0, 1, 5000):
        w = oq.ans_encode(np.zeros(n, np.uint8), F)
        assert w.tolist() == [0, 1]


def test_long_streams_come_close_to_the_model_entropy():
    rng = np.random.default_rng(7)
    p = np.array([0.4, 0.25, 0.15, 0.1, 0.05, 0.03, 0.015, 0.005])
    sym = rng.choice(8, size=200000, p=p).astype(np.uint8)
    F = oq.ans_table(np.bincount(sym, minlength=8))
    w = oq.ans_encode(sym, F)
    assert 16 * w.size <= 1.0005 * cost_bits(sym, F) + 64


def np_codes(codes, bits):
    """Codes j [..., 128] of packed words [..., 4*bits] (code c at bits [b c, b c + b))."""
    w = codes.astype(np.uint64)
    out = np.zeros(codes.shape[:-1] + (128,), np.int64)
    for c in range(128):
        for k in range(bits):
            p = bits * c + k
            out[..., c] |= ((w[..., p >> 5] >> np.uint64(p & 31)) & np.uint64(1)).astype(np.int64) << k
    return out


def np_streams(j, bits, delta, seg=oq.ANS_SEG):
    """Per (unit, head): list of (segment, coordinate) symbol arrays, stream order."""
    units, heads, n, _ = j.shape
    res = []
    for u in range(units):
        for h in range(heads):
            streams = []
            for g in range(0, n, seg):
                blk = j[u, h, g:g + seg]
                if delta:
                    d = np.diff(blk, axis=0, prepend=0) % (1 << bits)
                else:
                    d = blk
                for c in range(128):
                    streams.append(d[:, c].astype(np.uint8))
            res.append(streams)
    return res


@pytest.mark.parametrize("bits,n,delta", [(3, 1, True), (2, 2047, True), (3, 2048, False),
                                          (3, 2049, True), (2, 3000, False)])
def test_store_layout_matches_a_numpy_restatement(bits, n, delta):
    rng = np.random.default_rng(n + bits)
    units, heads = 2, 3
    # codes with token-to-token correlation: a random walk on the code values
    j = np.cumsum(rng.integers(-1, 2, (units, heads, n, 128)), axis=2) % (1 << bits)
    codes = np.zeros((units, heads, n, 4 * bits), np.uint32)
    for c in range(128):
        for k in range(bits):
            p = bits * c + k
            codes[..., p >> 5] |= (((j[..., c] >> k) & 1).astype(np.uint32) << np.uint32(p & 31))
    assert np.array_equal(np_codes(codes, bits), j)
    freq, offsets, words = oq.entropy_encode_store(codes, bits, delta)
    streams = np_streams(j, bits, delta)
    A = 1 << bits
    s = 0
    for uh, st in enumerate(streams):
        counts = np.bincount(np.concatenate(st), minlength=A)
        F = freq.reshape(-1, A)[uh]
        assert np.array_equal(F, oq.ans_table(counts))
        for sym in st:
            seg = words[offsets[s]:offsets[s + 1]]
            back, used = oq.ans_decode(seg, F, sym.size)
            assert used == seg.size and np.array_equal(back, sym)
            s += 1
    assert s == offsets.size - 1 == oq.entropy_streams(units, heads, n)
    assert offsets[-1] == words.size
    back = oq.entropy_decode_store(words, offsets, freq, units, heads, n, bits, delta)
    assert np.array_equal(back, codes)


def test_differences_pay_off_on_correlated_codes():
    # a slow random walk: differences take 3 values, the codes all 8
    rng = np.random.default_rng(3)
    n = 4096
    j = np.cumsum(rng.integers(-1, 2, (1, 1, n, 128)) * (rng.random((1, 1, n, 128)) < 0.2),
                  axis=2) % 8
    codes = np.zeros((1, 1, n, 12), np.uint32)
    for c in range(128):
        for k in range(3):
            p = 3 * c + k
            codes[..., p >> 5] |= (((j[..., c] >> k) & 1).astype(np.uint32) << np.uint32(p & 31))
    _, _, w_delta = oq.entropy_encode_store(codes, 3, True)
    _, _, w_plain = oq.entropy_encode_store(codes, 3, False)
    assert w_delta.size < 0.5 * w_plain.size


GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rans_examples.txt")


def load_rans_golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        f, s, w = (part.split() for part in line.split("|"))
        rows.append((np.array(f, np.uint16), np.array(s, np.uint8), [int(x) for x in w]))
    return rows


def test_hand_worked_streams():
    rows = load_rans_golden()
    assert len(rows) == 3
    for F, sym, words in rows:
        w = oq.ans_encode(sym, F)
        assert w.tolist() == words
        back, used = oq.ans_decode(np.array(words, np.uint16), F, sym.size)
        assert used == len(words) and np.array_equal(back, sym)

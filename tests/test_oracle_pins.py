"""Pins of the oracle to things other than itself.

Each check compares the oracle with brute force, a closed form, an invariant, a textbook
library routine, or a hand-derived tiny case -- chosen so that a dropped term, a wrong sign or
index, or a transposed operand anywhere in the oracle fails at least one of them.

Sources of the method, by page and section: "EntroPack lattice compression" (documentation page
Principles / Lattice-rANS), sections "Lattice quantization and integer fields" (LQ), "Rate
selection and refinement" (RS), "Encoding and reconstruction" (ER); the EntroPack arXiv abstract.

Pin map (oracle function -> test):
  orc_e8_nearest          -> test_e8_matches_brute_force, test_e8_adversarial_ties
  orc_point_to_fields /
  orc_fields_to_point     -> test_fields_bijection_and_parity, test_fields_enumerated_box
  orc_quantize_table      -> test_table_hand_cases, test_table_invariants
  orc_encode_tile /
  orc_decode_tile         -> test_rans_closed_form_one_bit_symbols, test_rans_all_escape_closed_form,
                             test_rans_lone_symbols_closed_form, test_rans_roundtrip_random,
                             test_rans_size_near_cross_entropy
  orc_dtype_to_f64        -> test_dtype_decode_vs_numpy_torch
  orc_f32_to_bf16/f16/
  e4m3/i8, orc_round_f32  -> test_conversions_vs_library
  INT8 store and read     -> test_int8_container_round_trip
  orc_compress (RMS, LS,
  scale search, tiling)   -> test_end_to_end_fields_vs_independent_quantiser, test_rms_scale_invariance,
                             test_least_squares_orthogonality, test_constant_rows_exact,
                             test_high_rate_distortion_closed_form, test_shannon_bound,
                             test_estimate_full_sample_vs_actual, test_estimate_sampled_vs_actual
  row-maximum section     -> test_end_to_end_fields_vs_independent_quantiser
  orc_row_gain /
  orc_row_sigma           -> test_fp8_row_scale_closed_forms
  orc_decompress_rowscaled_tiles -> test_fp8_rowscaled_payload
  prob_bits (12 / 10)     -> every table and rANS pin at both totals, test_rans_totals_are_not_interchangeable,
                             test_twelve_bit_totals_code_no_longer_than_ten_bit
  orc_actual_bpp          -> test_actual_bpp_definition
  rd refinement           -> test_rd_refinement_off_is_the_default,
                             test_rd_refinement_gives_loud_rows_finer_resolution,
                             test_rd_refinement_meets_budget_and_lowers_error
  target range            -> test_target_range
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W

RNG = np.random.Generator(np.random.PCG64(7))


# ---------------------------------------------------------------------------------------------
# E8 nearest point: brute force over the box [floor(t) - 1, ceil(t) + 1]^8 for both cosets.
# ---------------------------------------------------------------------------------------------

def _brute_e8(t):
    """Minimum squared distance from t to E8 and the (unique or first) argmin, by enumeration."""
    best = (np.inf, None)
    for half in (0.0, 0.5):
        base = np.floor(t - half) + half
        opts = base[:, None] + np.arange(-1, 3)[None, :]          # 8 x 4 candidates
        cost = (t[:, None] - opts) ** 2
        # all 4^8 combinations
        idx = np.indices((4,) * 8).reshape(8, -1)
        pts = opts[np.arange(8)[:, None], idx]                     # 8 x 65536
        d = cost[np.arange(8)[:, None], idx].sum(axis=0)
        z = pts - half
        even = (np.rint(z).astype(np.int64).sum(axis=0) % 2) == 0
        d = np.where(even, d, np.inf)
        k = int(np.argmin(d))
        if d[k] < best[0]:
            best = (d[k], pts[:, k].copy())
    return best


def _in_e8(y):
    y = np.asarray(y)
    twice = 2 * y
    if not np.allclose(twice, np.rint(twice)):
        return False
    frac = y - np.floor(y)
    if not (np.all(frac == 0) or np.all(frac == 0.5)):
        return False
    z = y - frac[0]
    return int(np.rint(z).sum()) % 2 == 0


def test_e8_matches_brute_force():
    n = 1500
    t = np.concatenate([RNG.normal(0, 1.5, (n // 3, 8)), RNG.normal(0, 6, (n // 3, 8)),
                        RNG.uniform(-3, 3, (n - 2 * (n // 3), 8))])
    y, c = oracle.e8_nearest(t)
    for i in range(n):
        assert _in_e8(y[i]), y[i]
        assert (c[i] == 1) == (y[i, 0] - np.floor(y[i, 0]) == 0.5)
        dmin, arg = _brute_e8(t[i])
        d = ((t[i] - y[i]) ** 2).sum()
        assert abs(d - dmin) <= 1e-12 * max(1.0, dmin), (t[i], y[i], arg)


def test_e8_adversarial_ties():
    cases = [np.zeros(8), np.full(8, 0.5), np.full(8, 0.25), np.full(8, -0.25),
             np.array([1, 0, 0, 0, 0, 0, 0, 0.0]),               # integer vector, odd sum
             np.array([0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, -0.5]),
             np.array([1.5, -2.5, 0.5, 3.5, -0.5, 0.5, 7.5, 2.5]),
             np.array([0.75] * 8), np.array([-0.75] * 8), np.arange(8) * 0.5 - 2.0,
             np.array([32764.0, -32764.0, 32763.5, 0.1, 0.2, 0.3, -0.4, 0.49])]
    rnd = np.round(RNG.normal(0, 3, (300, 8)) * 4) / 4                # quarter-integer grid: many ties
    for t in list(cases) + list(rnd):
        y, c = oracle.e8_nearest(t)
        assert _in_e8(y[0])
        dmin, _ = _brute_e8(t)
        assert abs(((t - y[0]) ** 2).sum() - dmin) <= 1e-9


# ---------------------------------------------------------------------------------------------
# Coset bit + fields: bijection, even-sum invariant, inverse exact.
# ---------------------------------------------------------------------------------------------

def _random_e8_points(n, spread):
    z = RNG.integers(-spread, spread + 1, (n, 8))
    z[:, 7] += z.sum(axis=1) % 2                                   # make the sum even
    c = RNG.integers(0, 2, n)
    return z + 0.5 * c[:, None], c, z


def test_fields_bijection_and_parity():
    y, c, z = _random_e8_points(200_000, 300)
    f = oracle.point_to_fields(y, c)
    assert np.all(z.sum(axis=1) % 2 == 0)
    # fields 1..7 are the D8 coordinates; the 8th is compacted by the parity of the first seven
    assert np.array_equal(f[:, :7], z[:, :7])
    par = z[:, :7].sum(axis=1) % 2
    assert np.array_equal(2 * f[:, 7] + par, z[:, 7])
    assert np.all(np.abs(f[:, 7]) <= (np.abs(z[:, 7]) + 1) // 2)
    y2 = oracle.fields_to_point(c, f)
    assert np.array_equal(y2, y)


def test_fields_enumerated_box():
    # every E8 point with coordinates in [-2, 2] (both cosets): fields distinct, inverse exact
    vals = np.arange(-2, 3)
    grid = np.array(np.meshgrid(*([vals] * 8), indexing="ij")).reshape(8, -1).T
    ints = grid[grid.sum(axis=1) % 2 == 0]
    halves = np.array(np.meshgrid(*([np.arange(-2, 2) + 0.5] * 8), indexing="ij")).reshape(8, -1).T
    halves = halves[(halves - 0.5).sum(axis=1) % 2 == 0]
    y = np.concatenate([ints, halves]).astype(np.float64)
    c = np.concatenate([np.zeros(len(ints), np.int32), np.ones(len(halves), np.int32)])
    f = oracle.point_to_fields(y, c)
    keys = np.concatenate([c[:, None], f], axis=1)
    assert len(np.unique(keys, axis=0)) == len(keys)
    assert np.array_equal(oracle.fields_to_point(c, f), y)


# ---------------------------------------------------------------------------------------------
# Frequency tables: every table sums to M = 2^prob_bits, 4096 (12-bit totals, the format's
# default) or 1024 (10-bit).
# ---------------------------------------------------------------------------------------------

PBS = (12, 10)
M = 4096        # the default total


def _q(counts, pb=12):
    a = np.zeros(256, np.uint64)
    for s, n in counts.items():
        a[s] = n
    return oracle.quantize_table(a, pb)


def test_table_hand_cases():
    # 12-bit totals
    q = _q({0: 1, 1: 1}); assert (q[0], q[1]) == (2048, 2048)
    q = _q({5: 3, 9: 1}); assert (q[5], q[9]) == (3072, 1024)
    q = _q({200: 17}); assert q[200] == 4096 and q.sum() == 4096
    # 4096/3 = 1365.33 -> 1365 each, sum 4095 -> +1 to the largest count, lowest symbol first
    q = _q({1: 1, 2: 1, 3: 1}); assert (q[1], q[2], q[3]) == (1366, 1365, 1365)
    # a rare symbol keeps frequency 1; the big one (4096 * 10^6 / (10^6 + 1) -> 4096) gives back one
    q = _q({0: 1_000_000, 255: 1}); assert (q[0], q[255]) == (4095, 1)
    counts = {s: 1 for s in range(200)}
    counts[250] = 1_000_000
    q = _q(counts)
    assert all(q[s] == 1 for s in range(200)) and q[250] == 4096 - 200
    assert _q({}).sum() == 0
    # 10-bit totals
    q = _q({0: 1, 1: 1}, 10); assert (q[0], q[1]) == (512, 512)
    q = _q({5: 3, 9: 1}, 10); assert (q[5], q[9]) == (768, 256)
    q = _q({200: 17}, 10); assert q[200] == 1024 and q.sum() == 1024
    q = _q({1: 1, 2: 1, 3: 1}, 10); assert (q[1], q[2], q[3]) == (342, 341, 341)
    q = _q({0: 1_000_000, 255: 1}, 10); assert (q[0], q[255]) == (1023, 1)
    q = _q(counts, 10)
    assert all(q[s] == 1 for s in range(200)) and q[250] == 1024 - 200


@pytest.mark.parametrize("pb", PBS)
def test_table_invariants(pb):
    Mp = 1 << pb
    for _ in range(300):
        n = np.zeros(256, np.uint64)
        k = RNG.integers(1, 257)
        sel = RNG.choice(256, k, replace=False)
        n[sel] = RNG.integers(1, 10 ** RNG.integers(1, 7), k)
        q = oracle.quantize_table(n, pb)
        assert int(q.sum()) == Mp
        assert np.array_equal(q > 0, n > 0)
        ideal = Mp * n / n.sum()
        # Rounding moves each symbol at most 1/2 from its share (less than 1 for the r symbols
        # raised to 1), so the excess or deficit the repair loop removes is at most k/2 + r/2,
        # and it can all land on one symbol.
        r = int(((ideal < 0.5) & (n > 0)).sum())
        assert np.all(np.abs(q - ideal) <= 1.0 + k / 2 + r / 2)
        assert np.abs(q - ideal).sum() <= 2.0 * (k / 2 + r / 2) + 1e-9


def test_joint_coset_f1_table():
    """Contexts 0 and 8 (field 1 given coset 0 / 1) are one table over the 512 pairs (c, f1):
    the same quantisation rule on the concatenated counts, coset 0 first on ties."""
    counts = np.zeros((16, 256), np.uint64)
    counts[0, 5], counts[8, 5] = 3, 1                   # 3 : 1 over the pair -> 3072 : 1024
    counts[1, [0, 1]] = 1                               # a context on its own -> 2048 : 2048
    q = oracle.build_tables16(counts)
    assert (q[0, 5], q[8, 5]) == (3072, 1024) and (q[1, 0], q[1, 1]) == (2048, 2048)
    assert q[2:8].sum() == 0 and q[9:].sum() == 0       # empty contexts stay empty
    q = oracle.build_tables16(counts, 10)
    assert (q[0, 5], q[8, 5]) == (768, 256) and (q[1, 0], q[1, 1]) == (512, 512)
    counts = np.zeros((16, 256), np.uint64)
    counts[0, 7], counts[8, 7] = 1, 1                   # 4096 / 3 -> 1365 each, sum 4095: the
    counts[0, 8] = 1                                    # first largest count (coset 0, 7) gets +1
    q = oracle.build_tables16(counts)
    assert (q[0, 7], q[0, 8], q[8, 7]) == (1366, 1365, 1365)
    for pb in PBS:
        Mp = 1 << pb
        for _ in range(50):
            c = np.zeros((16, 256), np.uint64)
            for ctx in range(16):
                k = RNG.integers(0, 60)
                c[ctx, RNG.choice(256, k, replace=False)] = RNG.integers(1, 10 ** 4, k)
            if c[0].sum() + c[8].sum() == 0:
                c[0, 127] = 1
            q = oracle.build_tables16(c, pb)
            assert int(q[0].sum()) + int(q[8].sum()) == Mp
            assert np.array_equal(q[[0, 8]] > 0, c[[0, 8]] > 0)
            for ctx in set(range(16)) - {0, 8}:
                assert int(q[ctx].sum()) in (0, Mp) and np.array_equal(q[ctx], oracle.quantize_table(c[ctx], pb))


# ---------------------------------------------------------------------------------------------
# rANS tiles.
# ---------------------------------------------------------------------------------------------

def _tables(field_q: dict):
    """16 x 256 tables for vectors that are all in coset 0: the joint (coset, f1) table is field_q
    on its coset-0 half (context 0) and empty on its coset-1 half (context 8); every other
    context equals field_q."""
    q16 = np.zeros((16, 256), np.uint16)
    for ctx in range(16):
        if ctx == 8:
            continue
        for s, q in field_q.items():
            q16[ctx, s] = q
    return q16


@pytest.mark.parametrize("pb", PBS)
def test_rans_closed_form_one_bit_symbols(pb):
    """Two steps, 32 lanes, every field one bit (q = M/2 = 2^(pb-1) for f = 0 and f = 1), coset
    free.  Encoding x <- floor(x/q)*M + (x mod q) + q*b = 2x + q*b (x stays a multiple of q) from
    x = 2^16 gives, after n bits b_1..b_n (first encoded first), x = 2^(16+n) + q * B_n with
    B_n = sum_i b_i 2^(n-i), while x < 2^31 (the renormalisation bound q * (L/M) * 2^16 = 2^31
    for any M).  A lane meets its 16 bits in reverse reading order: step 1 f8..f1, then step 0
    f8..f2, then step 0 f1; before the 16th, x = 2^31 + q*B15 >= 2^31, so it emits the low 16
    bits q * (B15 mod 2^(17-pb)) and keeps 2^15 + (B15 >> (17-pb)); encoding f1 then gives the
    initial state 2^16 + q*f1 + (B15 >> (17-pb)).  Every lane has exactly one word, so each
    region holds 2 words: lane 2p's (read forward from the region start) then lane 2p+1's (read
    backward from the region end) -- lane order overall."""
    q = 1 << (pb - 1)
    q16 = _tables({127: q, 128: q})
    bits = RNG.integers(0, 2, (64, 8))                              # vector v = 32k + lane
    sym9 = np.zeros((64, 9), np.uint8)
    sym9[:, 1:] = 127 + bits
    raw8 = np.zeros((64, 8), np.int16)
    tile = oracle.encode_tile(sym9, raw8, q16, pb)
    assert len(tile) == 160 + 64
    states = np.frombuffer(tile[:128], "<u4")
    counts = np.frombuffer(tile[128:160], "<u2")
    words = np.frombuffer(tile[160:], "<u2")
    assert np.all(counts == 2)
    sh = 17 - pb
    for lane in range(32):
        f0 = bits[lane]            # step 0: f1..f8 at indices 0..7
        f1 = bits[32 + lane]       # step 1
        step1 = sum(int(f1[j]) << j for j in range(8))             # f8 most significant
        step0_hi = sum(int(f0[j]) << (j - 1) for j in range(1, 8))  # f8..f2, f8 most significant
        b15 = (step1 << 7) | step0_hi
        assert states[lane] == 65536 + q * int(f0[0]) + (b15 >> sh)
        assert words[lane] == q * (b15 & ((1 << sh) - 1))
    rc, s9, r8, st = oracle.decode_tile(tile, 64, q16, pb)
    assert rc == 0 and np.array_equal(s9, sym9) and np.all(st == 65536)


@pytest.mark.parametrize("pb", PBS)
def test_rans_all_escape_closed_form(pb):
    """Coset free, every field the escape symbol with q = M: no state ever changes, so each
    lane's words are its raw values in step, field order; region p holds lane 2p's words forward
    and lane 2p+1's words backward from the region end."""
    q16 = _tables({255: 1 << pb})
    nvec = 70                                                       # 3 steps, the last partial
    sym9 = np.zeros((nvec, 9), np.uint8)
    sym9[:, 1:] = 255
    raw8 = RNG.integers(-32768, 32768, (nvec, 8)).astype(np.int16)
    tile = oracle.encode_tile(sym9, raw8, q16, pb)
    states = np.frombuffer(tile[:128], "<u4")
    assert np.all(states == 65536)
    lane_words = []
    for lane in range(32):
        w = [raw8[32 * k + lane, j] for k in range(3) if 32 * k + lane < nvec for j in range(8)]
        lane_words.append(np.array(w, np.int16).view(np.uint16))
    expect, counts = [], []
    for p in range(16):
        e, o = lane_words[2 * p], lane_words[2 * p + 1]
        expect += list(e) + list(o[::-1])
        counts.append(len(e) + len(o))
    expect = np.array(expect, np.uint16)
    assert np.array_equal(np.frombuffer(tile[128:160], "<u2"), np.array(counts))
    words = np.frombuffer(tile[160:160 + 2 * len(expect)], "<u2")
    assert np.array_equal(words, expect)
    assert len(tile) == (160 + 2 * len(expect) + 15) // 16 * 16
    assert all(b == 0 for b in tile[160 + 2 * len(expect):])
    rc, s9, r8, st = oracle.decode_tile(tile, nvec, q16, pb)
    assert rc == 0 and np.array_equal(s9, sym9) and np.array_equal(r8, raw8)


@pytest.mark.parametrize("pb", PBS)
def test_rans_lone_symbols_closed_form(pb):
    """Every context holds one symbol with q = M: coding it costs nothing, so the tile is
    exactly the 32 states, all 2^16, and 16 zero region counts."""
    q16 = _tables({127: 1 << pb})
    for nvec in (1, 31, 32, 33, 1000):
        sym9 = np.full((nvec, 9), 127, np.uint8)
        sym9[:, 0] = 0
        tile = oracle.encode_tile(sym9, np.zeros((nvec, 8), np.int16), q16, pb)
        assert tile == np.full(32, 65536, "<u4").tobytes() + bytes(32)
        rc, s9, _, _ = oracle.decode_tile(tile, nvec, q16, pb)
        assert rc == 0 and np.array_equal(s9, sym9)


def _random_tables(nsym_max=40, pb=12):
    counts = np.zeros((16, 256), np.uint64)
    for ctx in range(16):
        k = RNG.integers(1, nsym_max)
        sel = RNG.choice(256, k, replace=False)
        counts[ctx, sel] = RNG.integers(1, 1000, k) ** 2
    return oracle.build_tables16(counts, pb)


def _draw(q16, nvec, pb=12):
    """Vectors drawn from the tables: (coset, f1) from the joint table, then f2..f8 given c."""
    sym9 = np.zeros((nvec, 9), np.uint8)
    joint = np.concatenate([q16[0], q16[8]]).astype(np.float64)
    jt = RNG.choice(512, nvec, p=joint / joint.sum())
    sym9[:, 0], sym9[:, 1] = jt // 256, jt % 256
    for u in range(2, 9):
        for c in (0, 1):
            m = sym9[:, 0] == c
            p = q16[8 * c + u - 1] / float(1 << pb)
            sym9[m, u] = RNG.choice(256, int(m.sum()), p=p)
    raw8 = RNG.integers(-32768, 32768, (nvec, 8)).astype(np.int16)
    return sym9, raw8


@pytest.mark.parametrize("pb", PBS)
def test_rans_roundtrip_random(pb):
    for nvec in (1, 5, 32, 33, 63, 64, 65, 1000, 32 * 64):
        q16 = _random_tables(pb=pb)
        sym9, raw8 = _draw(q16, nvec, pb)
        tile = oracle.encode_tile(sym9, raw8, q16, pb)
        assert len(tile) % 16 == 0
        rc, s9, r8, st = oracle.decode_tile(tile, nvec, q16, pb)
        assert rc == 0
        assert np.array_equal(s9, sym9)
        esc = sym9[:, 1:] == 255
        assert np.array_equal(r8[esc], raw8[esc])
        assert np.all(st == 65536)


def test_rans_totals_are_not_interchangeable():
    """A tile coded with 12-bit totals does not decode under 10-bit ones (or back): the total is
    part of the code, which is why the blob header carries it."""
    for pb, other in ((12, 10), (10, 12)):
        q16 = _random_tables(pb=pb)
        sym9, raw8 = _draw(q16, 2048, pb)
        tile = oracle.encode_tile(sym9, raw8, q16, pb)
        q_other = (q16.astype(np.int64) * (1 << other) // (1 << pb)).astype(np.uint16)
        rc, s9, *_ = oracle.decode_tile(tile, 2048, q_other, other)
        assert rc != 0 or not np.array_equal(s9, sym9)


def test_rans_corruption_detected():
    q16 = _random_tables()
    sym9, raw8 = _draw(q16, 2048)
    tile = bytearray(oracle.encode_tile(sym9, raw8, q16))
    tile[5] ^= 0x10                                                  # flip a bit of lane 1's state
    rc, *_ = oracle.decode_tile(bytes(tile), 2048, q16)
    assert rc != 0
    tile[5] ^= 0x10
    tile[130] ^= 0x01                                                # a region count off by one
    rc, *_ = oracle.decode_tile(bytes(tile), 2048, q16)
    assert rc != 0
    tile[130] ^= 0x01
    rc, *_ = oracle.decode_tile(bytes(tile[:-32]), 2048, q16)       # truncated
    assert rc != 0


@pytest.mark.parametrize("pb", PBS)
def test_rans_size_near_cross_entropy(pb):
    """Coded words carry the symbols' information: 16 * words + the information held by the
    final states (at most 16 bits per lane above 2^16) is the sum of -log2(q/M)."""
    q16 = _random_tables(30, pb)
    nvec = 32 * 256
    sym9, raw8 = _draw(q16, nvec, pb)
    tile = oracle.encode_tile(sym9, raw8, q16, pb)
    ctx = 8 * sym9[:, :1].astype(np.int64) + np.arange(8)[None, :]          # field j: 8c + j - 1
    q = q16[ctx, sym9[:, 1:]].astype(np.float64)                             # j = 1: joint (c, f1)
    info = -np.log2(q / float(1 << pb)).sum() + 16.0 * (sym9[:, 1:] == 255).sum()
    states = np.frombuffer(tile[:128], "<u4").astype(np.float64)
    held = np.log2(states / 65536.0).sum()                          # bits parked in the states
    words_bits = 16.0 * int(np.frombuffer(tile[128:160], "<u2").astype(np.int64).sum())
    # Each encode step stores log2(M / q) bits up to its floor(x / q) rounding (a fraction of a
    # bit over the whole tile here), and each lane's final state holds its last partial word:
    # within one bit per lane.  A wrong frequency or context would be off by kilobits.
    assert abs(words_bits + held - info) <= 32 * 1.0


# ---------------------------------------------------------------------------------------------
# Number formats against library routines (numpy / torch, both round to nearest even).
# ---------------------------------------------------------------------------------------------

def _f32_patterns():
    hi = np.arange(65536, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x3FFF, 0x7FFF, 0x8000, 0x8001, 0xBFFF, 0xFFFF], np.uint32)
    pats = (hi[:, None] | lows[None, :]).ravel()
    rnd = RNG.integers(0, 2 ** 32, 400_000, dtype=np.uint64).astype(np.uint32)
    return np.concatenate([pats, rnd])


def test_conversions_vs_library():
    p = _f32_patterns()
    f = p.view(np.float32)
    fin = np.isfinite(f)
    # BF16: torch's float32 -> bfloat16 rounds to nearest even
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.cvt_f32(p, oracle.BF16)
    assert np.array_equal(got[fin], ref[fin])
    assert np.all((got[~fin] & 0x7F80) == 0x7F80)
    # FP16: numpy's float32 -> float16 rounds to nearest even, overflows to inf, keeps subnormals
    with np.errstate(over="ignore"):
        ref16 = f.astype(np.float16).view(np.uint16)
    got16 = oracle.cvt_f32(p, oracle.FP16)
    assert np.array_equal(got16[fin], ref16[fin])
    # E4M3: torch's float32 -> float8_e4m3fn below the saturation point; at and above
    # 464 (halfway to the next step) the container saturates to 448 by definition.
    got8 = oracle.cvt_f32(p, oracle.E4M3)
    small = fin & (np.abs(f) < 464.0)
    ref8 = torch.from_numpy(f[small].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got8[small], ref8)
    big = fin & (np.abs(f) >= 464.0)
    assert np.all((got8[big] & 0x7F) == 0x7E)
    assert np.array_equal(got8[big] >> 7, (p[big] >> 31).astype(np.uint8))
    # INT8: numpy's rint (nearest, ties to even) clipped to [-128, 127]; ties and the saturation
    # edges are drawn explicitly as well
    ties = np.concatenate([np.arange(-300, 301, dtype=np.float64) + 0.5, [127.49, 127.5, -128.5, -128.51]])
    pi = np.concatenate([p, ties.astype(np.float32).view(np.uint32)])
    fi = pi.view(np.float32)
    got_i = oracle.cvt_f32(pi, oracle.INT8).view(np.int8)
    fin_i = np.isfinite(fi)
    ref_i = np.clip(np.rint(fi[fin_i].astype(np.float64)), -128, 127).astype(np.int8)
    assert np.array_equal(got_i[fin_i], ref_i)
    inf = np.isinf(fi)
    assert np.array_equal(got_i[inf], np.where(fi[inf] > 0, 127, -128).astype(np.int8))
    assert np.all(got_i[np.isnan(fi)] == 0)
    assert list(oracle.cvt_f32(np.array([0.5, 1.5, 2.5, -0.5, -1.5], np.float32).view(np.uint32),
                               oracle.INT8).view(np.int8)) == [0, 2, 2, 0, -2]
    # fp32 rounding of exact doubles: numpy's float64 -> float32 cast
    v = np.concatenate([RNG.normal(0, 1, 100_000) * 10.0 ** RNG.integers(-30, 30, 100_000),
                        (RNG.normal(0, 1, 1000).astype(np.float32).astype(np.float64)
                         * RNG.integers(-65531, 65532, 1000) / 2.0)])
    assert np.array_equal(oracle.round_f32(v), v.astype(np.float32).view(np.uint32))


def test_dtype_decode_vs_numpy_torch():
    allp = np.arange(65536, dtype=np.uint16)
    bf = torch.from_numpy(allp.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = oracle.dtype_to_f64(allp, oracle.BF16)
    assert np.array_equal(np.isnan(got), np.isnan(bf))
    assert np.array_equal(got[~np.isnan(bf)], bf[~np.isnan(bf)])
    h = allp.view(np.float16).astype(np.float64)
    got = oracle.dtype_to_f64(allp, oracle.FP16)
    assert np.array_equal(np.isnan(got), np.isnan(h))
    assert np.array_equal(got[~np.isnan(h)], h[~np.isnan(h)])
    p8 = np.arange(256, dtype=np.uint8)
    e = torch.from_numpy(p8.copy()).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.dtype_to_f64(p8, oracle.E4M3)
    assert np.array_equal(np.isnan(got), np.isnan(e))
    assert np.array_equal(got[~np.isnan(e)], e[~np.isnan(e)])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9
    got = oracle.dtype_to_f64(p8, oracle.INT8)
    assert np.array_equal(got, p8.view(np.int8).astype(np.float64))


# ---------------------------------------------------------------------------------------------
# The encoder end to end.
# ---------------------------------------------------------------------------------------------

def _np_e8(t):
    """Independent nearest point of E8: for each coset, the exact minimum over the 2 integer
    candidates per coordinate subject to even parity (dynamic programming over parity)."""
    best_y = None
    best_d = None
    for half in (0.0, 0.5):
        u = t - half
        a = np.floor(u)
        ca, cb = (u - a) ** 2, (u - a - 1) ** 2
        pa = (a.astype(np.int64) % 2)                                 # parity of choosing a
        # dp over coordinates: cost[parity], choice history kept by backtracking arrays
        INF = np.inf
        cost = np.stack([np.zeros(len(t)), np.full(len(t), INF)], 1)  # before any coordinate
        choices = []
        for i in range(8):
            new = np.full_like(cost, INF)
            ch = np.zeros(cost.shape, np.int8)
            for par in (0, 1):
                for pick, c_, p_ in ((0, ca[:, i], pa[:, i]), (1, cb[:, i], 1 - pa[:, i])):
                    prev = (par - p_) % 2
                    cand = cost[np.arange(len(t)), prev] + c_
                    better = cand < new[:, par]
                    new[better, par] = cand[better]
                    ch[better, par] = pick
            cost = new
            choices.append(ch)
        par = np.zeros(len(t), np.int64)
        z = np.zeros_like(t)
        for i in reversed(range(8)):
            pick = choices[i][np.arange(len(t)), par]
            z[:, i] = a[:, i] + pick
            p_ = np.where(pick == 0, pa[:, i], 1 - pa[:, i])
            par = (par - p_) % 2
        y = z + half
        d = ((t - y) ** 2).sum(1)
        if best_d is None:
            best_y, best_d = y, d
        else:
            m = d < best_d
            best_y[m], best_d[m] = y[m], d[m]
    return best_y


def _values(bits, dtype):
    return oracle.dtype_to_f64(bits, dtype)


def test_end_to_end_fields_vs_independent_quantiser():
    m = W.small()
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
    info = oracle.blob_info(blob)
    w = _values(m.bits, m.dtype)
    rms = np.sqrt((w * w).sum(1) / w.shape[1])
    t = np.clip(w / rms[:, None] / info["scale"], -32764, 32764).reshape(-1, 8)
    y = _np_e8(t)
    c = (y[:, 0] - np.floor(y[:, 0]) == 0.5).astype(np.int16)
    z = (y - 0.5 * c[:, None]).astype(np.int64)
    par = z[:, :7].sum(1) % 2
    expect = np.concatenate([c[:, None], z[:, :7], ((z[:, 7] - par) // 2)[:, None]], 1)
    got = oracle.decode_fields(blob)
    # BF16 inputs repeat values exactly, so some vectors sit at equal distance from two lattice
    # points: there the nearest point is not unique and only the distance is compared.
    y_got = oracle.fields_to_point(got[:, 0], got[:, 1:])
    d_got, d_np = ((t - y_got) ** 2).sum(1), ((t - y) ** 2).sum(1)
    assert np.allclose(d_got, d_np, rtol=0, atol=1e-12)
    same = np.all(y_got == y, axis=1)
    assert same.mean() > 0.99          # the rest are exact ties, where only the distance is fixed
    assert np.array_equal(got[same], expect[same].astype(np.int16))
    # the row-maximum section: each row's largest |2 y| over its real columns
    rm = _rowmax(blob)
    y_rows = np.abs(2 * y_got).reshape(w.shape[0], -1)[:, :w.shape[1]]
    assert np.array_equal(rm, y_rows.max(1).astype(np.int64))
    rows_same = same.reshape(w.shape[0], -1).all(1)
    assert np.array_equal(rm[rows_same], np.abs(2 * y).reshape(w.shape[0], -1)[rows_same].max(1).astype(np.int64))


def _rowmax(blob):
    off = int.from_bytes(blob[80:88], "little")
    rows = int.from_bytes(blob[8:16], "little")
    return np.frombuffer(blob[off:off + 2 * rows], "<u2").astype(np.int64)


def _alpha(blob):
    off = int.from_bytes(blob[56:64], "little")
    rows = int.from_bytes(blob[8:16], "little")
    return np.frombuffer(blob[off:off + 4 * rows], "<f4").astype(np.float64)


def _nearest_f32(x: Fraction) -> np.float32:
    """The float32 nearest to the exact rational x, ties to even (by exact comparison)."""
    f = np.float32(float(x))
    best = None
    for cand in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - x)
        key = (d, int(np.array(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return best[1]


def test_fp8_row_scale_closed_forms():
    """g_r = RNE_fp32(896 / m) with alpha's sign and sigma_r = RNE_fp32(|alpha| m / 896), each
    rounded once from its exact rational value; 0 for an all-zero row."""
    ms = list(range(1, 400)) + [511, 512, 513, 896, 897, 1793, 4095, 4096, 65529] + \
        [int(v) for v in RNG.integers(1, 65530, 2000)]
    alphas = [float(np.float32(v)) for v in list(RNG.normal(0, 0.02, 400)) + [1e-30, -3.5, 448.0, 2.0 ** -126]]
    for m in ms:
        g = oracle.row_gain(1.0, m)
        assert np.float32(g) == np.float32(896) / np.float32(m)       # IEEE float division
        assert np.float32(g) == _nearest_f32(Fraction(896, m))
        assert oracle.row_gain(-1.0, m) == -g
    for a in alphas:
        for m in ms[::37]:
            assert np.float32(oracle.row_sigma(a, m)) == _nearest_f32(abs(Fraction(a)) * m / 896)
    assert oracle.row_gain(0.0, 5) == 0.0 and oracle.row_gain(0.3, 0) == 0.0
    assert oracle.row_sigma(0.3, 0) == 0.0 and oracle.row_sigma(0.0, 7) == 0.0


def test_fp8_rowscaled_payload():
    """The FP8 container with a per-row scale: the payload is E4M3(RNE_fp32(y g_r)) (torch's
    float32 -> float8_e4m3fn conversion, round to nearest even, after the saturating clamp to
    +-448); every nonzero row reaches +-448; sigma_r * payload restores alpha_r * y to E4M3
    precision."""
    m = W.square(rows=96, cols=512)
    for pb in PBS:
        blob = oracle.compress(m.bits, m.dtype, 4.0, prob_bits=pb)
        pay, sigma = oracle.decompress_rowscaled(blob)
        f = oracle.decode_fields(blob)
        y = oracle.fields_to_point(f[:, 0], f[:, 1:]).reshape(96, 512)
        a = _alpha(blob).astype(np.float32)
        rm = _rowmax(blob)
        g = np.array([oracle.row_gain(float(a[r]), int(rm[r])) for r in range(96)], np.float32)
        v = np.clip(y.astype(np.float32) * g[:, None], -448, 448)
        want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(pay, want)
        pv = torch.from_numpy(pay).view(torch.float8_e4m3fn).float().numpy()
        assert np.all(np.abs(pv).max(1) == 448.0)
        assert np.array_equal(sigma, np.array([oracle.row_sigma(float(a[r]), int(rm[r])) for r in range(96)],
                                              np.float32))
        ref = a[:, None].astype(np.float64) * y
        got = sigma[:, None].astype(np.float64) * pv
        big = np.abs(pv) >= 2.0 ** -6                                 # E4M3 normal range
        assert np.all(np.abs(got - ref)[big] <= 2.0 ** -4 * np.abs(ref)[big] * (1 + 1e-6))
        # tile by tile gives the same bytes
        part, _ = oracle.decompress_rowscaled(blob, 1, 3)
        info = oracle.blob_info(blob)
        v0, v1 = 32 * info["S"], 3 * 32 * info["S"]
        sel = np.zeros(96 * 64, bool)
        sel[v0:v1] = True
        sel = np.repeat(sel.reshape(96, 64), 8, axis=1)
        assert np.array_equal(part[sel], pay[sel]) and np.all(part[~sel] == 0)


def test_twelve_bit_totals_code_no_longer_than_ten_bit():
    """At one fixed lattice scale the fields are the same; 12-bit frequencies follow the counts
    more closely, so the coded stream is no longer (a 10-bit table loses up to +0.4% of the bits)."""
    m = W.square(rows=256, cols=1024)
    b12 = oracle.compress(m.bits, m.dtype, 4.0, prob_bits=12)
    s = oracle.blob_info(b12)["scale"]
    b10 = oracle.compress(m.bits, m.dtype, 4.0, scale=s, prob_bits=10)
    b12 = oracle.compress(m.bits, m.dtype, 4.0, scale=s, prob_bits=12)
    assert np.array_equal(oracle.decode_fields(b10), oracle.decode_fields(b12))
    assert oracle.blob_info(b10)["prob_bits"] == 10 and oracle.blob_info(b12)["prob_bits"] == 12
    st = lambda b: len(b) - oracle.blob_info(b)["off_stream"]
    assert st(b12) <= st(b10) <= 1.01 * st(b12)


def test_least_squares_orthogonality():
    """alpha_r minimises ||w_r - alpha y_r||: the residual is orthogonal to y_r (up to the fp32
    rounding of alpha)."""
    m = W.square(rows=64, cols=512)
    blob = oracle.compress(m.bits, m.dtype, 3.0)
    f = oracle.decode_fields(blob)
    y = oracle.fields_to_point(f[:, 0], f[:, 1:]).reshape(64, 512)
    w = _values(m.bits, m.dtype)
    a = _alpha(blob)
    resid = ((w - a[:, None] * y) * y).sum(1)
    scale = (np.abs(w * y)).sum(1)
    assert np.all(np.abs(resid) <= 1e-6 * scale)
    a_ls = (w * y).sum(1) / (y * y).sum(1)
    assert np.array_equal(a.astype(np.float32), a_ls.astype(np.float32))


def test_rms_scale_invariance():
    """Rows are normalised by their RMS before quantisation: scaling rows by powers of two
    leaves every field and the shared scale unchanged and scales alpha_r exactly."""
    m = W.small(rows=64, cols=256)
    w = _values(m.bits, m.dtype)
    k = RNG.integers(-6, 7, 64)
    w2 = w * (2.0 ** k)[:, None]
    bits2 = W.to_bf16_bits(w2)
    assert np.array_equal(_values(bits2, m.dtype), w2)
    b1 = oracle.compress(m.bits, m.dtype, 3.5)
    b2 = oracle.compress(bits2, m.dtype, 3.5)
    assert oracle.blob_info(b1)["scale"] == oracle.blob_info(b2)["scale"]
    assert np.array_equal(oracle.decode_fields(b1), oracle.decode_fields(b2))
    assert np.array_equal(_alpha(b2), _alpha(b1) * 2.0 ** k)


def test_constant_rows_exact():
    """A row of one repeated value quantises to a constant lattice vector m*1 (the sum 8m is
    always even), so alpha = c/m and the reconstruction rounds back to c exactly."""
    # (large enough that the table and row-scale bytes leave room for nonzero fields)
    c = W.to_bf16_bits(RNG.normal(0, 0.05, (64, 1)) * np.ones((1, 1024)))
    c[3] = W.to_bf16_bits(np.zeros((1, 1024)))                       # an all-zero row: alpha = 0
    blob = oracle.compress(c, oracle.BF16, 4.0)
    f = oracle.decode_fields(blob)
    assert np.all(f[:, 1] != 0) or np.all(f[f[:, 1] == 0, 1:] == 0)
    assert np.array_equal(oracle.decompress(blob), c)


def test_high_rate_distortion_closed_form():
    """At fine spacing the E8 quantiser's mean squared error per coordinate is G(E8) s^2 with
    G(E8) = 929/12960 (unit-covolume E8), so the relative L2 error of an RMS-normalised row is
    about sqrt(G) s = 0.2677 s; least squares can only lower it slightly."""
    m = W.sweep(6.0, rows=128, cols=2048)
    for target in (3.5, 6.0):
        blob = oracle.compress(m.bits, m.dtype, target)
        s = oracle.blob_info(blob)["scale"]
        w = _values(m.bits, m.dtype)
        out = oracle.decompress(blob, oracle.F32).view(np.float32).astype(np.float64)
        rel = np.linalg.norm(out - w) / np.linalg.norm(w)
        assert 0.85 * 0.26773 * s <= rel <= 1.02 * 0.26773 * s, (target, s, rel)


def test_shannon_bound():
    """No code beats the Gaussian rate-distortion bound: rel-L2 >= 2^-R for R bits/element."""
    m = W.sweep(2.0, rows=64, cols=2048)
    w = _values(m.bits, m.dtype)
    for target in (0.5, 2.0, 3.5, 6.0):
        blob = oracle.compress(m.bits, m.dtype, target)
        out = oracle.decompress(blob, oracle.F32).view(np.float32).astype(np.float64)
        rel = np.linalg.norm(out - w) / np.linalg.norm(w)
        assert rel >= 2.0 ** -oracle.actual_bpp(blob)


def test_actual_bpp_definition():
    m = W.small(rows=100, cols=200)
    blob = oracle.compress(m.bits, m.dtype, 3.5)
    assert oracle.actual_bpp(blob) == 8.0 * len(blob) / (100 * 200)
    assert int.from_bytes(blob[40:48], "little") == len(blob)


def test_estimate_full_sample_vs_actual():
    """With every row sampled the estimate sees the final tables: it must agree with the real
    size to 0.5% plus 4 bytes per lane per tile (the information parked in the final states
    and the tile padding)."""
    for m in (W.small(), W.square(rows=512, cols=1024), W.sweep(2.0, rows=256, cols=2048)):
        blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
        info = oracle.blob_info(blob)
        est = oracle.estimate_bpp(m.bits, m.dtype, info["scale"], info["S"], True)
        n = m.bits.size
        est_bytes, act = est * n / 8.0, float(len(blob))
        assert abs(est_bytes - act) <= 0.005 * act + 4 * 32 * info["n_tiles"], (est_bytes, act)


def test_estimate_sampled_vs_actual():
    """The sampled estimate (256 of the rows) meets the target and lands within 3% of it."""
    for m in (W.square(rows=1024, cols=2048), W.sweep(3.5, rows=1024, cols=1376)):
        blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
        b = oracle.actual_bpp(blob)
        assert abs(b - m.target_bpp) <= 0.03 * m.target_bpp, b


def test_target_range():
    m = W.small(rows=8, cols=16)
    for bad in (0.0009, 11.0001, float("nan"), float("inf"), -1.0):
        with pytest.raises(ValueError):
            oracle.compress(m.bits, m.dtype, bad)
    for ok in (0.001, 11.0):
        blob = oracle.compress(m.bits, m.dtype, ok)
        assert oracle.decompress(blob).shape == (8, 16)


@pytest.mark.parametrize("shape", [(1, 1), (1, 8), (3, 13), (7, 9), (33, 7), (5, 1000)])
def test_ragged_shapes_roundtrip(shape):
    g = np.random.Generator(np.random.PCG64(shape[0] * 1000 + shape[1]))
    bits = W.to_bf16_bits(g.normal(0, 0.02, shape))
    blob = oracle.compress(bits, oracle.BF16, 4.0)
    out = oracle.decompress(blob)
    assert out.shape == shape
    f = oracle.decode_fields(blob)
    y = oracle.fields_to_point(f[:, 0], f[:, 1:])
    assert y.shape[0] == shape[0] * ((shape[1] + 7) // 8)


def test_int8_container_round_trip():
    """The integer container ([abstract]: INT8 among the weight containers): an INT8 input is read
    as exact integers and restored as INT8, each element the fp32 reconstruction rounded to the
    nearest integer (ties to even) and saturated -- numpy's rint and clip of the FP32 decode."""
    m = W.int8(rows=64, cols=256)
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
    assert oracle.blob_info(blob)["dtype"] == oracle.INT8
    o8 = oracle.decompress(blob)
    o32 = oracle.decompress(blob, oracle.F32).view(np.float32).astype(np.float64)
    assert o8.dtype == np.uint8
    assert np.array_equal(o8.view(np.int8), np.clip(np.rint(o32), -128, 127).astype(np.int8))
    x = m.bits.view(np.int8).astype(np.float64)
    assert np.linalg.norm(o8.view(np.int8) - x) / np.linalg.norm(x) < 0.3


# ---------------------------------------------------------------------------------------------
# Per-row rate-distortion refinement ("Rate selection and refinement": optional, off by default).
# ---------------------------------------------------------------------------------------------

def _two_group_matrix(rows=64, cols=512, ratio=100.0, seed=11):
    """Rows of N(0, 1) and rows of N(0, 1/ratio^2), interleaved."""
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal((rows, cols))
    x[1::2] /= ratio
    return W.Matrix(W.to_bf16_bits(x * 0.02), W.BF16, 4.0), x


def test_rd_refinement_off_is_the_default():
    m = W.square(rows=64, cols=512)
    assert oracle.compress(m.bits, m.dtype, 4.0, rd_refine=False) == oracle.compress(m.bits, m.dtype, 4.0)


def test_rd_refinement_gives_loud_rows_finer_resolution():
    """The squared error a row can save per coded bit grows with its RMS^2, so under one budget
    the loud rows must get the finer resolutions.  A row's resolution is visible in its stored
    scale: alpha_r ~ rms_r * s_r, so alpha_r / rms_r compares s_r across rows."""
    m, _ = _two_group_matrix()
    blob = oracle.compress(m.bits, m.dtype, 4.0, rd_refine=True)
    x = oracle.dtype_to_f64(m.bits, m.dtype)
    rms = np.sqrt((x ** 2).mean(axis=1))
    off = int.from_bytes(blob[56:64], "little")
    alpha = np.frombuffer(blob[off:off + 4 * m.shape[0]], "<f4").astype(np.float64)
    res = alpha / rms
    assert res[0::2].max() < res[1::2].min()          # every loud row finer than every quiet row
    base = oracle.compress(m.bits, m.dtype, 4.0)
    off_b = int.from_bytes(base[56:64], "little")
    ab = np.frombuffer(base[off_b:off_b + 4 * m.shape[0]], "<f4").astype(np.float64) / rms
    assert np.ptp(np.log2(ab)) < 0.1                   # without refinement: one resolution
    assert np.ptp(np.log2(res)) > 1.0                  # with it: at least two, a factor 2 apart


def test_rd_refinement_meets_budget_and_lowers_error():
    """At the same target the refined blob stays within the rate the plain search reaches (the
    budget is the target, checked with the same metadata count) and has lower squared error on
    a matrix whose row scales spread 10x."""
    m = W.square(rows=256, cols=1024)
    ref = oracle.dtype_to_f64(m.bits, m.dtype)
    for target in (2.0, 4.0, 6.0):
        plain = oracle.compress(m.bits, m.dtype, target)
        rd = oracle.compress(m.bits, m.dtype, target, rd_refine=True)
        bpp = lambda b: 8.0 * len(b) / m.bits.size
        assert bpp(rd) <= target + 0.05 and abs(bpp(rd) - bpp(plain)) < 0.1
        err = lambda b: np.linalg.norm(oracle.dtype_to_f64(oracle.decompress(b), m.dtype) - ref)
        assert err(rd) < 0.95 * err(plain)
        # the decode format is unchanged: fields and reconstruction decode as any blob does
        assert oracle.decode_fields(rd).shape == (m.bits.size // 8, 9)

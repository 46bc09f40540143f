"""Pins for the oracle's codec, checked against what the ZipFusion summary
("Run AI Faster With Lossless Compressed Memory", 'Twelve Bits and One
Addition') and plain arithmetic fix:

* lossless: every bit pattern survives the round trip;
* an eligible block costs exactly 12 bits per value (75% of BF16);
* the offset is 4 bits: exponent spread 15 is compressed, 16 falls back raw;
* the value is rebuilt from base + offset (one integer addition);
* hand-derived payloads for specially built blocks (closed forms of the
  documented layout).
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def mk(s, e, m):
    """bf16 bit pattern from sign, 8-bit exponent field and 7-bit mantissa."""
    return ((np.asarray(s, np.uint32) << 15) | (np.asarray(e, np.uint32) << 7) | np.asarray(m, np.uint32)).astype(np.uint16)


def test_page_size_figures():
    facts = json.load(open(GOLD))["facts"]
    # an eligible 64-value block: 64 values x 12 bits = 96 bytes = 6 units of 16 B
    n = 64
    elig_bytes = oracle.lib().zfo_block_bytes(n, 1)
    raw_bytes = oracle.lib().zfo_block_bytes(n, 0)
    assert elig_bytes * 8 == n * facts["eligible_bits_per_value"]
    assert elig_bytes / raw_bytes == facts["eligible_fraction_of_bf16"]
    assert facts["offset_bits"] + 7 + 1 == facts["eligible_bits_per_value"]  # offset + mantissa + sign
    c = oracle.compress(np.full(64, 0x3F80, np.uint16))
    assert c.payload.size == 96 and list(c.offs) == [0, 6]


def test_roundtrip_every_bf16_pattern():
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(7)
    for arr in (allv, rng.permutation(allv), allv.reshape(-1, 64).T.copy().reshape(-1)):
        c = oracle.compress(arr)
        assert np.array_equal(oracle.decompress(c), arr)


def test_threshold_every_exponent_pair():
    """All 256x256 (emin <= emax) pairs: spread <= 15 compressed, else raw."""
    rng = np.random.default_rng(11)
    pairs = [(lo, hi) for lo in range(256) for hi in range(lo, 256)]
    lo = np.array([p[0] for p in pairs])
    hi = np.array([p[1] for p in pairs])
    nb = lo.size
    e = lo[:, None] + (rng.random((nb, 64)) * (hi - lo + 1)[:, None]).astype(np.int64)
    e = np.minimum(e, hi[:, None])
    # pin the extremes at seeded positions
    p0 = rng.integers(0, 64, nb)
    p1 = (p0 + 1 + rng.integers(0, 63, nb)) % 64
    e[np.arange(nb), p0] = lo
    e[np.arange(nb), p1] = hi
    s = rng.integers(0, 2, (nb, 64))
    m = rng.integers(0, 128, (nb, 64))
    vals = mk(s, e, m).reshape(-1)
    c = oracle.compress(vals)
    expect = (hi - lo) <= 15
    assert np.array_equal(c.eligible(), expect)
    assert np.array_equal(c.base, lo.astype(np.uint8))
    sizes = np.diff(c.offs.astype(np.int64))
    assert np.array_equal(sizes, np.where(expect, 6, 8))
    assert np.array_equal(oracle.decompress(c), vals)


def test_size_closed_form_and_offsets():
    rng = np.random.default_rng(3)
    vals = rng.integers(0, 1 << 16, size=64 * 5000).astype(np.uint16)
    # make ~half the blocks narrow so both kinds occur
    narrow = rng.random(5000) < 0.5
    v = vals.reshape(-1, 64)
    v[narrow] = mk(rng.integers(0, 2, (narrow.sum(), 64)), 120 + rng.integers(0, 16, (narrow.sum(), 64)),
                   rng.integers(0, 128, (narrow.sum(), 64)))
    c = oracle.compress(vals)
    el = c.eligible()
    assert np.all(el[narrow])
    n_el = int(el.sum())
    n_raw = el.size - n_el
    assert c.units == 6 * n_el + 8 * n_raw
    assert c.offs[0] == 0
    assert np.array_equal(np.diff(c.offs.astype(np.int64)), np.where(el, 6, 8))
    # unused high bits of the last mask word are zero
    c2 = oracle.compress(np.full(64 * 33, 0x3F80, np.uint16))
    assert c2.elig.size == 2 and c2.elig[0] == 0xFFFFFFFF and c2.elig[1] == 1


def test_bruteforce_two_value_blocks():
    """Block size 2: every (exponent, exponent) pair x every sign pair, with
    mantissas 0, 0x7F and seeded ones: round trip and threshold."""
    rng = np.random.default_rng(5)
    e0, e1 = np.meshgrid(np.arange(256), np.arange(256), indexing="ij")
    e0 = e0.reshape(-1)
    e1 = e1.reshape(-1)
    for s0 in (0, 1):
        for s1 in (0, 1):
            for mm in ("zero", "full", "rand"):
                if mm == "zero":
                    m0 = m1 = np.zeros_like(e0)
                elif mm == "full":
                    m0 = m1 = np.full_like(e0, 0x7F)
                else:
                    m0 = rng.integers(0, 128, e0.size)
                    m1 = rng.integers(0, 128, e0.size)
                vals = np.stack([mk(s0, e0, m0), mk(s1, e1, m1)], axis=1).reshape(-1)
                payload, offs, base, elig = oracle.compress_general(vals, 2)
                expect = np.abs(e0 - e1) <= 15
                assert np.array_equal(elig.astype(bool), expect)
                assert np.array_equal(base, np.minimum(e0, e1).astype(np.uint8))
                assert np.array_equal(np.diff(offs), np.where(expect, 3, 4))
                assert np.array_equal(oracle.decompress_general(payload, offs, base, elig, 2), vals)


def test_bruteforce_four_value_blocks_window():
    """Block size 4: every exponent 4-tuple inside a 20-wide window."""
    rng = np.random.default_rng(9)
    for lo in (0, 100, 236):
        g = np.stack(np.meshgrid(*[np.arange(20)] * 4, indexing="ij"), -1).reshape(-1, 4) + lo
        s = rng.integers(0, 2, g.shape)
        m = rng.integers(0, 128, g.shape)
        vals = mk(s, g, m).reshape(-1)
        payload, offs, base, elig = oracle.compress_general(vals, 4)
        expect = (g.max(1) - g.min(1)) <= 15
        assert np.array_equal(elig.astype(bool), expect)
        assert np.array_equal(base, g.min(1).astype(np.uint8))
        assert np.array_equal(oracle.decompress_general(payload, offs, base, elig, 4), vals)


def test_decode_is_base_plus_offset():
    """Rebuild identity over every (base, offset, sign, mantissa) with
    base + offset <= 255: a block whose exponents are exactly base + off
    decodes to sign | (base + off) << 7 | mantissa, and its stored nibbles are
    the offsets."""
    rng = np.random.default_rng(13)
    for base in range(256):
        offs = np.arange(16)
        offs = offs[base + offs <= 255]
        for s in (0, 1):
            # 64 values: exponent base + off (cycling), one value pinned at base
            off = np.resize(offs, 64)
            off[0] = 0
            m = rng.integers(0, 128, 64)
            vals = mk(s, base + off, m)
            c = oracle.compress(vals)
            assert c.eligible()[0] and c.base[0] == base
            nib = c.payload[64:96]
            got_off = np.concatenate([nib & 0xF, nib >> 4])
            assert np.array_equal(got_off, off)
            assert np.array_equal(oracle.decompress(c), vals)


def test_hand_derived_payloads():
    """Closed forms of the documented layout for specially built blocks:
    sign/mantissa byte j = (mantissa_j << 1) | sign_(j^1); nibble byte k =
    offset_k | offset_(k+32) << 4; raw = sign/mantissa plane then exponent plane."""
    # 64 x 1.0: base 127, all offsets 0, all mantissas and signs 0
    c = oracle.compress(np.full(64, 0x3F80, np.uint16))
    assert c.base[0] == 127 and bytes(c.payload) == bytes(96)
    # 64 x -1.0: each byte carries its partner's sign bit
    c = oracle.compress(np.full(64, 0xBF80, np.uint16))
    assert bytes(c.payload) == bytes([1] * 64 + [0] * 32)
    # alternating 1.0, -2.0: base 127, odd values offset 1, even bytes hold the
    # odd partner's sign
    v = np.array([0x3F80, 0xC000] * 32, np.uint16)
    c = oracle.compress(v)
    assert c.base[0] == 127
    assert bytes(c.payload) == bytes([1, 0] * 32 + [0x00, 0x11] * 16)
    # exponent 120 + j%16 (spread 15), mantissa j, positive
    j = np.arange(64)
    v = mk(0, 120 + j % 16, j)
    c = oracle.compress(v)
    assert c.eligible()[0] and c.base[0] == 120
    assert bytes(c.payload) == bytes([2 * x for x in range(64)] + [0x11 * (k % 16) for k in range(32)])
    # spread 16: raw, two byte planes: the same sign/mantissa bytes as an
    # eligible block (value j here: mantissa j, sign 0), then each value's
    # 8-bit exponent field (120 + j%16, and 136 for value 5)
    v2 = v.copy()
    v2[5] = mk(0, 136, 5)
    c = oracle.compress(v2)
    assert not c.eligible()[0]
    exps = [120 + x % 16 for x in range(64)]
    exps[5] = 136
    assert bytes(c.payload) == bytes([2 * x for x in range(64)] + exps)
    # a raw block with negative values: each sign/mantissa byte carries its
    # partner's sign; exponents 0 (zero) and 255 (Inf/NaN) stay whole
    v3 = mk(np.arange(64) % 2, np.where(np.arange(64) < 32, 0, 255), 3)
    c = oracle.compress(v3)
    assert not c.eligible()[0]
    assert bytes(c.payload) == bytes([6 | (1 - x % 2) for x in range(64)] + [0] * 32 + [255] * 32)
    assert np.array_equal(oracle.decompress(c), v3)
    # three blocks: eligible, raw, eligible
    c = oracle.compress(np.concatenate([np.full(64, 0x3F80, np.uint16), v2, np.full(64, 0x3F80, np.uint16)]))
    assert list(c.offs) == [0, 6, 14, 20]


def test_special_values_are_plain_exponents():
    """Zeros, subnormals, Inf and NaN use their raw exponent field."""
    zeros = np.zeros(64, np.uint16)
    c = oracle.compress(zeros)
    assert c.eligible()[0] and c.base[0] == 0
    sub = mk(np.arange(64) % 2, 0, np.arange(64))            # +-subnormals, exponent 0
    c = oracle.compress(sub)
    assert c.eligible()[0] and c.base[0] == 0
    naninf = mk(np.arange(64) % 2, 255, np.arange(64) % 3)    # +-Inf and NaNs
    c = oracle.compress(naninf)
    assert c.eligible()[0] and c.base[0] == 255
    mix = np.full(64, 0x3F80, np.uint16)
    mix[17] = 0                                              # exact zero next to 1.0
    c = oracle.compress(mix)
    assert not c.eligible()[0]
    for arr in (zeros, sub, naninf, mix):
        assert np.array_equal(oracle.decompress(oracle.compress(arr)), arr)


def test_decompress_block_range():
    rng = np.random.default_rng(17)
    vals = rng.integers(0, 1 << 16, 64 * 100).astype(np.uint16)
    vals[: 64 * 50] = mk(0, 127, rng.integers(0, 128, 64 * 50))
    c = oracle.compress(vals)
    assert np.array_equal(oracle.decompress(c, 37, 81), vals[64 * 37: 64 * 81])


@pytest.mark.parametrize("n", [2, 4, 64])
def test_general_matches_canonical(n):
    """The block-size-64 general form and the canonical form agree."""
    rng = np.random.default_rng(19)
    vals = mk(rng.integers(0, 2, 64 * 40), 110 + rng.integers(0, 18, 64 * 40), rng.integers(0, 128, 64 * 40))
    payload, offs, base, elig = oracle.compress_general(vals, n)
    assert np.array_equal(oracle.decompress_general(payload, offs, base, elig, n), vals)
    if n == 64:
        c = oracle.compress(vals)
        assert np.array_equal(c.offs.astype(np.int64) * 16, offs)
        assert np.array_equal(c.payload, payload)
        assert np.array_equal(c.eligible(), elig.astype(bool))

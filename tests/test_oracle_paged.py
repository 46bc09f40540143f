"""Pins of the oracle's paged form (reading R9): one extent per (page, kv head)
chunk = 48-byte header + its blocks.  Checked against the flat canonical form
(pinned in test_oracle_codec.py): the same block bytes, bases and eligibility
bits, and a round trip."""
import numpy as np

import oracle
import zfsynth


def pool(seed, n_chunks, inelig):
    case = zfsynth.make_case(f"paged-{seed}", B=1, Hq=2, Hkv=1, ctx=16 * n_chunks, sigma=0.7, inelig=inelig,
                             seed=seed)
    return case.k_pool.reshape(-1)


def test_paged_equals_flat_blocks():
    v = pool(31, 12, 0.2)
    flat = oracle.compress(v)
    data, tab = oracle.compress_paged(v)
    nc = v.size // 2048
    assert tab.shape == (nc, 2)
    assert int(tab[-1, 0] + tab[-1, 1]) * 16 == data.size == flat.units * 16 + 48 * nc
    el = flat.eligible()
    for c in range(nc):
        start, ext = int(tab[c, 0]) * 16, int(tab[c, 1]) * 16
        hdr = data[start:start + 48]
        assert np.array_equal(hdr[:32], flat.base[32 * c:32 * c + 32])
        assert int(hdr[32:36].view(np.uint32)[0]) == int(flat.elig[c])
        assert not hdr[36:].any()
        f0, f1 = int(flat.offs[32 * c]) * 16, int(flat.offs[32 * c + 32]) * 16
        assert ext == 48 + f1 - f0
        assert np.array_equal(data[start + 48:start + ext], flat.payload[f0:f1])
        assert ext == 48 + sum(96 if e else 128 for e in el[32 * c:32 * c + 32])
    # chunks laid end to end in order
    assert np.array_equal(tab[1:, 0], tab[:-1, 0] + tab[:-1, 1])


def test_round_trip_and_partial_chunks():
    v = pool(32, 5, 0.5)
    data, tab = oracle.compress_paged(v)
    assert np.array_equal(oracle.decompress_paged(data, tab), v)
    c0 = v[:2048]
    for n in (0, 1, 2, 17, 31, 32):
        part = oracle.pack_chunk(c0, n)
        full = oracle.pack_chunk(c0, 32)
        # a partial chunk is the full chunk's prefix, with a header that only
        # names the blocks written so far
        assert np.array_equal(part[48:], full[48:part.size])
        mask = int(part[32:36].view(np.uint32)[0])
        assert mask == int(full[32:36].view(np.uint32)[0]) & ((1 << n) - 1 if n < 32 else 0xFFFFFFFF)
        assert np.array_equal(part[:n], full[:n]) and not part[n:32].any()
        out = oracle.decompress_paged(part, np.array([[0, part.size // 16]], np.uint32), n)
        assert np.array_equal(out[:64 * n], c0[:64 * n])

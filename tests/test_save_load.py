"""save()/load() of compressed buffers (host logic, no GPU): a buffer in the
flat or the paged form is written with its header and read back byte for
byte; damaged files are refused.  The buffers are filled with the oracle's
encoding of seeded values, held in host tensors."""
import os
import struct

import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_build")


def values(n_chunks, seed):
    case = zfsynth.make_case(f"io-{seed}", B=1, Hq=2, Hkv=1, ctx=16 * n_chunks, sigma=0.7, inelig=0.2, seed=seed)
    return case.k_pool.reshape(-1)


def flat_buffer(v):
    ref = oracle.compress(v)
    z = zf.CompressedKV.empty(v.size, "cpu")
    nb = ref.n_blocks
    z.offs.copy_(torch.from_numpy(ref.offs.view(np.int32)))
    z.base[:nb].copy_(torch.from_numpy(ref.base))
    z.elig[: ref.elig.size].copy_(torch.from_numpy(ref.elig.view(np.int32)))
    z.payload.zero_()
    z.payload[: ref.units * 16].copy_(torch.from_numpy(ref.payload[: ref.units * 16]))
    return z, ref


def path(name):
    os.makedirs(OUT, exist_ok=True)
    return os.path.join(OUT, name)


def test_flat_round_trip():
    v = values(5, 61)
    z, ref = flat_buffer(v)
    p = path("flat.zf")
    zf.save(z, p)
    nb = ref.n_blocks
    assert os.path.getsize(p) == 32 + 4 * (nb + 1) + nb + 4 * ref.elig.size + ref.units * 16
    y = zf.load(p, "cpu")
    assert isinstance(y, zf.CompressedKV) and y.n_values == v.size
    assert np.array_equal(y.offs.numpy().view(np.uint32), ref.offs)
    assert np.array_equal(y.base[:nb].numpy(), ref.base)
    assert np.array_equal(y.elig[: ref.elig.size].numpy().view(np.uint32), ref.elig)
    assert np.array_equal(y.payload[: ref.units * 16].numpy(), ref.payload[: ref.units * 16])
    assert y.payload.numel() >= 2 * v.size      # full capacity for a later compress


def test_paged_round_trip():
    v = values(6, 62)
    data, tab = oracle.compress_paged(v)
    z = zf.PagedKV.empty(tab.shape[0], "cpu")
    z.data[: data.size].copy_(torch.from_numpy(data))
    z.chunk_tab[: tab.shape[0]].copy_(torch.from_numpy(tab.view(np.int32)))
    p = path("paged.zf")
    zf.save(z, p)
    y = zf.load(p, "cpu")
    assert isinstance(y, zf.PagedKV) and y.num_chunks == tab.shape[0]
    assert np.array_equal(y.chunk_tab[: tab.shape[0]].numpy().view(np.uint32), tab)
    assert np.array_equal(y.data[: data.size].numpy(), data)
    assert np.array_equal(oracle.decompress_paged(y.data[: data.size].numpy(), tab), v)


def test_damaged_files_are_refused():
    z, _ = flat_buffer(values(2, 63))
    p = path("bad.zf")
    zf.save(z, p)
    good = open(p, "rb").read()
    cases = {
        "magic": b"XX01" + good[4:],
        "block size": good[:4] + struct.pack("<I", 32) + good[8:],
        "truncated": good[:-1],
        "trailing": good + bytes(1),
    }
    # the offset table's last entry no longer matches the payload units
    last = 32 + 4 * z.n_blocks
    cases["offset total"] = good[:last] + struct.pack("<I", z.units() + 1) + good[last + 4:]
    for what, blob in cases.items():
        with open(p, "wb") as f:
            f.write(blob)
        with pytest.raises(ValueError):
            zf.load(p, "cpu")
    with pytest.raises(TypeError):
        zf.save(object(), p)

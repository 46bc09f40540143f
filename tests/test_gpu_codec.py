"""GPU codec parity: compressed bytes (offset table, bases, eligibility words,
payload up to the total) and decompressed values bit-exact to the oracle."""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth
from gpu_util import dev_bf16, host_u16, host_u32

pytestmark = pytest.mark.gpu


def check_codec(vals: np.ndarray):
    vals = np.ascontiguousarray(vals, dtype=np.uint16).reshape(-1)
    ref = oracle.compress(vals)
    x = dev_bf16(vals)
    z = zf.compress(x)
    torch.cuda.synchronize()
    nb = ref.n_blocks
    assert z.units() == ref.units
    assert np.array_equal(host_u32(z.offs), ref.offs)
    assert np.array_equal(z.base[:nb].cpu().numpy(), ref.base)
    assert np.array_equal(host_u32(z.elig)[: ref.elig.size], ref.elig)
    assert np.array_equal(z.payload[: ref.units * 16].cpu().numpy(), ref.payload)
    out = zf.decompress(z)
    assert np.array_equal(host_u16(out), vals)
    assert zf.validate(z) == 0
    return ref


def test_every_bf16_pattern():
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    check_codec(allv)
    check_codec(np.random.default_rng(1).permutation(allv))


def test_exponent_pair_threshold():
    rng = np.random.default_rng(2)
    lo, hi = np.triu_indices(256)
    nb = lo.size
    e = np.minimum(lo[:, None] + (rng.random((nb, 64)) * (hi - lo + 1)[:, None]).astype(np.int64), hi[:, None])
    e[:, 0] = lo
    e[:, 63] = hi
    vals = ((rng.integers(0, 2, (nb, 64)) << 15) | (e << 7) | rng.integers(0, 128, (nb, 64))).astype(np.uint16)
    ref = check_codec(vals)
    assert np.array_equal(ref.eligible(), (hi - lo) <= 15)


@pytest.mark.parametrize("n_blocks", [1, 31, 32, 33, 255, 256, 257, 256 * 9 + 37, 4096 * 3 + 1])
def test_ragged_lengths(n_blocks):
    rng = np.random.default_rng(n_blocks)
    raw = rng.integers(0, 1 << 16, 64 * n_blocks).astype(np.uint16)
    narrow = ((rng.integers(0, 2, 64 * n_blocks) << 15) | ((118 + rng.integers(0, 16, 64 * n_blocks)) << 7)
              | rng.integers(0, 128, 64 * n_blocks)).astype(np.uint16)
    pick = np.repeat(rng.random(n_blocks) < 0.7, 64)
    check_codec(np.where(pick, narrow, raw))


# The compress kernel works in tiles of 384 blocks, one persistent CTA per SM
# (148 on a B200) cycling through four shared-memory stages: sizes just
# around one tile, one wave of tiles, and several trips round the stages.
@pytest.mark.parametrize("n_blocks", [383, 384, 385, 384 * 148 - 1, 384 * 148, 384 * 148 + 1,
                                      384 * 148 * 4 + 7, 384 * 148 * 9 + 101])
def test_tile_and_wave_boundaries(n_blocks):
    rng = np.random.default_rng(1000 + n_blocks)
    narrow = ((rng.integers(0, 2, 64 * n_blocks) << 15) | ((100 + rng.integers(0, 16, 64 * n_blocks)) << 7)
              | rng.integers(0, 128, 64 * n_blocks)).astype(np.uint16)
    raw_blocks = np.repeat(rng.random(n_blocks) < 0.1, 64)
    wide = rng.integers(0, 1 << 16, 64 * n_blocks).astype(np.uint16)
    check_codec(np.where(raw_blocks, wide, narrow))


def test_empty_buffer():
    z = zf.CompressedKV.empty(0, "cuda")
    z.offs.fill_(123)
    zf.compress(torch.empty(0, dtype=torch.bfloat16, device="cuda"), out=z)
    assert z.units() == 0
    assert zf.decompress(z).numel() == 0


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_benchmark_pools_scaled(cfg):
    case = zfsynth.config(cfg, scale_ctx=1 / 32 if cfg else 1.0)
    check_codec(case.k_pool)
    check_codec(case.v_pool)


@pytest.mark.parametrize("cfg", [2, 3])
def test_full_size_long_and_ragged_pools(cfg):
    """The long-context and ragged workloads' full K and V pools (about 1 GB
    each): offsets, bases, eligibility words and the payload byte for byte
    equal to the oracle's, and the round trip exact."""
    case = zfsynth.config(cfg)
    for pool in (case.k_pool, case.v_pool):
        check_codec(pool)


def test_full_size_llama_pools():
    case = zfsynth.config(1)
    for pool in (case.k_pool, case.v_pool):
        ref = check_codec(pool)
        assert abs((~ref.eligible()).mean() - 0.05) < 1e-6


def test_decompress_of_oracle_bytes():
    """Decompress buffers written by the oracle (independent of GPU compress)."""
    case = zfsynth.config(3, scale_ctx=1 / 32)
    vals = case.k_pool.reshape(-1)
    ref = oracle.compress(vals)
    nb = ref.n_blocks
    z = zf.CompressedKV.empty(vals.size, "cuda", payload_cap=max(16, ref.payload.size))
    z.payload[: ref.payload.size].copy_(torch.from_numpy(ref.payload))
    z.offs.copy_(torch.from_numpy(ref.offs.view(np.int32)))
    z.base[:nb].copy_(torch.from_numpy(ref.base))
    z.elig.copy_(torch.from_numpy(ref.elig.view(np.int32)))
    assert np.array_equal(host_u16(zf.decompress(z)), vals)
    assert zf.validate(z) == 0


def test_validate_flags_corruption():
    case = zfsynth.config(0)
    z = zf.compress(dev_bf16(case.k_pool))
    torch.cuda.synchronize()
    assert zf.validate(z) == 0
    z.offs[5] += 2            # blocks 4 and 5 get wrong sizes
    assert zf.validate(z) == 2
    z.offs[5] -= 2
    e = z.elig.clone()
    z.elig[0] ^= 1            # block 0: eligibility bit disagrees with its size
    assert zf.validate(z) == 1
    z.elig.copy_(e)
    assert zf.validate(z) == 0


def test_compress_reuses_workspace_and_output():
    rng = np.random.default_rng(4)
    a = zfsynth.config(1, scale_ctx=1 / 64).k_pool.reshape(-1)
    b = rng.integers(0, 1 << 16, a.size).astype(np.uint16)
    z = zf.CompressedKV.empty(a.size, "cuda")
    ws = torch.empty(zf.lib().zf_compress_workspace_size(a.size), dtype=torch.uint8, device="cuda")
    for vals in (a, b, a):
        zf.compress(dev_bf16(vals), out=z, ws=ws)
        assert np.array_equal(host_u16(zf.decompress(z)), vals)
        assert z.units() == oracle.compress(vals).units


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_codec_pool_extremes_scaled(frac):
    k, v = zfsynth.codec_pool(num_pages=256, inelig=frac)
    for pool in (k, v):
        ref = check_codec(pool)
        assert (~ref.eligible()).mean() == frac


def test_codec_pool_full_size_sampled_blocks():
    """The 4 GiB codec workload (K and V pools of 65536 pages, 10% raw
    blocks) compressed on the GPU: sampled blocks byte for byte equal to the
    oracle's encoding, the eligible share exact, and the round trip exact."""
    import zfsynth as zs
    for f, k_np, v_np in zs.codec_pool_sweep(fracs=(0.10,)):
        for arr in (k_np, v_np):
            vals = arr.reshape(-1)
            x = dev_bf16(vals)
            z = zf.compress(x)
            torch.cuda.synchronize()
            nb = vals.size // 64
            offs = z.offs.cpu().numpy().view(np.uint32)
            base = z.base[:nb].cpu().numpy()
            elig = z.elig.cpu().numpy().view(np.uint32)
            el = ((elig[np.arange(nb) // 32] >> (np.arange(nb) % 32)) & 1).astype(bool)
            assert int((~el).sum()) == int(round(f * nb))
            rng = np.random.default_rng(77)
            for i in np.concatenate([[0, nb - 1], rng.integers(0, nb, 62)]):
                ref = oracle.compress(vals[64 * i:64 * i + 64])
                got = z.payload[int(offs[i]) * 16:int(offs[i + 1]) * 16].cpu().numpy()
                assert np.array_equal(got, ref.payload)
                assert base[i] == ref.base[0] and bool(el[i]) == bool(ref.eligible()[0])
            back = zf.decompress(z)
            assert torch.equal(back.view(torch.int16), x.view(torch.int16))
            del x, z, back
            torch.cuda.empty_cache()


def test_decompress_of_exact_size_payload():
    """After shrink() the payload is exactly offs[n_blocks] units long, so the
    last block ends at the capacity: every block, the last raw or eligible
    one included, still decompresses (the capacity guard skips only blocks
    that would pass the end)."""
    for last_raw in (False, True):
        vals = zfsynth.config(0).k_pool.reshape(-1).copy()
        if last_raw:                      # make the final block raw
            vals[-64] = zfsynth.to_bf16_bits(np.array([2.0 ** 20], np.float32))[0]
            vals[-63] = zfsynth.to_bf16_bits(np.array([2.0 ** -20], np.float32))[0]
        z = zf.compress(dev_bf16(vals)).shrink()
        torch.cuda.synchronize()
        assert z.payload.numel() == z.units() * 16
        el = host_u32(z.elig)
        nb = vals.size // 64
        assert bool((el[(nb - 1) // 32] >> ((nb - 1) % 32)) & 1) == (not last_raw)
        assert np.array_equal(host_u16(zf.decompress(z)), vals)
        assert zf.validate(z) == 0

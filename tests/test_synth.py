"""The seeded input generator: determinism, layout, and the exact share of raw
(ineligible) blocks, checked with the oracle's codec."""
import numpy as np
import pytest

import oracle
import zfsynth


def raw_share(pool, used_blocks_mask=None):
    c = oracle.compress(pool.reshape(-1))
    el = c.eligible()
    if used_blocks_mask is not None:
        el = el[used_blocks_mask]
    return 1.0 - el.mean(), c


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-5], np.float32)
    bits = zfsynth.to_bf16_bits(x)
    ref = torch_bits(x)
    assert np.array_equal(bits, ref)


def torch_bits(x):
    import torch
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_rounding_matches_torch_on_random_values():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37
    assert np.array_equal(zfsynth.to_bf16_bits(x), torch_bits(x))


def test_deterministic():
    a = zfsynth.config(1, scale_ctx=1 / 64)
    b = zfsynth.config(1, scale_ctx=1 / 64)
    for f in ("q", "k_pool", "v_pool", "page_table", "seq_lens"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_exact_raw_share(cfg):
    case = zfsynth.config(cfg, scale_ctx=1 / 64 if cfg else 1.0)
    target = case.meta["inelig_target"]
    used = case.meta["used_blocks"]
    for pool, key in ((case.k_pool, "forced_raw_k"), (case.v_pool, "forced_raw_v")):
        c = oracle.compress(pool.reshape(-1))
        n_raw = int((~c.eligible()).sum())
        assert n_raw == case.meta[key] == int(round(target * used))


def test_layout_and_tail_slots():
    case = zfsynth.config(3, scale_ctx=1 / 64)
    assert case.page_table.dtype == np.int32 and case.seq_lens.dtype == np.int32
    assert case.k_pool.shape[1:] == (8, 16, 128)
    # every page is used once, tail slots are zero
    used = []
    for b in range(case.B):
        n = (case.seq_lens[b] + 15) // 16
        used += list(case.page_table[b, :n])
        tail = case.seq_lens[b] - 16 * (n - 1)
        assert np.all(case.k_pool[case.page_table[b, n - 1], :, tail:] == 0)
    assert sorted(used) == list(range(case.num_pages))


def test_config_shapes():
    c1 = zfsynth.config(1, scale_ctx=1 / 16)
    assert (c1.B, c1.Hq, c1.Hkv) == (32, 32, 8) and c1.max_seq_len == 256
    c0 = zfsynth.config(0)
    assert (c0.B, c0.Hq, c0.Hkv, c0.max_seq_len, c0.num_pages) == (2, 4, 1, 512, 64)
    assert np.array_equal(c0.page_table.reshape(-1), np.arange(64))


def test_codec_pool_sweep_exact_shares():
    """The codec sweep injects exactly the asked raw-block share into copies
    of one base draw (checked with the oracle's eligibility rule)."""
    import oracle
    base_k = None
    for f, k, v in zfsynth.codec_pool_sweep(num_pages=64):
        nb = k.size // 64
        for pool in (k, v):
            el = oracle.compress(pool.reshape(-1)).eligible()
            assert int((~el.astype(bool)).sum()) == int(round(f * nb))
        if base_k is None:
            base_k = k
        elif f > 0:
            # only the injected blocks differ from the share-0 draw
            changed = (k.reshape(-1, 64) != base_k.reshape(-1, 64)).any(axis=1)
            assert changed.sum() <= int(round(f * nb))

"""Pins for the oracle's fp64 paged GQA decode attention.

Decode attention is the textbook softmax(q.K^T * scale) V over the tokens of a
sequence (the pages give no formula; they only say decoding reads the cached
K/V at every step).  Pins: a library routine (torch's float64
scaled_dot_product_attention on gathered, head-repeated K/V), brute-force
closed forms for special inputs, and invariants.
"""
import numpy as np
import pytest
import torch

import oracle
import zfsynth


def gathered(case, b):
    """Contiguous K/V [Hkv][L][D] of sequence b, read through the page table."""
    L = int(case.seq_lens[b])
    pages = case.page_table[b, : (L + 15) // 16]
    k = case.k_pool[pages].transpose(1, 0, 2, 3).reshape(case.Hkv, -1, 128)[:, :L]
    v = case.v_pool[pages].transpose(1, 0, 2, 3).reshape(case.Hkv, -1, 128)[:, :L]
    return k, v


def f64(bits):
    return zfsynth.bf16_bits_to_f32(bits).astype(np.float64)


def small_case(seed=0, B=3, Hq=8, Hkv=2, ctx=(37, 16, 70)):
    return zfsynth.make_case("t", B=B, Hq=Hq, Hkv=Hkv, ctx=list(ctx), sigma=0.7, seed=seed, inelig=0.1,
                             k_outlier_channels=2)


@pytest.mark.parametrize("which", ["small", "tiny", "llama-reduced"])
def test_matches_library_sdpa(which):
    """Against torch's float64 scaled_dot_product_attention on the gathered,
    head-repeated K/V: a small ragged case, the tiny workload, and the
    Llama-3.1-8B decode shape with its context cut to 256 tokens."""
    case = {"small": small_case, "tiny": lambda: zfsynth.config(0),
            "llama-reduced": lambda: zfsynth.config(1, scale_ctx=1 / 16)}[which]()
    out, lse, _ = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens,
                                   case.sm_scale)
    g = case.Hq // case.Hkv
    for b in range(case.B):
        k, v = gathered(case, b)
        qt = torch.from_numpy(f64(case.q[b]))[None, :, None, :]
        kt = torch.from_numpy(f64(k)).repeat_interleave(g, 0)[None]
        vt = torch.from_numpy(f64(v)).repeat_interleave(g, 0)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=case.sm_scale)[0, :, 0]
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)
        s = torch.einsum("hd,htd->ht", qt[0, :, 0], kt[0]) * case.sm_scale
        np.testing.assert_allclose(lse[b], torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_weights_sum_to_one_and_zero_past_end():
    case = small_case(seed=1)
    _, _, p = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens,
                               case.sm_scale, want_p=True)
    for b in range(case.B):
        L = case.seq_lens[b]
        np.testing.assert_allclose(p[b, :, :L].sum(-1), 1.0, rtol=0, atol=1e-12)
        assert np.all(p[b, :, L:] == 0) and np.all(p[b, :, :L] >= 0)


def test_constant_v_gives_constant_output():
    case = small_case(seed=2)
    c = zfsynth.to_bf16_bits(np.array([1.375], np.float32))[0]
    v = np.full_like(case.v_pool, c)
    out, _, _ = oracle.attention(case.q, case.k_pool, v, case.page_table, case.seq_lens, case.sm_scale)
    np.testing.assert_allclose(out, 1.375, rtol=1e-14)


def test_single_token_returns_its_value():
    case = small_case(seed=3, ctx=(1, 1, 1))
    out, lse, _ = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens,
                                   case.sm_scale)
    g = case.Hq // case.Hkv
    for b in range(case.B):
        v0 = f64(case.v_pool[case.page_table[b, 0], :, 0])      # [Hkv][D]
        np.testing.assert_array_equal(out[b], np.repeat(v0, g, 0))
        k0 = f64(case.k_pool[case.page_table[b, 0], :, 0])
        s = (f64(case.q[b]) * np.repeat(k0, g, 0)).sum(-1) * case.sm_scale
        np.testing.assert_allclose(lse[b], s, rtol=1e-14)


def test_zero_query_is_mean_of_values():
    case = small_case(seed=4)
    q = np.zeros_like(case.q)
    out, lse, _ = oracle.attention(q, case.k_pool, case.v_pool, case.page_table, case.seq_lens, case.sm_scale)
    g = case.Hq // case.Hkv
    for b in range(case.B):
        _, v = gathered(case, b)
        np.testing.assert_allclose(out[b], np.repeat(f64(v).mean(1), g, 0), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[b], np.log(case.seq_lens[b]), rtol=1e-14)


def test_identical_keys_give_mean():
    case = small_case(seed=5)
    k = np.broadcast_to(case.k_pool[:1, :, :1], case.k_pool.shape).copy()
    out, _, _ = oracle.attention(case.q, k, case.v_pool, case.page_table, case.seq_lens, case.sm_scale)
    g = case.Hq // case.Hkv
    for b in range(case.B):
        _, v = gathered(case, b)
        np.testing.assert_allclose(out[b], np.repeat(f64(v).mean(1), g, 0), rtol=1e-12, atol=1e-13)


def test_page_permutation_invariance():
    case = small_case(seed=6)
    out, lse, _ = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens,
                                   case.sm_scale)
    perm = np.random.default_rng(0).permutation(case.num_pages)
    inv = np.argsort(perm)
    k2 = case.k_pool[perm]
    v2 = case.v_pool[perm]
    table2 = inv[case.page_table].astype(np.int32)
    out2, lse2, _ = oracle.attention(case.q, k2, v2, table2, case.seq_lens, case.sm_scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_gqa_grouping():
    """Query head h reads kv head h // (Hq/Hkv): with Hkv copies of one kv
    head the output equals the MHA result of that head."""
    case = small_case(seed=7, Hq=8, Hkv=2)
    k = case.k_pool.copy()
    v = case.v_pool.copy()
    k[:, 1] = k[:, 0]
    v[:, 1] = v[:, 0]
    out, _, _ = oracle.attention(case.q, k, v, case.page_table, case.seq_lens, case.sm_scale)
    out1, _, _ = oracle.attention(case.q, k[:, :1], v[:, :1], case.page_table, case.seq_lens, case.sm_scale)
    np.testing.assert_array_equal(out, out1)


def test_empty_sequence():
    case = small_case(seed=8)
    lens = case.seq_lens.copy()
    lens[1] = 0
    out, lse, _ = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, lens, case.sm_scale)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(lse[0]))


def test_rejects_bad_page_ids():
    case = small_case(seed=9)
    t = case.page_table.copy()
    t[0, 0] = case.num_pages
    with pytest.raises(ValueError):
        oracle.attention(case.q, case.k_pool, case.v_pool, t, case.seq_lens, case.sm_scale)


def test_compressed_attention_equals_raw():
    case = small_case(seed=10)
    kc = oracle.compress(case.k_pool.reshape(-1))
    vc = oracle.compress(case.v_pool.reshape(-1))
    a = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens, case.sm_scale)
    b = oracle.attention_compressed(case.q, kc, vc, case.num_pages, case.Hkv, case.page_table, case.seq_lens,
                                    case.sm_scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_two_tokens_closed_form():
    """Two tokens with exactly known scores: q = e_0 and keys whose first
    channel is a and b give scores scale*a and scale*b, so the weights are
    1/(1+e^(s1-s0)) and its complement and lse = ln(e^s0 + e^s1)."""
    case = small_case(seed=5, B=1, Hq=1, Hkv=1, ctx=(2,))
    q = np.zeros_like(case.q)
    q[0, 0, 0] = zfsynth.to_bf16_bits(np.array([1.0], np.float32))[0]
    k = np.zeros_like(case.k_pool)
    v = np.zeros_like(case.v_pool)
    pid = case.page_table[0, 0]
    k[pid, 0, 0, 0], k[pid, 0, 1, 0] = zfsynth.to_bf16_bits(np.array([3.0, -1.0], np.float32))
    v[pid, 0, 0, :] = zfsynth.to_bf16_bits(np.full(128, 2.0, np.float32))
    v[pid, 0, 1, :] = zfsynth.to_bf16_bits(np.full(128, -4.0, np.float32))
    scale = 0.5
    out, lse, p = oracle.attention(q, k, v, case.page_table, case.seq_lens, scale, want_p=True)
    s0, s1 = 1.5, -0.5
    p0 = 1.0 / (1.0 + np.exp(s1 - s0))
    np.testing.assert_allclose(p[0, 0, :2], [p0, 1.0 - p0], rtol=1e-14)
    np.testing.assert_allclose(out[0, 0], 2.0 * p0 - 4.0 * (1.0 - p0), rtol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(np.exp(s0) + np.exp(s1)), rtol=1e-14)

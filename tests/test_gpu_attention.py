"""GPU decode-attention parity.

* compressed-cache output and lse bitwise equal to the library's raw-BF16
  kernel (same plan, same reduction order);
* both within max |err| <= 1e-2 * max(1, |ref|) of the fp64 oracle;
* edge cases: empty / one-token / ragged sequences, every GQA group size,
  all-raw and all-eligible caches, page permutation, corrupt page ids.
"""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth
from gpu_util import DeviceCase, assert_attention_close, bf16_to_f64, host_u16, oracle_attention_rows

pytestmark = pytest.mark.gpu


def check_case(case, rows=None, lse_check=True):
    d = DeviceCase(case)
    out_c, lse_c = d.run(compressed=True)
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    oc, orr = host_u16(out_c), host_u16(out_r)
    assert np.array_equal(oc, orr), "compressed and raw outputs differ"
    assert torch.equal(lse_c, lse_r)
    if rows is None:
        ref, ref_lse = oracle_attention_rows(case)
        got, got_lse = oc, lse_c.cpu().numpy()
    else:
        ref, ref_lse = oracle_attention_rows(case, rows)
        got, got_lse = oc[rows], lse_c.cpu().numpy()[rows]
    worst = assert_attention_close(got, ref, case.name)
    if lse_check:
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(got_lse), fin)
        np.testing.assert_allclose(got_lse[fin], ref_lse[fin], rtol=1e-5, atol=1e-3)
    return d, oc, worst


def small(seed, B, Hq, Hkv, ctx, **kw):
    kw.setdefault("sigma", 0.7)
    kw.setdefault("inelig", 0.1)
    return zfsynth.make_case(f"small-{seed}", B=B, Hq=Hq, Hkv=Hkv, ctx=ctx, seed=seed, **kw)


def test_tiny_config_full():
    check_case(zfsynth.config(0))


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (32, 8), (8, 1), (64, 8), (16, 16)])
def test_group_sizes(Hq, Hkv):
    check_case(small(Hq * 100 + Hkv, B=3, Hq=Hq, Hkv=Hkv, ctx=[37, 200, 1]))


def test_ragged_lengths_and_empty_sequences():
    lens = [0, 1, 15, 16, 17, 31, 32, 33, 0, 511, 512, 513, 1000, 4, 0]
    check_case(small(7, B=len(lens), Hq=8, Hkv=2, ctx=lens, k_outlier_channels=3))


def test_all_empty():
    d, oc, _ = check_case(small(8, B=3, Hq=8, Hkv=2, ctx=[0, 0, 0], pool_pages=4))
    assert np.all(oc == 0)


@pytest.mark.parametrize("inelig", [0.0, 1.0])
def test_all_eligible_and_all_raw(inelig):
    check_case(small(9, B=4, Hq=32, Hkv=8, ctx=[300, 77, 512, 129], inelig=inelig))


def test_ragged_config_scaled():
    check_case(zfsynth.config(3, scale_ctx=1 / 16))


def test_llama_config_full_size():
    """Batch 32, 32/8 heads, 4096 tokens: the benchmark's launch."""
    check_case(zfsynth.config(1))


def test_long_context_full_size_every_row():
    """Batch 16, 32/8 heads, 32768 tokens: every output row and lse against
    the fp64 oracle."""
    check_case(zfsynth.config(2))


def test_ragged_config_full_size_every_row():
    """Batch 64 with lengths in [1024, 16384] over a shuffled shared pool:
    every output row against the oracle."""
    check_case(zfsynth.config(3))


def test_extreme_context_full_size_every_row():
    """Batch 4, 131072 tokens each, over 32768 pages of a 65536-page pool:
    every output row against the oracle."""
    check_case(zfsynth.config(4))


def test_constant_values_exact():
    case = small(10, B=3, Hq=8, Hkv=2, ctx=[100, 1, 700])
    c = zfsynth.to_bf16_bits(np.array([-2.625], np.float32))[0]
    case.v_pool[:] = c
    d = DeviceCase(case)
    out, _ = d.run()
    assert np.all(host_u16(out) == c)


def test_page_permutation_bitwise():
    case = small(11, B=4, Hq=32, Hkv=8, ctx=[300, 700, 64, 1000])
    d1, o1, _ = check_case(case)
    perm = np.random.default_rng(0).permutation(case.num_pages)
    inv = np.argsort(perm)
    case2 = zfsynth.Case(case.name, case.q, case.k_pool[perm].copy(), case.v_pool[perm].copy(),
                         inv[case.page_table].astype(np.int32), case.seq_lens, case.B, case.Hq, case.Hkv,
                         case.sm_scale)
    d2 = DeviceCase(case2)
    o2, _ = d2.run()
    assert np.array_equal(host_u16(o2), o1)


def test_split_plan_does_not_change_results_beyond_tolerance():
    """A larger host bound changes the grid (the split points) but not the answer."""
    case = small(12, B=2, Hq=8, Hkv=2, ctx=[33, 20])
    d = DeviceCase(case)
    o1, _ = d.run(max_seq_len=case.max_seq_len)
    d.ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, 8000, "cuda")
    o2, _ = d.run(max_seq_len=8000)
    ref, _, _ = oracle.attention(case.q, case.k_pool, case.v_pool, case.page_table, case.seq_lens, case.sm_scale)
    assert_attention_close(host_u16(o1), ref)
    assert_attention_close(host_u16(o2), ref)


def test_bad_page_id_is_clamped_and_flagged():
    case = small(13, B=2, Hq=8, Hkv=2, ctx=[40, 40])
    case.page_table[1, 1] = case.num_pages + 5
    d = DeviceCase(case)
    out, _ = d.run()
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) & zf.DEVERR_PAGE_ID
    assert np.all(np.isfinite(bf16_to_f64(host_u16(out))))
    zf.clear_device_error(d.ws)
    assert zf.get_device_error(d.ws) == 0


def test_bad_seq_len_is_clamped_and_flagged():
    case = small(14, B=2, Hq=8, Hkv=2, ctx=[40, 40])
    d = DeviceCase(case)
    d.sl[0] = 10_000          # longer than its page-table row (3 pages)
    d.ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, 10_000, "cuda")
    out, _ = d.run(max_seq_len=10_000)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) & zf.DEVERR_SEQ_LEN


def test_repeat_calls_are_deterministic():
    case = zfsynth.config(1, scale_ctx=1 / 8)
    d = DeviceCase(case)
    o1, l1 = d.run()
    o2, l2 = d.run()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_single_long_sequence_one_kv_head():
    """One sequence split across every CTA of the grid (many partial slots)."""
    check_case(small(15, B=1, Hq=4, Hkv=1, ctx=[20000], inelig=0.05))


def test_back_to_back_calls_on_one_stream():
    """Consecutive calls (programmatic dependent launch) see each other's
    results in order: alternating inputs give alternating outputs."""
    c1 = small(16, B=4, Hq=32, Hkv=8, ctx=[300, 1000, 64, 700])
    c2 = small(17, B=4, Hq=32, Hkv=8, ctx=[900, 20, 640, 33])
    d1, d2 = DeviceCase(c1), DeviceCase(c2)
    r1, _ = d1.run()
    r2, _ = d2.run()
    torch.cuda.synchronize()
    ref1, ref2 = host_u16(r1).copy(), host_u16(r2).copy()
    out = torch.empty_like(r1)
    for _ in range(5):
        d1.run(out=out)
        a = host_u16(out).copy()
        d2.run(out=out)
        b = host_u16(out).copy()
        assert np.array_equal(a, ref1) and np.array_equal(b, ref2)


def test_workspace_reused_across_shapes():
    """One zero-filled workspace serves calls of different shapes in any
    order: the split counters sit in a fixed region that no shape's partial
    slots reach, and every call leaves them at zero."""
    rng = np.random.default_rng(5)
    cases = [small(11, B=3, Hq=8, Hkv=2, ctx=[900, 5, 300]),
             small(12, B=20, Hq=32, Hkv=8, ctx=list(rng.integers(1, 2000, size=20))),
             zfsynth.config(1, scale_ctx=1 / 16)]
    devs = [DeviceCase(c) for c in cases]
    size = max(zf.decode_workspace_size(c.B, c.Hq, c.Hkv, c.max_seq_len,
                                        torch.cuda.get_device_properties(0).multi_processor_count)
               for c in cases)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    for d in devs + devs[:1] + devs[::-1]:
        c = d.case
        d.ws = ws
        out_c, lse_c = d.run(compressed=True)
        out_r, lse_r = d.run(compressed=False)
        torch.cuda.synchronize()
        assert zf.get_device_error(ws) == 0
        # counters of every segment are back at zero
        counters = ws[256:256 + 4 * c.B * c.Hkv].cpu().numpy()
        assert not counters.any()
        oc = host_u16(out_c)
        assert np.array_equal(oc, host_u16(out_r))
        ref, _, _ = oracle.attention(c.q, c.k_pool, c.v_pool, c.page_table, c.seq_lens, c.sm_scale)
        assert_attention_close(oc, ref, c.name)


@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffer_entry_equals_device_call(pinned):
    """zf_decode_attention_host (inputs and outputs in host memory) gives the
    device call's out and lse bit for bit, and its workspace starts with the
    decode workspace (device error word read the same way)."""
    case = zfsynth.make_case("host-io", B=5, Hq=16, Hkv=4, ctx=[700, 1, 0, 129, 2048], sigma=0.7, inelig=0.05,
                             k_outlier_channels=3, seed=77)
    d = DeviceCase(case)
    out_d, lse_d = d.run()

    def host(a, dtype):
        t = torch.from_numpy(np.ascontiguousarray(a)).view(dtype)
        return t.pin_memory() if pinned else t.clone()
    q_h = host(case.q, torch.bfloat16)
    pt_h = host(case.page_table, torch.int32)
    sl_h = host(case.seq_lens, torch.int32)
    out_h = torch.full((case.B, case.Hq, 128), 7.0, dtype=torch.bfloat16)
    lse_h = torch.zeros((case.B, case.Hq), dtype=torch.float32)
    if pinned:
        out_h, lse_h = out_h.pin_memory(), lse_h.pin_memory()
    ws = zf.decode_host_workspace(case.B, case.Hq, case.Hkv, case.page_table.shape[1], case.max_seq_len, "cuda")
    for _ in range(2):                                       # the workspace is reusable
        zf.decode_attention_host(q_h, d.kz, d.vz, pt_h, sl_h, case.max_seq_len, num_pages=case.num_pages,
                                 Hkv=case.Hkv, sm_scale=case.sm_scale, out=out_h, lse=lse_h, ws=ws)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))
        assert torch.equal(lse_h, lse_d.cpu())
    assert zf.get_device_error(ws) == 0


def test_maximum_batch_and_segment_count():
    """B = 4096 sequences (the largest batch) x 32 kv heads = 2^17 (sequence,
    kv head) segments, the largest split-counter count: short and empty
    sequences over a shared 256-page pool.  Compressed equals the raw twin
    bit for bit on every row; sampled rows match the oracle."""
    B, Hq, Hkv = 4096, 32, 32
    pool = zfsynth.make_case("max-pool", B=1, Hq=Hq, Hkv=Hkv, ctx=16 * 256, sigma=0.7, inelig=0.05, seed=88)
    rng = np.random.default_rng(89)
    seq_lens = rng.integers(1, 41, size=B).astype(np.int32)
    seq_lens[::7] = 0
    page_table = rng.integers(0, pool.num_pages, size=(B, 3)).astype(np.int32)
    q = zfsynth.to_bf16_bits(rng.standard_normal((B, Hq, 128)).astype(np.float32))
    case = zfsynth.Case("max batch: B=4096 Hq=32 Hkv=32 ctx<=40", q, pool.k_pool, pool.v_pool, page_table,
                        seq_lens, B, Hq, Hkv, pool.sm_scale)
    d = DeviceCase(case)
    out_c, lse_c = d.run()
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert np.array_equal(host_u16(out_c), host_u16(out_r)) and torch.equal(lse_c, lse_r)
    rows = np.array([1, 7, 1000, 2048, 4094])
    ref, ref_lse, _ = oracle.attention(case.q[rows], case.k_pool, case.v_pool, case.page_table[rows],
                                       case.seq_lens[rows], case.sm_scale)
    assert_attention_close(host_u16(out_c)[rows], ref, case.name)
    got_lse = lse_c.cpu().numpy()[rows]
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin) and not fin[1].any()      # row 7 is empty
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], rtol=1e-5, atol=1e-3)
    assert not host_u16(out_c)[rows[1]].any()

"""GPU parity of the paged form (reading R9) and of append-time compression.

* zf_compress_paged: data and chunk table bit for bit equal to the oracle's
  paged form; decompress round trip;
* decode attention over paged pools: bitwise equal to the raw twin, within
  tolerance of the fp64 oracle;
* append-time compression token by token: every chunk (full or filling)
  equals the oracle's chunk of the tokens written so far, full pages end up
  packed, and decode attention over the appended pools equals the raw twin.
"""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth
from gpu_util import DeviceCase, assert_attention_close, dev_bf16, dev_i32, host_u16

pytestmark = pytest.mark.gpu


def tab_host(pk):
    return pk.chunk_tab[: pk.num_chunks].cpu().numpy().view(np.uint32).copy()


@pytest.mark.parametrize("inelig", [0.0, 0.1, 1.0])
def test_compress_paged_bitwise(inelig):
    case = zfsynth.make_case(f"paged-{inelig}", B=3, Hq=8, Hkv=2, ctx=[300, 47, 512], sigma=0.7, inelig=inelig,
                             k_outlier_channels=3, seed=400)
    x = dev_bf16(case.k_pool)
    pk = zf.compress_paged(x)
    torch.cuda.synchronize()
    data_ref, tab_ref = oracle.compress_paged(case.k_pool)
    tab = tab_host(pk)
    assert np.array_equal(tab, tab_ref)
    n = data_ref.size
    assert np.array_equal(pk.data[:n].cpu().numpy(), data_ref)
    back = zf.decompress_paged(pk)
    assert torch.equal(back.view(torch.int16), x.reshape(-1).view(torch.int16))


# Pools of whole chunks around the compress kernel's tile (12 chunks) and wave
# (148 tiles) boundaries: data and chunk table equal to the oracle's.
@pytest.mark.parametrize("n_chunks", [11, 12, 13, 12 * 148 - 1, 12 * 148 + 1, 12 * 148 * 4 + 3])
def test_compress_paged_tile_boundaries(n_chunks):
    rng = np.random.default_rng(2000 + n_chunks)
    n = n_chunks * 2048
    narrow = ((rng.integers(0, 2, n) << 15) | ((110 + rng.integers(0, 16, n)) << 7)
              | rng.integers(0, 128, n)).astype(np.uint16)
    wide = rng.integers(0, 1 << 16, n).astype(np.uint16)
    vals = np.where(np.repeat(rng.random(n // 64) < 0.1, 64), wide, narrow)
    x = dev_bf16(vals)
    pk = zf.compress_paged(x)
    torch.cuda.synchronize()
    data_ref, tab_ref = oracle.compress_paged(vals)
    assert np.array_equal(tab_host(pk), tab_ref)
    assert np.array_equal(pk.data[: data_ref.size].cpu().numpy(), data_ref)
    back = zf.decompress_paged(pk)
    assert torch.equal(back.view(torch.int16), x.reshape(-1).view(torch.int16))


def run_paged(d, pk, pv):
    c = d.case
    lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
    return zf.decode_attention_paged(d.q, pk, pv, d.pt, d.sl, c.max_seq_len, num_pages=c.num_pages, Hkv=c.Hkv,
                                     sm_scale=c.sm_scale, lse=lse, ws=d.ws)


@pytest.mark.parametrize("cfg", [0, 3])
def test_decode_paged_equals_raw(cfg):
    case = zfsynth.config(cfg, scale_ctx=1 / 16 if cfg else 1.0)
    d = DeviceCase(case, compress=False)
    pk, pv = zf.compress_paged(d.k), zf.compress_paged(d.v)
    out_p, lse_p = run_paged(d, pk, pv)
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert np.array_equal(host_u16(out_p), host_u16(out_r))
    assert torch.equal(lse_p, lse_r)
    rows = np.arange(min(case.B, 6))
    ref, _, _ = oracle.attention(case.q[rows], case.k_pool, case.v_pool, case.page_table[rows],
                                 case.seq_lens[rows], case.sm_scale)
    assert_attention_close(host_u16(out_p)[rows], ref, case.name + " (paged)")


def token_values(case, pool, b, t):
    """[Hkv][128] values of token t of sequence b."""
    pid = int(case.page_table[b, t // 16])
    return pool[pid, :, t % 16, :]


def check_appended_pool(case, lens, ap, host_pool):
    """Every used chunk equals the oracle's chunk of the tokens written so
    far; full pages sit packed, filling pages in staging."""
    B, Hkv = case.B, case.Hkv
    tab = tab_host(ap.pool)
    data = ap.pool.data.cpu().numpy()
    full_units = 0
    for b in range(B):
        for pg in range((lens[b] + 15) // 16):
            pid = int(case.page_table[b, pg])
            n_tok = min(16, lens[b] - 16 * pg)
            for h in range(Hkv):
                c = pid * Hkv + h
                want = oracle.pack_chunk(host_pool[pid, h].reshape(-1), 2 * n_tok)
                start, ext = int(tab[c, 0]) * 16, int(tab[c, 1]) * 16
                assert ext == want.size
                got = data[start:start + ext]
                assert np.array_equal(got[:36], want[:36]) and np.array_equal(got[48:], want[48:])
                if n_tok == 16:
                    full_units += ext // 16
                    assert start + ext <= ap.staging_offset      # packed
                else:
                    assert start >= ap.staging_offset             # still in staging
    assert int(ap.cursor.item()) == full_units


def step_tokens(case, lens, host_pool, t):
    pos = np.array([t if t < L else -1 for L in lens], dtype=np.int32)
    vals = np.zeros((case.B, case.Hkv, 128), dtype=np.uint16)
    for b in range(case.B):
        if pos[b] >= 0:
            vals[b] = token_values(case, host_pool, b, t)
    return pos, vals


APPEND_LENS = [100, 17, 64, 1, 0, 33]


def append_case():
    return zfsynth.make_case("append", B=len(APPEND_LENS), Hq=8, Hkv=2, ctx=APPEND_LENS, sigma=0.7, inelig=0.1,
                             k_outlier_channels=3, seed=410)


def new_pool(case):
    return zf.AppendPool(case.num_pages * case.Hkv, case.B, case.Hkv, packed_bytes=case.num_pages * case.Hkv * 4144,
                         device="cuda")


def test_append_token_by_token():
    lens = APPEND_LENS
    case = append_case()
    d = DeviceCase(case, compress=False)
    pools = {}
    for name, host_pool in (("k", case.k_pool), ("v", case.v_pool)):
        ap = new_pool(case)
        for t in range(max(lens)):
            pos, vals = step_tokens(case, lens, host_pool, t)
            ap.append(dev_bf16(vals), d.pt, dev_i32(pos))
        torch.cuda.synchronize()
        assert int(ap.err.item()) == 0
        pools[name] = ap
        check_appended_pool(case, lens, ap, host_pool)
    out_a, lse_a = run_paged(d, pools["k"].pool, pools["v"].pool)
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert np.array_equal(host_u16(out_a), host_u16(out_r))
    assert torch.equal(lse_a, lse_r)


def test_append_kv_in_one_launch():
    """zf_append_paged_kv: K and V of each step in one launch give the same
    chunks as two zf_append_paged calls, and decode over them equals the raw
    twin."""
    lens = APPEND_LENS
    case = append_case()
    d = DeviceCase(case, compress=False)
    kp, vp = new_pool(case), new_pool(case)
    for t in range(max(lens)):
        pos, kvals = step_tokens(case, lens, case.k_pool, t)
        _, vvals = step_tokens(case, lens, case.v_pool, t)
        zf.append_kv(kp, vp, dev_bf16(kvals), dev_bf16(vvals), d.pt, dev_i32(pos))
    torch.cuda.synchronize()
    assert int(kp.err.item()) == 0 and int(vp.err.item()) == 0
    check_appended_pool(case, lens, kp, case.k_pool)
    check_appended_pool(case, lens, vp, case.v_pool)
    out_a, lse_a = run_paged(d, kp.pool, vp.pool)
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert np.array_equal(host_u16(out_a), host_u16(out_r))
    assert torch.equal(lse_a, lse_r)


def test_decode_while_appending():
    """Decode attention over the paged pools after every few append steps
    (sequence lengths = tokens appended so far, pages still filling in
    staging) equals the raw twin bit for bit at every checkpoint."""
    lens = APPEND_LENS
    case = append_case()
    d = DeviceCase(case, compress=False)
    kp, vp = new_pool(case), new_pool(case)
    for t in range(max(lens)):
        pos, kvals = step_tokens(case, lens, case.k_pool, t)
        _, vvals = step_tokens(case, lens, case.v_pool, t)
        zf.append_kv(kp, vp, dev_bf16(kvals), dev_bf16(vvals), d.pt, dev_i32(pos))
        if t % 7 == 6 or t == max(lens) - 1:
            now = np.minimum(np.array(lens, dtype=np.int32), t + 1)
            sl = dev_i32(now)
            lse_a = torch.empty((case.B, case.Hq), dtype=torch.float32, device="cuda")
            lse_r = torch.empty_like(lse_a)
            out_a, _ = zf.decode_attention_paged(d.q, kp.pool, vp.pool, d.pt, sl, case.max_seq_len,
                                                 num_pages=case.num_pages, Hkv=case.Hkv, sm_scale=case.sm_scale,
                                                 lse=lse_a, ws=d.ws)
            out_r, _ = zf.decode_attention_raw(d.q, d.k, d.v, d.pt, sl, case.max_seq_len, sm_scale=case.sm_scale,
                                               lse=lse_r, ws=d.ws)
            torch.cuda.synchronize()
            assert np.array_equal(host_u16(out_a), host_u16(out_r)), t
            assert torch.equal(lse_a, lse_r), t
    assert zf.get_device_error(d.ws) == 0
    assert int(kp.err.item()) == 0 and int(vp.err.item()) == 0


def test_append_kv_flags_a_bad_page_id():
    """A page-table entry outside the pool: the fused append sets the page-id
    error bit, leaves that sequence's chunk untouched, and appends every
    other sequence's token as usual."""
    lens = APPEND_LENS
    case = append_case()
    d = DeviceCase(case, compress=False)
    kp, vp = new_pool(case), new_pool(case)
    bad_pt = case.page_table.copy()
    bad_pt[2, 0] = case.num_pages + 5        # sequence 2's first page id is out of range
    pt_bad = dev_i32(bad_pt)
    pos, kvals = step_tokens(case, lens, case.k_pool, 0)
    _, vvals = step_tokens(case, lens, case.v_pool, 0)
    tab_before = tab_host(kp.pool).copy()
    zf.append_kv(kp, vp, dev_bf16(kvals), dev_bf16(vvals), pt_bad, dev_i32(pos))
    torch.cuda.synchronize()
    assert int(kp.err.item()) & zf.DEVERR_PAGE_ID
    tab = tab_host(kp.pool)
    for b in range(case.B):
        if lens[b] == 0:
            continue
        for h in range(case.Hkv):
            c = int(bad_pt[b, 0]) * case.Hkv + h if b != 2 else None
            if c is None:
                continue
            want = oracle.pack_chunk(case.k_pool[int(case.page_table[b, 0]), h].reshape(-1), 2)
            start, ext = int(tab[c, 0]) * 16, int(tab[c, 1]) * 16
            assert ext == want.size
            got = kp.pool.data[start:start + ext].cpu().numpy()
            assert np.array_equal(got[:36], want[:36]) and np.array_equal(got[48:], want[48:])
    # sequence 2's own page (the one the bad entry replaced) was not written
    c2 = int(case.page_table[2, 0]) * case.Hkv
    assert np.array_equal(tab[c2:c2 + case.Hkv], tab_before[c2:c2 + case.Hkv])


def test_paged_full_size_llama():
    """The benchmark's workload in the paged form: bitwise equal to the raw
    twin on every row, sampled rows within tolerance of the oracle."""
    case = zfsynth.config(1)
    d = DeviceCase(case, compress=False)
    pk, pv = zf.compress_paged(d.k), zf.compress_paged(d.v)
    out_p, lse_p = run_paged(d, pk, pv)
    out_r, lse_r = d.run(compressed=False)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    assert np.array_equal(host_u16(out_p), host_u16(out_r)) and torch.equal(lse_p, lse_r)
    rows = np.array([0, 17, 31])
    ref, _, _ = oracle.attention(case.q[rows], case.k_pool, case.v_pool, case.page_table[rows],
                                 case.seq_lens[rows], case.sm_scale)
    assert_attention_close(host_u16(out_p)[rows], ref, "llama (paged)")

"""GPU parity of the FP8 E4M3 comparator (reading R8) against the oracle:
quantization bit for bit, attention within the attention tolerance of the
fp64 oracle over the dequantized pools."""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import oracle
import zfsynth
from gpu_util import DeviceCase, assert_attention_close, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def pool_scale(pool_bits):
    amax = float(np.abs(zfsynth.bf16_bits_to_f32(pool_bits)).max())
    return max(amax, 1e-30) / 448.0


def test_quantize_bitwise():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.standard_normal(1 << 16) * 10.0 ** rng.uniform(-4, 3, 1 << 16),
                        [0.0, -0.0, 1e30, -1e30, np.inf, -np.inf, 2.0 ** -130, 448.0, 464.0, -465.0]])
    x = np.concatenate([x, np.zeros((-x.size) % 8)]).astype(np.float32)
    w = zfsynth.to_bf16_bits(x)
    for scale in (1.0, 0.37, 2.0 ** -7, 1e-3):
        got = zf.fp8_quantize(dev_bf16(w), scale).cpu().numpy()
        inv = np.float32(1.0) / np.float32(scale)
        ref = oracle.fp8_quantize(w, inv)
        assert np.array_equal(got, ref), f"scale {scale}: {np.count_nonzero(got != ref)} codes differ"


def check_fp8(case, rows=None):
    d = DeviceCase(case, compress=False)
    ks, vs = pool_scale(case.k_pool), pool_scale(case.v_pool)
    k8 = zf.fp8_quantize(d.k, ks)
    v8 = zf.fp8_quantize(d.v, vs)
    lse = torch.empty((case.B, case.Hq), dtype=torch.float32, device="cuda")
    out, lse = zf.decode_attention_fp8(d.q, k8, v8, ks, vs, d.pt, d.sl, case.max_seq_len, sm_scale=case.sm_scale,
                                       lse=lse, ws=d.ws)
    torch.cuda.synchronize()
    assert zf.get_device_error(d.ws) == 0
    kc, vc = k8.cpu().numpy(), v8.cpu().numpy()
    # the codes the oracle would choose
    assert np.array_equal(kc, oracle.fp8_quantize(case.k_pool, np.float32(1.0) / np.float32(ks)))
    sel = slice(None) if rows is None else rows
    ref, ref_lse, _ = oracle.attention_fp8(case.q[sel], kc, vc, ks, vs, case.page_table[sel], case.seq_lens[sel],
                                           case.sm_scale)
    got = host_u16(out)[sel]
    worst = assert_attention_close(got, ref, case.name + " (fp8)")
    got_lse = lse.cpu().numpy()[sel]
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin)
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], rtol=1e-5, atol=1e-3)
    return worst


def test_tiny_config():
    check_fp8(zfsynth.config(0))


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (32, 8), (8, 1), (64, 8)])
def test_group_sizes(Hq, Hkv):
    check_fp8(zfsynth.make_case(f"fp8-{Hq}-{Hkv}", B=3, Hq=Hq, Hkv=Hkv, ctx=[37, 200, 1], sigma=0.7, seed=300 + Hq))


def test_ragged_and_empty():
    lens = [0, 1, 15, 16, 17, 511, 512, 513, 0, 1000]
    check_fp8(zfsynth.make_case("fp8-ragged", B=len(lens), Hq=8, Hkv=2, ctx=lens, sigma=0.7, k_outlier_channels=3,
                                seed=310))


def test_llama_config_scaled():
    check_fp8(zfsynth.config(1, scale_ctx=1 / 16), rows=np.array([0, 13, 31]))


def test_llama_config_full_size_sampled():
    check_fp8(zfsynth.config(1), rows=np.array([0, 31]))

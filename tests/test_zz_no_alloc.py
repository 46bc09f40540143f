"""The no-allocation decode-attention entry point, for callers that cannot
hand the library scratch memory (a plugin given only input and output
buffers, or a process that forbids device allocation while it serves).

It is called through the C ABI and must match the regular entry point, which
takes a caller-allocated workspace, on two calls in a row with different
inputs (the fixed scratch array keeps the previous call's contents).  This
file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import zfsynth
from decode_attention_zipfusion_b200 import build as zbuild
from gpu_util import DeviceCase, assert_attention_close, bf16_to_f64, host_u16

pytestmark = pytest.mark.gpu


def noalloc_fn():
    zbuild.build()
    f = zf.lib().zf_decode_attention_noalloc
    P, i32 = ctypes.c_void_p, ctypes.c_int
    D = ctypes.POINTER(zf.CompressedDesc)
    f.argtypes = [P, D, D, i32, P, i32, P, i32, i32, i32, i32, i32, ctypes.c_float, P, P, P]
    f.restype = i32
    return f


def call_noalloc(f, d: DeviceCase, max_seq_len=None):
    c = d.case
    msl = c.max_seq_len if max_seq_len is None else max_seq_len
    out = torch.empty((c.B, c.Hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
    kd, vd = d.kz.desc(), d.vz.desc()
    st = f(ctypes.c_void_p(d.q.data_ptr()), ctypes.byref(kd), ctypes.byref(vd), c.num_pages,
           ctypes.c_void_p(d.pt.data_ptr()), c.max_pages, ctypes.c_void_p(d.sl.data_ptr()), msl, c.B, c.Hq, c.Hkv,
           128, ctypes.c_float(c.sm_scale), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def test_matches_workspace_entry_point_on_two_calls():
    f = noalloc_fn()
    cases = [zfsynth.config(1, scale_ctx=1 / 4),
             zfsynth.make_case("second", B=5, Hq=16, Hkv=4, ctx=[700, 1, 33, 0, 2048], sigma=0.7, inelig=0.1,
                               seed=77)]
    devs = [DeviceCase(c) for c in cases]
    for d in devs:
        st, out, lse = call_noalloc(f, d)
        assert st == 0, zf.lib().zf_status_string(st)
        ref_out, ref_lse = d.run()
        torch.cuda.synchronize()
        got, ref = host_u16(out), host_u16(ref_out)
        assert_attention_close(got, bf16_to_f64(ref), "no-alloc vs workspace entry point")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=1e-5, atol=1e-3)
        assert np.array_equal(got, ref)   # same kernels and split plan


def test_rejects_shapes_beyond_the_scratch_limit():
    f = noalloc_fn()
    # 1024 sequences x 64 query heads: the partial results alone need ~36 MB
    d = DeviceCase(zfsynth.make_case("big", B=1024, Hq=64, Hkv=8, ctx=16, sigma=0.5, seed=78))
    assert zf.decode_workspace_size(1024, 64, 8, 16) > (8 << 20)
    st, _, _ = call_noalloc(f, d)
    assert st == 3                      # ZF_ERR_WORKSPACE, before any launch


def test_error_word_per_call_and_clean_state_after_a_bad_call():
    """A call that meets an out-of-range page id (clamped on the device and
    flagged) reports it through zf_noalloc_device_error; the next valid call
    starts with a clear error word and leaves the shared scratch in a state
    that gives the workspace entry point's result bit for bit."""
    import copy
    f = noalloc_fn()
    get_err = zf.lib().zf_noalloc_device_error
    get_err.argtypes = [ctypes.POINTER(ctypes.c_int)]
    get_err.restype = ctypes.c_int
    case = zfsynth.config(1, scale_ctx=1 / 4)
    d = DeviceCase(case)
    bad = copy.copy(d)
    bad.pt = d.pt.clone()
    bad.pt[3, 1] = case.num_pages + 7
    code = ctypes.c_int(-1)
    st, _, _ = call_noalloc(f, bad)
    assert st == 0
    assert get_err(ctypes.byref(code)) == 0
    assert code.value & zf.DEVERR_PAGE_ID
    st, out, lse = call_noalloc(f, d)
    assert st == 0
    assert get_err(ctypes.byref(code)) == 0
    assert code.value == 0
    ref_out, ref_lse = d.run()
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(out), host_u16(ref_out))
    assert torch.equal(lse, ref_lse)

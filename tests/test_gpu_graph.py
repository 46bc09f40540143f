"""The decode calls inside a CUDA graph: captured once, then replayed, they
give the direct call's out and lse bit for bit, and each replay runs the
captured copies again (new host inputs give the new result)."""
import numpy as np
import pytest
import torch

import decode_attention_zipfusion_b200 as zf
import zfsynth
from gpu_util import DeviceCase, dev_bf16

pytestmark = pytest.mark.gpu


def graph_case(seed):
    return zfsynth.make_case("graph", B=6, Hq=16, Hkv=4, ctx=[700, 1, 0, 129, 2048, 300], sigma=0.7, inelig=0.05,
                             k_outlier_channels=3, seed=seed)


def capture(fn):
    """Capture fn() into a CUDA graph (after one warm-up call on a side stream)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        fn()
    return g


def test_device_call_replays_from_a_graph():
    case = graph_case(91)
    d = DeviceCase(case)
    out_d, lse_d = d.run()
    out = torch.empty_like(out_d)
    lse = torch.empty_like(lse_d)
    g = capture(lambda: zf.decode_attention(d.q, d.kz, d.vz, d.pt, d.sl, case.max_seq_len, num_pages=case.num_pages,
                                            Hkv=case.Hkv, sm_scale=case.sm_scale, out=out, lse=lse, ws=d.ws))
    for _ in range(3):
        out.fill_(7.0)
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out_d.view(torch.int16))
        assert torch.equal(lse, lse_d)
    assert zf.get_device_error(d.ws) == 0


def test_host_buffer_call_replays_from_a_graph():
    """zf_decode_attention_host captured with pinned host buffers: each replay
    copies the current host inputs in and the result out."""
    case = graph_case(92)
    d = DeviceCase(case)
    out_a, lse_a = d.run()
    q_b = zfsynth.to_bf16_bits(np.random.default_rng(93).standard_normal(case.q.shape).astype(np.float32))
    d_b = DeviceCase(case)
    d_b.q = dev_bf16(q_b)
    out_b, lse_b = d_b.run()

    def pinned(a, dtype):
        return torch.from_numpy(np.ascontiguousarray(a)).view(dtype).pin_memory()
    q_h = pinned(case.q, torch.bfloat16)
    pt_h = pinned(case.page_table, torch.int32)
    sl_h = pinned(case.seq_lens, torch.int32)
    out_h = torch.zeros((case.B, case.Hq, 128), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.zeros((case.B, case.Hq), dtype=torch.float32).pin_memory()
    ws = zf.decode_host_workspace(case.B, case.Hq, case.Hkv, case.page_table.shape[1], case.max_seq_len, "cuda")
    g = capture(lambda: zf.decode_attention_host(q_h, d.kz, d.vz, pt_h, sl_h, case.max_seq_len,
                                                 num_pages=case.num_pages, Hkv=case.Hkv, sm_scale=case.sm_scale,
                                                 out=out_h, lse=lse_h, ws=ws))
    for q_now, out_want, lse_want in ((case.q, out_a, lse_a), (q_b, out_b, lse_b), (case.q, out_a, lse_a)):
        q_h.copy_(torch.from_numpy(np.ascontiguousarray(q_now)).view(torch.bfloat16))
        out_h.fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.int16), out_want.cpu().view(torch.int16))
        assert torch.equal(lse_h, lse_want.cpu())
    assert zf.get_device_error(ws) == 0

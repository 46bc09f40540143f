"""Helpers shared by the GPU parity tests (host <-> device marshalling and the
tolerance of the attention comparison)."""
import numpy as np
import torch

import decode_attention_zipfusion_b200 as zf

# Attention tolerance fixed for this path: max |err| <= 1e-2 * max(1, |ref|),
# element by element, against the fp64 oracle.
RTOL = 1e-2


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_u32(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy().view(np.uint32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_attention_close(got_bits: np.ndarray, ref: np.ndarray, what=""):
    got = bf16_to_f64(got_bits)
    err = np.abs(got - ref)
    tol = RTOL * np.maximum(1.0, np.abs(ref))
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: got {got[i]} "
                             f"ref {ref[i]} err {err[i]:.3g} tol {tol[i]:.3g}")
    return float((err / np.maximum(1.0, np.abs(ref))).max())


class DeviceCase:
    """A zfsynth.Case uploaded to the GPU, with its compressed pools."""

    def __init__(self, case, compress=True):
        self.case = case
        self.q = dev_bf16(case.q)
        self.k = dev_bf16(case.k_pool)
        self.v = dev_bf16(case.v_pool)
        self.pt = dev_i32(case.page_table)
        self.sl = dev_i32(case.seq_lens)
        self.kz = zf.compress(self.k) if compress else None
        self.vz = zf.compress(self.v) if compress else None
        self.ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, case.max_seq_len, self.q.device)

    def run(self, compressed=True, max_seq_len=None, out=None, lse=None):
        c = self.case
        msl = c.max_seq_len if max_seq_len is None else max_seq_len
        if lse is None:
            lse = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
        if compressed:
            out, lse = zf.decode_attention(self.q, self.kz, self.vz, self.pt, self.sl, msl,
                                           num_pages=c.num_pages, Hkv=c.Hkv, sm_scale=c.sm_scale,
                                           out=out, lse=lse, ws=self.ws)
        else:
            out, lse = zf.decode_attention_raw(self.q, self.k, self.v, self.pt, self.sl, msl,
                                               sm_scale=c.sm_scale, out=out, lse=lse, ws=self.ws)
        return out, lse


def oracle_attention_rows(case, rows=None):
    """The fp64 oracle's attention for the given rows (all when None), one
    sequence per task of a thread pool (the oracle's C call releases the
    GIL), so full-size workloads take seconds.  Returns (out, lse) stacked in
    row order."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    rows = np.arange(case.B) if rows is None else np.asarray(rows)

    def one(b):
        sel = slice(int(b), int(b) + 1)
        out, lse, _ = oracle.attention(case.q[sel], case.k_pool, case.v_pool, case.page_table[sel],
                                       case.seq_lens[sel], case.sm_scale)
        return out[0], lse[0]
    with ThreadPoolExecutor(max_workers=min(len(rows), os.cpu_count() or 1)) as ex:
        res = list(ex.map(one, rows))
    return np.stack([r[0] for r in res]), np.stack([r[1] for r in res])

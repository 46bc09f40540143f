"""Lossless BF16 KV-cache compression with fused decode attention for B200.

Python binding of ``libzf.so`` (the C ABI declared in ``include/zf.h``).  This
module only marshals arguments: torch provides device memory and the current
stream, every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing the calls raise.

Method: "Run AI Faster With Lossless Compressed Memory" (the ZipFusion
summary): one shared base exponent per 64-value block, a 4-bit exponent offset
per value, sign and mantissa verbatim (12 bits per value for eligible blocks,
raw fallback otherwise), values rebuilt in registers inside attention with a
single integer addition.
"""
from __future__ import annotations

import ctypes
import math
import os
import struct

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzf.so")

BLOCK = 64          # values per codec block
UNIT = 16           # bytes per offset-table unit
PAGE = 16           # tokens per KV page
HEAD_DIM = 128

# kernels launched per call (for launch accounting)
LAUNCHES_DECODE = 1        # attention with the split merge fused in
LAUNCHES_COMPRESS = 1      # plus one memset of the scan state
LAUNCHES_DECOMPRESS = 1

ZF_OK = 0
_STATUS = {0: "ZF_OK", 1: "ZF_ERR_INVALID_ARG", 2: "ZF_ERR_UNSUPPORTED", 3: "ZF_ERR_WORKSPACE",
           4: "ZF_ERR_CUDA", 5: "ZF_ERR_BAD_INPUT", 6: "ZF_ERR_TIMEOUT"}
DEVERR_PAGE_ID, DEVERR_SEQ_LEN, DEVERR_EXTENT, DEVERR_TIMEOUT = 1, 2, 4, 8


class ZfError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


class CompressedDesc(ctypes.Structure):
    """Mirror of zf_kv_compressed."""
    _fields_ = [("payload", ctypes.c_void_p), ("offs", ctypes.c_void_p), ("base", ctypes.c_void_p),
                ("elig", ctypes.c_void_p), ("n_values", ctypes.c_int64), ("payload_cap_bytes", ctypes.c_int64)]


class PagedDesc(ctypes.Structure):
    """Mirror of zf_kv_paged."""
    _fields_ = [("data", ctypes.c_void_p), ("chunk_tab", ctypes.c_void_p), ("num_chunks", ctypes.c_int64),
                ("data_cap_bytes", ctypes.c_int64)]


_lib = None


def lib():
    """Load libzf.so (built by ``python -m decode_attention_zipfusion_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m decode_attention_zipfusion_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        D = ctypes.POINTER(CompressedDesc)
        L.zf_version.restype = i32
        L.zf_status_string.argtypes = [i32]
        L.zf_status_string.restype = ctypes.c_char_p
        L.zf_compressed_bound.argtypes = [i64]
        L.zf_compressed_bound.restype = sz
        L.zf_compress_workspace_size.argtypes = [i64]
        L.zf_compress_workspace_size.restype = sz
        L.zf_compress_kv.argtypes = [P, i64, D, P, sz, P]
        L.zf_decompress_kv.argtypes = [D, P, P]
        L.zf_validate_compressed.argtypes = [D, P, P]
        L.zf_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.zf_decode_workspace_size.restype = sz
        attn = [P, D, D, i32, P, i32, P, i32, i32, i32, i32, i32, ctypes.c_float, P, P, P, sz, P]
        L.zf_decode_attention.argtypes = attn
        L.zf_decode_attention_raw.argtypes = [P, P, P] + attn[3:]
        L.zf_fp8_quantize.argtypes = [P, i64, ctypes.c_float, P, P]
        PD = ctypes.POINTER(PagedDesc)
        L.zf_paged_bound.argtypes = [i64]
        L.zf_paged_bound.restype = sz
        L.zf_compress_paged.argtypes = [P, i64, PD, P, sz, P]
        L.zf_decompress_paged.argtypes = [PD, P, P]
        L.zf_decode_attention_paged.argtypes = [P, PD, PD] + attn[3:]
        L.zf_append_staging_bytes.argtypes = [i32, i32]
        L.zf_append_staging_bytes.restype = sz
        L.zf_append_paged.argtypes = [PD, P, P, i32, P, i32, i32, i64, P, P, P]
        L.zf_append_paged_kv.argtypes = [PD, PD, P, P, P, i32, P, i32, i32, i64, i64, P, P, P, P]
        L.zf_decode_attention_fp8.argtypes = [P, P, P, ctypes.c_float, ctypes.c_float] + attn[3:]
        L.zf_decode_host_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.zf_decode_host_workspace_size.restype = sz
        L.zf_decode_attention_host.argtypes = attn
        L.zf_check_bounded_wait.argtypes = [i32, P, P, P]
        L.zf_clear_device_error.argtypes = [P, P]
        L.zf_get_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
        for f in ("zf_compress_kv", "zf_decompress_kv", "zf_validate_compressed", "zf_decode_attention",
                  "zf_decode_attention_raw", "zf_clear_device_error", "zf_get_device_error", "zf_fp8_quantize",
                  "zf_decode_attention_fp8", "zf_compress_paged", "zf_decompress_paged",
                  "zf_decode_attention_paged", "zf_append_paged", "zf_append_paged_kv", "zf_decode_attention_host",
                  "zf_check_bounded_wait"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != ZF_OK:
        raise ZfError(status, what)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _bits(x: torch.Tensor) -> torch.Tensor:
    """bf16 / int16 / uint16 tensor -> contiguous 16-bit storage."""
    if x.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected a 16-bit (bf16) tensor, got {x.dtype}")
    return x.contiguous()


class CompressedKV:
    """A compressed flat BF16 buffer on the device (see include/zf.h)."""

    def __init__(self, payload, offs, base, elig, n_values):
        self.payload = payload    # uint8 [cap]
        self.offs = offs          # int32 [n_blocks + 1]  (u32 bits)
        self.base = base          # uint8 [>= n_blocks]
        self.elig = elig          # int32 [ceil(n_blocks / 32)]  (u32 bits)
        self.n_values = int(n_values)

    @property
    def n_blocks(self) -> int:
        return self.n_values // BLOCK

    @classmethod
    def empty(cls, n_values: int, device, payload_cap: int | None = None) -> "CompressedKV":
        if n_values % BLOCK:
            raise ValueError("n_values must be a multiple of 64")
        nb = n_values // BLOCK
        cap = int(lib().zf_compressed_bound(n_values)) if payload_cap is None else int(payload_cap)
        return cls(torch.empty(max(cap, 16), dtype=torch.uint8, device=device),
                   torch.empty(nb + 1, dtype=torch.int32, device=device),
                   torch.empty(max(16, (nb + 15) // 16 * 16), dtype=torch.uint8, device=device),
                   torch.empty(max(1, (nb + 31) // 32), dtype=torch.int32, device=device), n_values)

    def desc(self) -> CompressedDesc:
        return CompressedDesc(self.payload.data_ptr(), self.offs.data_ptr(), self.base.data_ptr(),
                              self.elig.data_ptr(), self.n_values, self.payload.numel())

    def units(self) -> int:
        """Total payload size in 16-byte units (reads offs[n_blocks]; syncs)."""
        return int(self.offs[-1].item()) & 0xFFFFFFFF

    def compressed_bytes(self) -> int:
        """Payload plus metadata (offsets, bases, eligibility bits) in bytes."""
        nb = self.n_blocks
        return self.units() * UNIT + 4 * (nb + 1) + nb + 4 * ((nb + 31) // 32)

    def shrink(self) -> "CompressedKV":
        """Copy the payload into an exact-size buffer (syncs once)."""
        n = self.units() * UNIT
        self.payload = self.payload[: max(n, 16)].clone()
        return self


def compress(x: torch.Tensor, out: CompressedKV | None = None, ws: torch.Tensor | None = None,
             stream=None) -> CompressedKV:
    """Compress a CUDA bf16 tensor (any shape, numel % 64 == 0)."""
    x = _bits(x)
    n = x.numel()
    if out is None:
        out = CompressedKV.empty(n, x.device)
    if ws is None:
        ws = torch.empty(max(16, int(lib().zf_compress_workspace_size(n))), dtype=torch.uint8, device=x.device)
    d = out.desc()
    _check(lib().zf_compress_kv(_ptr(x), n, ctypes.byref(d), _ptr(ws), ws.numel(), _stream(stream)),
           "zf_compress_kv")
    return out


def decompress(z: CompressedKV, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rebuild the bf16 values (flat tensor of z.n_values)."""
    if out is None:
        out = torch.empty(z.n_values, dtype=torch.bfloat16, device=z.payload.device)
    d = z.desc()
    _check(lib().zf_decompress_kv(ctypes.byref(d), _ptr(out), _stream(stream)), "zf_decompress_kv")
    return out


def validate(z: CompressedKV, stream=None) -> int:
    """Number of inconsistent blocks (0 for a well-formed buffer; syncs)."""
    bad = torch.zeros(1, dtype=torch.int32, device=z.payload.device)
    d = z.desc()
    _check(lib().zf_validate_compressed(ctypes.byref(d), _ptr(bad), _stream(stream)), "zf_validate_compressed")
    return int(bad.item())


def decode_workspace_size(B: int, Hq: int, Hkv: int, max_seq_len: int, num_sms: int = 0) -> int:
    return int(lib().zf_decode_workspace_size(B, Hq, Hkv, max_seq_len, num_sms))


def decode_workspace(B: int, Hq: int, Hkv: int, max_seq_len: int, device) -> torch.Tensor:
    """Allocate a zero-filled decode workspace (the split counters and the
    device error word must start at zero; every call leaves the counters at
    zero, so the workspace may be reused for any shape that fits)."""
    props = torch.cuda.get_device_properties(device)
    n = decode_workspace_size(B, Hq, Hkv, max_seq_len, props.multi_processor_count)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


WAITCHECK_TIMEOUT, WAITCHECK_ABORT, WAITCHECK_COMPLETE, WAITCHECK_PLAIN_TIMEOUT = 0, 1, 2, 3
WAITCHECK_LOOKBACK_TIMEOUT, WAITCHECK_LOOKBACK_COMPLETE, WAITCHECK_COMPRESS_STALL = 4, 5, 6


def check_bounded_wait(mode: int, err_ws: torch.Tensor, stream=None) -> tuple[int, int]:
    """Run the kernels' bounded barrier wait in one of the zf_waitcheck_mode
    situations; returns (outcome, nanoseconds): outcome 1 completed (the
    look-back modes: with the right prefix), 2 look-back completed with a
    wrong prefix, 0 called off, -1 gave up (which also sets DEVERR_TIMEOUT in
    err_ws's error word).  Synchronises."""
    result = torch.zeros(2, dtype=torch.int64, device=err_ws.device)
    _check(lib().zf_check_bounded_wait(mode, _ptr(result), _ptr(err_ws), _stream(stream)), "zf_check_bounded_wait")
    r = result.cpu().tolist()
    return int(r[0]), int(r[1])


def clear_device_error(ws: torch.Tensor, stream=None):
    _check(lib().zf_clear_device_error(_ptr(ws), _stream(stream)), "zf_clear_device_error")


def get_device_error(ws: torch.Tensor) -> int:
    """Device error word bits (DEVERR_*); synchronises."""
    code = ctypes.c_int(0)
    lib().zf_get_device_error(_ptr(ws), ctypes.byref(code))
    return code.value


def _attn_common(q, page_table, seq_lens, max_seq_len, sm_scale, out, lse, ws, Hkv):
    q = _bits(q)
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if ws is None:
        ws = decode_workspace(B, Hq, Hkv, max_seq_len, q.device)
    if page_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("page_table and seq_lens must be int32")
    return q, B, Hq, D, out, sm_scale, ws, page_table.contiguous(), seq_lens.contiguous()


def decode_attention(q, kz: CompressedKV, vz: CompressedKV, page_table, seq_lens, max_seq_len: int, *,
                     num_pages: int, Hkv: int, sm_scale=None, out=None, lse=None, ws=None, stream=None):
    """Decode attention over the compressed paged cache; returns (out, lse)."""
    q, B, Hq, D, out, sm_scale, ws, pt, sl = _attn_common(q, page_table, seq_lens, max_seq_len, sm_scale,
                                                          out, lse, ws, Hkv)
    kd, vd = kz.desc(), vz.desc()
    _check(lib().zf_decode_attention(_ptr(q), ctypes.byref(kd), ctypes.byref(vd), num_pages, _ptr(pt),
                                     pt.shape[1], _ptr(sl), max_seq_len, B, Hq, Hkv, D, float(sm_scale),
                                     _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "zf_decode_attention")
    return out, lse


def decode_host_workspace(B: int, Hq: int, Hkv: int, max_pages_per_seq: int, max_seq_len: int,
                          device) -> torch.Tensor:
    """Zero-filled device workspace for decode_attention_host."""
    props = torch.cuda.get_device_properties(device)
    n = int(lib().zf_decode_host_workspace_size(B, Hq, Hkv, max_pages_per_seq, max_seq_len,
                                                props.multi_processor_count))
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


_HALF = (torch.bfloat16, torch.int16, torch.uint16)


def _host(t, dtypes, name):
    if t.device.type != "cpu" or t.dtype not in dtypes or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {'/'.join(map(str, dtypes))} tensor in host memory")
    return t.data_ptr()


def decode_attention_host(q, kz: CompressedKV, vz: CompressedKV, page_table, seq_lens, max_seq_len: int, *,
                          num_pages: int, Hkv: int, sm_scale=None, out=None, lse=None, ws=None, stream=None):
    """Decode attention over the compressed cache with q, page_table,
    seq_lens, out (and lse if given) in HOST memory: one library call
    enqueues the input copies, the kernel and the output copies on the
    stream.  Returns (out, lse); synchronise the stream before reading them.
    Pinned host tensors make the copies asynchronous."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16).pin_memory()
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if ws is None:
        ws = decode_host_workspace(B, Hq, Hkv, page_table.shape[1], max_seq_len, kz.payload.device)
    kd, vd = kz.desc(), vz.desc()
    _check(lib().zf_decode_attention_host(
        _host(q, _HALF, "q"), ctypes.byref(kd), ctypes.byref(vd), num_pages,
        _host(page_table, (torch.int32,), "page_table"), page_table.shape[1],
        _host(seq_lens, (torch.int32,), "seq_lens"), max_seq_len, B, Hq, Hkv, D, float(sm_scale), _host(out, _HALF, "out"),
        None if lse is None else _host(lse, (torch.float32,), "lse"), _ptr(ws), ws.numel(), _stream(stream)),
        "zf_decode_attention_host")
    return out, lse


def decode_attention_raw(q, k_pool, v_pool, page_table, seq_lens, max_seq_len: int, *, sm_scale=None,
                         out=None, lse=None, ws=None, stream=None):
    """Decode attention over an uncompressed [P][Hkv][16][128] bf16 cache."""
    k_pool = _bits(k_pool)
    v_pool = _bits(v_pool)
    P, Hkv = k_pool.shape[0], k_pool.shape[1]
    q, B, Hq, D, out, sm_scale, ws, pt, sl = _attn_common(q, page_table, seq_lens, max_seq_len, sm_scale,
                                                          out, lse, ws, Hkv)
    _check(lib().zf_decode_attention_raw(_ptr(q), _ptr(k_pool), _ptr(v_pool), P, _ptr(pt), pt.shape[1],
                                         _ptr(sl), max_seq_len, B, Hq, Hkv, D, float(sm_scale), _ptr(out),
                                         _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "zf_decode_attention_raw")
    return out, lse


# ------------------------------------------------------- FP8 E4M3 comparator

def fp8_quantize(x: torch.Tensor, scale: float, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 tensor -> uint8 E4M3 codes of the same shape: code = E4M3 nearest
    to value / scale (single-precision product with 1/scale, ties to even,
    saturating at +-448).  The lossy comparator of the method."""
    x = _bits(x)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().zf_fp8_quantize(_ptr(x), x.numel(), float(np.float32(1.0) / np.float32(scale)), _ptr(out),
                                 _stream(stream)), "zf_fp8_quantize")
    return out


def decode_attention_fp8(q, k_fp8, v_fp8, k_scale: float, v_scale: float, page_table, seq_lens,
                         max_seq_len: int, *, sm_scale=None, out=None, lse=None, ws=None, stream=None):
    """Decode attention over E4M3 [P][Hkv][16][128] pools with one scale each."""
    if k_fp8.dtype != torch.uint8 or v_fp8.dtype != torch.uint8:
        raise TypeError("FP8 pools are uint8 E4M3 codes")
    k_fp8, v_fp8 = k_fp8.contiguous(), v_fp8.contiguous()
    P, Hkv = k_fp8.shape[0], k_fp8.shape[1]
    q, B, Hq, D, out, sm_scale, ws, pt, sl = _attn_common(q, page_table, seq_lens, max_seq_len, sm_scale,
                                                          out, lse, ws, Hkv)
    _check(lib().zf_decode_attention_fp8(_ptr(q), _ptr(k_fp8), _ptr(v_fp8), float(k_scale), float(v_scale), P,
                                         _ptr(pt), pt.shape[1], _ptr(sl), max_seq_len, B, Hq, Hkv, D,
                                         float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(stream)), "zf_decode_attention_fp8")
    return out, lse


# ---------------------------------------------------------------- paged form

CHUNK_VALUES = 2048


class PagedKV:
    """A K or V pool in the paged form on the device (see include/zf.h)."""

    def __init__(self, data, chunk_tab, num_chunks):
        self.data = data              # uint8 [cap]
        self.chunk_tab = chunk_tab    # int32 [num_chunks][2] (u32 {start, extent} in 16-byte units)
        self.num_chunks = num_chunks

    @staticmethod
    def empty(num_chunks: int, device) -> "PagedKV":
        cap = int(lib().zf_paged_bound(num_chunks))
        data = torch.empty(max(cap, 16), dtype=torch.uint8, device=device)
        tab = torch.zeros((max(num_chunks, 1), 2), dtype=torch.int32, device=device)
        return PagedKV(data, tab, num_chunks)

    def desc(self) -> PagedDesc:
        return PagedDesc(_ptr(self.data).value, _ptr(self.chunk_tab).value, self.num_chunks, self.data.numel())

    def units(self) -> int:
        """16-byte units up to the end of the last extent (syncs)."""
        t = self.chunk_tab[: self.num_chunks].cpu().numpy().view(np.uint32).astype(np.int64)
        return int((t[:, 0] + t[:, 1]).max()) if t.size else 0


def compress_paged(x: torch.Tensor, out: PagedKV | None = None, ws: torch.Tensor | None = None,
                   stream=None) -> PagedKV:
    """Paged form of a CUDA bf16 pool [num_pages][Hkv][16][128] (numel % 2048 == 0)."""
    x = _bits(x)
    n = x.numel()
    if n % CHUNK_VALUES:
        raise ValueError("the pool must hold whole 2048-value chunks")
    nc = n // CHUNK_VALUES
    if out is None:
        out = PagedKV.empty(nc, x.device)
    if ws is None:
        ws = torch.empty(max(16, int(lib().zf_compress_workspace_size(n))), dtype=torch.uint8, device=x.device)
    d = out.desc()
    _check(lib().zf_compress_paged(_ptr(x), nc, ctypes.byref(d), _ptr(ws), ws.numel(), _stream(stream)),
           "zf_compress_paged")
    return out


def decompress_paged(z: PagedKV, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rebuild the bf16 values of a paged pool (flat tensor of num_chunks * 2048)."""
    if out is None:
        out = torch.empty(z.num_chunks * CHUNK_VALUES, dtype=torch.bfloat16, device=z.data.device)
    d = z.desc()
    _check(lib().zf_decompress_paged(ctypes.byref(d), _ptr(out), _stream(stream)), "zf_decompress_paged")
    return out


def decode_attention_paged(q, pk: PagedKV, pv: PagedKV, page_table, seq_lens, max_seq_len: int, *, num_pages: int,
                           Hkv: int, sm_scale=None, out=None, lse=None, ws=None, stream=None):
    """Decode attention over paged-form K and V pools."""
    q, B, Hq, D, out, sm_scale, ws, pt, sl = _attn_common(q, page_table, seq_lens, max_seq_len, sm_scale,
                                                          out, lse, ws, Hkv)
    kd, vd = pk.desc(), pv.desc()
    _check(lib().zf_decode_attention_paged(_ptr(q), ctypes.byref(kd), ctypes.byref(vd), num_pages, _ptr(pt),
                                           pt.shape[1], _ptr(sl), max_seq_len, B, Hq, Hkv, D, float(sm_scale),
                                           _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "zf_decode_attention_paged")
    return out, lse


class AppendPool:
    """A paged pool filled token by token (zf_append_paged): data =
    [packed region | staging extents of B x Hkv (sequence, head) pairs]."""

    def __init__(self, num_chunks: int, B: int, Hkv: int, packed_bytes: int, device):
        self.B, self.Hkv = B, Hkv
        self.staging_offset = ((packed_bytes + 15) // 16) * 16
        cap = self.staging_offset + int(lib().zf_append_staging_bytes(B, Hkv))
        data = torch.empty(cap, dtype=torch.uint8, device=device)
        tab = torch.zeros((max(num_chunks, 1), 2), dtype=torch.int32, device=device)
        self.pool = PagedKV(data, tab, num_chunks)
        self.cursor = torch.zeros(1, dtype=torch.int32, device=device)   # u32 units of the packed region
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def append(self, vals: torch.Tensor, page_table: torch.Tensor, positions: torch.Tensor, stream=None):
        """vals [B][Hkv][128] bf16: the new token of each sequence at
        positions[b] (int32, -1 = none)."""
        vals = _bits(vals)
        if tuple(vals.shape) != (self.B, self.Hkv, 128):
            raise ValueError("vals must be [B][Hkv][128]")
        if page_table.dtype != torch.int32 or positions.dtype != torch.int32:
            raise TypeError("page_table and positions must be int32")
        pt = page_table.contiguous()
        d = self.pool.desc()
        _check(lib().zf_append_paged(ctypes.byref(d), _ptr(vals), _ptr(pt), pt.shape[1], _ptr(positions.contiguous()),
                                     self.B, self.Hkv, self.staging_offset, _ptr(self.cursor), _ptr(self.err),
                                     _stream(stream)), "zf_append_paged")


def append_kv(kp: AppendPool, vp: AppendPool, k_vals: torch.Tensor, v_vals: torch.Tensor, page_table: torch.Tensor,
              positions: torch.Tensor, stream=None):
    """K and V of one decode step in one launch (zf_append_paged_kv): the same
    as kp.append(k_vals, ...) and vp.append(v_vals, ...).  Device errors of
    both pools go to kp.err."""
    if (kp.B, kp.Hkv) != (vp.B, vp.Hkv) or kp is vp:
        raise ValueError("kp and vp must be two pools of the same shape")
    k_vals, v_vals = _bits(k_vals), _bits(v_vals)
    for x in (k_vals, v_vals):
        if tuple(x.shape) != (kp.B, kp.Hkv, 128):
            raise ValueError("k_vals and v_vals must be [B][Hkv][128]")
    if page_table.dtype != torch.int32 or positions.dtype != torch.int32:
        raise TypeError("page_table and positions must be int32")
    pt = page_table.contiguous()
    kd, vd = kp.pool.desc(), vp.pool.desc()
    _check(lib().zf_append_paged_kv(ctypes.byref(kd), ctypes.byref(vd), _ptr(k_vals), _ptr(v_vals), _ptr(pt),
                                    pt.shape[1], _ptr(positions.contiguous()), kp.B, kp.Hkv, kp.staging_offset,
                                    vp.staging_offset, _ptr(kp.cursor), _ptr(vp.cursor), _ptr(kp.err),
                                    _stream(stream)), "zf_append_paged_kv")


# ------------------------------------------------------------- save / load

# File = 32-byte little-endian header {magic, values per block, n_values (flat)
# or num_chunks (paged), payload units, reserved}, then the arrays as stored.
_FILE_HEADER = struct.Struct("<4sIqqq")
_MAGIC_FLAT = b"ZF01"
_MAGIC_PAGED = b"ZFP1"


def save(z, path: str) -> None:
    """Write a compressed buffer (CompressedKV or PagedKV) to a file: the
    header, then offsets, bases, eligibility words and payload (flat form) or
    the chunk table and data (paged form), exactly the bytes in use.  Copies
    to the host (syncs)."""
    if isinstance(z, CompressedKV):
        nb, units = z.n_blocks, z.units()
        head = _FILE_HEADER.pack(_MAGIC_FLAT, BLOCK, z.n_values, units, 0)
        arrays = [z.offs[: nb + 1], z.base[:nb], z.elig[: (nb + 31) // 32], z.payload[: units * UNIT]]
    elif isinstance(z, PagedKV):
        units = z.units()
        head = _FILE_HEADER.pack(_MAGIC_PAGED, BLOCK, z.num_chunks, units, 0)
        arrays = [z.chunk_tab[: z.num_chunks], z.data[: units * UNIT]]
    else:
        raise TypeError("save() takes a CompressedKV or a PagedKV")
    with open(path, "wb") as f:
        f.write(head)
        for a in arrays:
            f.write(a.contiguous().cpu().numpy().tobytes())


def load(path: str, device) -> "CompressedKV | PagedKV":
    """Read a file written by save() into a new buffer on `device` (with the
    full capacity a later compress into it needs).  Raises ValueError for a
    wrong magic, block size or length, or an offset table whose total does
    not match the payload."""
    with open(path, "rb") as f:
        raw = f.read()
    if len(raw) < _FILE_HEADER.size:
        raise ValueError(f"{path}: too short for a header")
    magic, block, n, units, _ = _FILE_HEADER.unpack_from(raw)
    if block != BLOCK or n < 0 or units < 0:
        raise ValueError(f"{path}: unsupported header")
    pos = _FILE_HEADER.size

    def take(count: int, dtype) -> torch.Tensor:
        nonlocal pos
        nbytes = count * np.dtype(dtype).itemsize
        if pos + nbytes > len(raw):
            raise ValueError(f"{path}: truncated")
        a = np.frombuffer(raw, dtype=dtype, count=count, offset=pos).copy()
        pos += nbytes
        return torch.from_numpy(a)

    if magic == _MAGIC_FLAT:
        if n % BLOCK:
            raise ValueError(f"{path}: n_values is not a multiple of {BLOCK}")
        nb = n // BLOCK
        offs, base = take(nb + 1, np.int32), take(nb, np.uint8)
        elig, payload = take((nb + 31) // 32, np.int32), take(units * UNIT, np.uint8)
        if int(offs[-1]) & 0xFFFFFFFF != units:
            raise ValueError(f"{path}: offset total does not match the payload")
        z = CompressedKV.empty(n, device)
        z.offs.copy_(offs)
        z.base[:nb].copy_(base)
        z.elig[: elig.numel()].copy_(elig)
        z.payload[: units * UNIT].copy_(payload)
    elif magic == _MAGIC_PAGED:
        tab, data = take(2 * n, np.int32).view(n, 2), take(units * UNIT, np.uint8)
        ends = tab.numpy().view(np.uint32).astype(np.int64).sum(1) if n else np.zeros(0, np.int64)
        if ends.size and int(ends.max()) != units:
            raise ValueError(f"{path}: chunk table does not match the data")
        z = PagedKV.empty(n, device)
        z.chunk_tab[:n].copy_(tab)
        z.data[: units * UNIT].copy_(data)
    else:
        raise ValueError(f"{path}: not a compressed KV file")
    if pos != len(raw):
        raise ValueError(f"{path}: trailing bytes")
    return z


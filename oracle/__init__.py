"""CPU oracle: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product (``decode_attention_zipfusion_b200``) never imports it and shares no
code with it.

The arithmetic lives in ``zf_oracle.c`` (one value at a time, fp64 for the
attention); this module only marshals numpy arrays through ctypes.  The method
is the one in "Run AI Faster With Lossless Compressed Memory" (the ZipFusion
summary, "Twelve Bits and One Addition"): a shared base exponent per block, a
4-bit offset per value, raw fallback for blocks whose exponent spread exceeds
15.  The readings taken where that page is silent are listed at the top of
``zf_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zf_oracle.c")
_LIB = os.path.join(_HERE, "libzf_oracle.so")

BLOCK = 64            # values per codec block (canonical form)
UNIT = 16             # bytes per offset-table unit (canonical form)
PAGE = 16             # tokens per KV page


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        L.zfo_block_stats.argtypes = [P, i32, P, P]
        L.zfo_block_eligible.argtypes = [P, i32]
        L.zfo_block_eligible.restype = i32
        L.zfo_block_bytes.argtypes = [i32, i32]
        L.zfo_block_bytes.restype = i64
        L.zfo_pack_block.argtypes = [P, i32, P, P, P]
        L.zfo_pack_block.restype = i64
        L.zfo_unpack_block.argtypes = [P, i32, ctypes.c_uint8, i32, P]
        L.zfo_compress_general.argtypes = [P, i64, i32, P, P, P, P]
        L.zfo_compress_general.restype = i64
        L.zfo_decompress_general.argtypes = [P, P, P, P, i32, i64, i64, P]
        L.zfo_compress.argtypes = [P, i64, P, P, P, P]
        L.zfo_compress.restype = i64
        L.zfo_decompress.argtypes = [P, P, P, P, i64, i64, P]
        L.zfo_attention.argtypes = [P, P, P, i64, P, i32, P, i32, i32, i32, i32, i32,
                                    ctypes.c_double, P, P, P]
        L.zfo_attention.restype = i32
        L.zfo_pack_chunk.argtypes = [P, i32, P]
        L.zfo_pack_chunk.restype = i64
        L.zfo_compress_paged.argtypes = [P, i64, P, P]
        L.zfo_compress_paged.restype = i64
        L.zfo_decompress_paged.argtypes = [P, P, i64, i32, P]
        L.zfo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.zfo_e4m3_decode.restype = ctypes.c_double
        L.zfo_e4m3_encode.argtypes = [ctypes.c_double]
        L.zfo_e4m3_encode.restype = ctypes.c_uint8
        L.zfo_fp8_quantize.argtypes = [P, i64, ctypes.c_float, P]
        L.zfo_fp8_dequantize.argtypes = [P, i64, ctypes.c_double, P]
        L.zfo_attention_fp8.argtypes = [P, P, P, ctypes.c_double, ctypes.c_double, i64, P, i32, P, i32, i32,
                                        i32, i32, i32, ctypes.c_double, P, P, P]
        L.zfo_attention_fp8.restype = i32
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------- codec

class Compressed:
    """Canonical compressed buffer: payload bytes, offset table (16-byte units,
    n_blocks + 1 entries), base exponents, eligibility bitmask (u32 words)."""

    def __init__(self, payload, offs, base, elig, n_values):
        self.payload = payload
        self.offs = offs
        self.base = base
        self.elig = elig
        self.n_values = n_values

    @property
    def n_blocks(self) -> int:
        return self.n_values // BLOCK

    @property
    def units(self) -> int:
        return int(self.offs[-1])

    def eligible(self) -> np.ndarray:
        """Per-block eligibility as a bool array (bit i%32 of word i/32)."""
        bits = (self.elig[:, None] >> np.arange(32, dtype=np.uint32)) & 1
        return bits.reshape(-1)[: self.n_blocks].astype(bool)


def compress(values: np.ndarray) -> Compressed:
    """Compress a flat uint16 (bf16 bit pattern) array, length % 64 == 0."""
    v = np.ascontiguousarray(values, dtype=np.uint16).reshape(-1)
    n = v.size
    if n % BLOCK:
        raise ValueError("length must be a multiple of 64")
    nb = n // BLOCK
    payload = np.zeros(2 * n + 16, dtype=np.uint8)
    offs = np.zeros(nb + 1, dtype=np.uint32)
    base = np.zeros(max(nb, 1), dtype=np.uint8)
    elig = np.zeros(max((nb + 31) // 32, 1), dtype=np.uint32)
    units = lib().zfo_compress(_ptr(v), n, _ptr(payload), _ptr(offs), _ptr(base), _ptr(elig))
    return Compressed(payload[: units * UNIT].copy(), offs, base[:nb], elig[: (nb + 31) // 32], n)


def decompress(c: Compressed, i0: int = 0, i1: int | None = None) -> np.ndarray:
    """Rebuild blocks [i0, i1) (default: all) as uint16 values."""
    i1 = c.n_blocks if i1 is None else i1
    out = np.empty((i1 - i0) * BLOCK, dtype=np.uint16)
    if i1 > i0:
        payload = c.payload if c.payload.size else np.zeros(16, np.uint8)
        lib().zfo_decompress(_ptr(payload), _ptr(c.offs), _ptr(c.base), _ptr(c.elig), i0, i1, _ptr(out))
    return out


def compress_general(values: np.ndarray, n: int):
    """Block size n (even) variant, offsets in bytes; for brute-force pins."""
    v = np.ascontiguousarray(values, dtype=np.uint16).reshape(-1)
    assert v.size % n == 0 and n % 2 == 0
    nb = v.size // n
    payload = np.zeros(2 * v.size + 16, dtype=np.uint8)
    offs = np.zeros(nb + 1, dtype=np.int64)
    base = np.zeros(max(nb, 1), dtype=np.uint8)
    elig = np.zeros(max(nb, 1), dtype=np.uint8)
    total = lib().zfo_compress_general(_ptr(v), v.size, n, _ptr(payload), _ptr(offs), _ptr(base), _ptr(elig))
    return payload[:total].copy(), offs, base[:nb], elig[:nb]


def decompress_general(payload, offs, base, elig, n: int) -> np.ndarray:
    nb = base.size
    out = np.empty(nb * n, dtype=np.uint16)
    pl = payload if payload.size else np.zeros(16, np.uint8)
    lib().zfo_decompress_general(_ptr(pl), _ptr(offs), _ptr(base), _ptr(elig), n, 0, nb, _ptr(out))
    return out


def block_stats(block: np.ndarray):
    b = np.ascontiguousarray(block, dtype=np.uint16)
    lo = ctypes.c_int()
    hi = ctypes.c_int()
    lib().zfo_block_stats(_ptr(b), b.size, ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


# --------------------------------------------------------------- attention

def attention(q, k_pool, v_pool, page_table, seq_lens, sm_scale, want_p=False):
    """fp64 paged GQA decode attention.

    q [B][Hq][D] u16, k_pool/v_pool [P][Hkv][16][D] u16, page_table [B][maxp]
    i32, seq_lens [B] i32.  Returns (out f64 [B][Hq][D], lse f64 [B][Hq]
    natural log, p f64 [B][Hq][maxp*16] or None)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_pool = np.ascontiguousarray(k_pool, dtype=np.uint16)
    v_pool = np.ascontiguousarray(v_pool, dtype=np.uint16)
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, D = q.shape
    P, Hkv, ps, D2 = k_pool.shape
    assert D2 == D and ps == PAGE and v_pool.shape == k_pool.shape
    maxp = page_table.shape[1]
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    p = np.zeros((B, Hq, maxp * PAGE), dtype=np.float64) if want_p else None
    rc = lib().zfo_attention(_ptr(q), _ptr(k_pool), _ptr(v_pool), P, _ptr(page_table), maxp,
                             _ptr(seq_lens), B, Hq, Hkv, D, PAGE, float(sm_scale), _ptr(out), _ptr(lse),
                             _ptr(p) if want_p else None)
    if rc != 0:
        raise ValueError("oracle attention: page id or sequence length out of range")
    return out, lse, p


def decompress_pool(c: Compressed, num_pages: int, Hkv: int, D: int = 128) -> np.ndarray:
    """Decompress a whole paged pool back to [P][Hkv][16][D] u16."""
    return decompress(c).reshape(num_pages, Hkv, PAGE, D)


def attention_compressed(q, kc: Compressed, vc: Compressed, num_pages, Hkv, page_table, seq_lens, sm_scale):
    """Attention over a compressed cache: decompress, then fp64 attention."""
    k = decompress_pool(kc, num_pages, Hkv, q.shape[2])
    v = decompress_pool(vc, num_pages, Hkv, q.shape[2])
    return attention(q, k, v, page_table, seq_lens, sm_scale)


# ------------------------------------------------------------ FP8 E4M3 (R8)

def e4m3_decode(code: int) -> float:
    return float(lib().zfo_e4m3_decode(int(code)))


def e4m3_encode(x: float) -> int:
    return int(lib().zfo_e4m3_encode(float(x)))


def fp8_quantize(words, inv_scale: float) -> np.ndarray:
    """bf16 words -> E4M3 codes of (float)value * (float)inv_scale."""
    w = np.ascontiguousarray(words, dtype=np.uint16)
    out = np.empty(w.shape, dtype=np.uint8)
    lib().zfo_fp8_quantize(_ptr(w), w.size, float(np.float32(inv_scale)), _ptr(out))
    return out


def fp8_dequantize(codes, scale: float) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    lib().zfo_fp8_dequantize(_ptr(c), c.size, float(scale), _ptr(out))
    return out


def attention_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens, sm_scale, want_p=False):
    """fp64 paged GQA decode attention over E4M3 pools: K/V value =
    decode(code) * scale (one scale per pool).  Same returns as attention()."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_codes = np.ascontiguousarray(k_codes, dtype=np.uint8)
    v_codes = np.ascontiguousarray(v_codes, dtype=np.uint8)
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, D = q.shape
    P, Hkv, ps, D2 = k_codes.shape
    assert D2 == D and ps == PAGE and v_codes.shape == k_codes.shape
    maxp = page_table.shape[1]
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    p = np.zeros((B, Hq, maxp * PAGE), dtype=np.float64) if want_p else None
    rc = lib().zfo_attention_fp8(_ptr(q), _ptr(k_codes), _ptr(v_codes), float(k_scale), float(v_scale), P,
                                 _ptr(page_table), maxp, _ptr(seq_lens), B, Hq, Hkv, D, PAGE, float(sm_scale),
                                 _ptr(out), _ptr(lse), _ptr(p) if want_p else None)
    if rc != 0:
        raise ValueError("oracle attention: page id or sequence length out of range")
    return out, lse, p


# ------------------------------------------------------------ paged form (R9)

CHUNK = 2048          # values per (page, kv head) chunk
CHUNK_HEADER = 48     # bytes: 32 base exponents, u32 eligibility mask, 12 zero


def pack_chunk(values, n_blocks: int = 32) -> np.ndarray:
    """Header + the first n_blocks blocks of one 2048-value chunk (bytes)."""
    v = np.ascontiguousarray(values, dtype=np.uint16).reshape(-1)
    assert v.size == CHUNK and 0 <= n_blocks <= 32
    out = np.zeros(CHUNK_HEADER + 2 * CHUNK, dtype=np.uint8)
    n = lib().zfo_pack_chunk(_ptr(v), int(n_blocks), _ptr(out))
    return out[:n].copy()


def compress_paged(values) -> tuple[np.ndarray, np.ndarray]:
    """Paged form of a flat pool (length a multiple of 2048): (data bytes,
    chunk_tab u32 [num_chunks][2] = start, extent in 16-byte units)."""
    v = np.ascontiguousarray(values, dtype=np.uint16).reshape(-1)
    if v.size % CHUNK:
        raise ValueError("length must be a multiple of 2048")
    nc = v.size // CHUNK
    data = np.zeros(nc * (CHUNK_HEADER + 2 * CHUNK) + 16, dtype=np.uint8)
    tab = np.zeros((max(nc, 1), 2), dtype=np.uint32)
    units = lib().zfo_compress_paged(_ptr(v), nc, _ptr(data), _ptr(tab))
    return data[: units * UNIT].copy(), tab[:nc]


def decompress_paged(data, chunk_tab, n_blocks: int = 32) -> np.ndarray:
    """Values of the first n_blocks blocks of every chunk (the rest zero)."""
    tab = np.ascontiguousarray(chunk_tab, dtype=np.uint32)
    nc = tab.shape[0]
    d = np.ascontiguousarray(data, dtype=np.uint8)
    if d.size == 0:
        d = np.zeros(16, np.uint8)
    out = np.zeros(nc * CHUNK, dtype=np.uint16)
    lib().zfo_decompress_paged(_ptr(d), _ptr(tab), nc, int(n_blocks), _ptr(out))
    return out

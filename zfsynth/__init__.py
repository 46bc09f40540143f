"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no arithmetic of the method: it draws values, rounds fp32 to
bf16 bit patterns, and shapes the exponent spread of each 64-value block with
plain magnitude operations (it never reads a bf16 exponent field).  Whether a
block really ends up eligible is checked by the tests with the oracle.

The value recipe follows the workloads the ZipFusion summary names (Llama 3.1
8B at batch 32, "Run AI Faster With Lossless Compressed Memory") and the five
benchmark configurations: N(0,1) values times a per-channel lognormal scale,
a few K outlier channels, and an exact share of 64-value blocks whose exponent
spread is forced above 15 so that they fall back to raw storage.

Random numbers come from numpy's PCG64 (``np.random.default_rng(seed)``), so
data never depends on a GPU generator.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

PAGE = 16
HEAD_DIM = 128
BLOCK = 64
_CHUNK = 1 << 24  # values processed at a time when shaping big pools


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (round to nearest even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(w: np.ndarray) -> np.ndarray:
    return (np.asarray(w, dtype=np.uint32) << 16).view(np.float32)


_BIG = None


def _patterns():
    global _BIG
    if _BIG is None:
        f = np.array([2.0 ** 12, -(2.0 ** 12), 2.0 ** -6, -(2.0 ** -6), 0.0], dtype=np.float32)
        _BIG = to_bf16_bits(f)
    return _BIG


@dataclass
class PoolSpec:
    """How one paged K or V pool [num_pages][Hkv][16][128] is drawn."""
    num_pages: int
    Hkv: int
    sigma: float                      # lognormal(0, sigma) per-channel scale
    outlier_channels: int = 0         # channels per kv head multiplied by ...
    outlier_mult: float = 20.0        # ... this factor
    inelig: float = 0.0               # exact share of used blocks forced raw
    zero_share: float = 0.0           # of those, the share that gets an exact 0.0


def _draw_pool(rng, spec: PoolSpec) -> np.ndarray:
    """fp32 draw -> block-spread shaping -> bf16 bits (all blocks eligible).

    The per-channel scales come from ``rng``; the values are drawn in chunks
    of pages, each chunk from its own generator seeded with (a draw of
    ``rng``, chunk index), so chunks can be filled by a thread pool and the
    bytes do not depend on how many threads there are."""
    H, D = spec.Hkv, HEAD_DIM
    scale = rng.lognormal(0.0, spec.sigma, size=(H, D)).astype(np.float32)
    if spec.outlier_channels:
        for h in range(H):
            ch = rng.choice(D, size=spec.outlier_channels, replace=False)
            scale[h, ch] *= np.float32(spec.outlier_mult)
    stream = int(rng.integers(0, 2 ** 62))
    n = spec.num_pages * H * PAGE * D
    out = np.empty(n, dtype=np.uint16)
    per_page = H * PAGE * D
    pages_per_chunk = max(1, _CHUNK // per_page)
    floor_factor = np.float32(2.0 ** -14)

    def fill(ci):
        p0 = ci * pages_per_chunk
        p1 = min(spec.num_pages, p0 + pages_per_chunk)
        r = np.random.default_rng([stream, ci])
        x = r.standard_normal(size=(p1 - p0, H, PAGE, D), dtype=np.float32)
        x *= scale[None, :, None, :]
        blocks = x.reshape(-1, BLOCK)
        # Raise magnitudes below (block max) * 2^-14 to that floor: after
        # rounding every value of a block is then within 2^15 of its largest,
        # which keeps the block eligible.
        floor = np.abs(blocks).max(axis=1, keepdims=True) * floor_factor
        small = np.abs(blocks) < floor
        sign = np.where(blocks < 0, np.float32(-1.0), np.float32(1.0))
        blocks[...] = np.where(small, sign * floor, blocks)
        out[p0 * per_page: p1 * per_page] = to_bf16_bits(blocks.reshape(-1))

    n_chunks = (spec.num_pages + pages_per_chunk - 1) // pages_per_chunk
    if n_chunks <= 1:
        for ci in range(n_chunks):
            fill(ci)
    else:
        with ThreadPoolExecutor(max_workers=min(n_chunks, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out.reshape(spec.num_pages, H, PAGE, D)


def _inject(rng, pool: np.ndarray, used_blocks: np.ndarray, inelig: float, zero_share: float):
    """Force an exact share of the used blocks to an exponent spread > 15:
    either one value of 2^12 next to one of 2^-6 (spread >= 18), or one exact
    zero next to normal values.  Returns the chosen block indices."""
    flat = pool.reshape(-1)
    k = int(round(inelig * used_blocks.size))
    chosen = rng.permutation(used_blocks)[:k]
    n_zero = int(round(zero_share * k))
    big, nbig, tiny, ntiny, zero = _patterns()
    pos = rng.integers(0, BLOCK, size=(k, 2))
    pos[:, 1] = (pos[:, 0] + 1 + rng.integers(0, BLOCK - 1, size=k)) % BLOCK  # distinct
    sgn = rng.integers(0, 2, size=(k, 2))
    idx0 = chosen.astype(np.int64) * BLOCK + pos[:, 0]
    idx1 = chosen.astype(np.int64) * BLOCK + pos[:, 1]
    zsel = np.zeros(k, dtype=bool)
    zsel[:n_zero] = True
    flat[idx0[zsel]] = zero
    o = ~zsel
    flat[idx0[o]] = np.where(sgn[o, 0] == 0, big, nbig)
    flat[idx1[o]] = np.where(sgn[o, 1] == 0, tiny, ntiny)
    return np.sort(chosen)


@dataclass
class Case:
    """One decode-attention workload (all arrays are host numpy)."""
    name: str
    q: np.ndarray               # [B][Hq][128] u16 (bf16 bits)
    k_pool: np.ndarray          # [P][Hkv][16][128] u16
    v_pool: np.ndarray
    page_table: np.ndarray      # [B][max_pages] i32
    seq_lens: np.ndarray        # [B] i32
    B: int
    Hq: int
    Hkv: int
    sm_scale: float
    meta: dict = field(default_factory=dict)

    @property
    def num_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.seq_lens.size else 0

    @property
    def max_pages(self) -> int:
        return self.page_table.shape[1]


def make_case(name, *, B, Hq, Hkv, ctx, sigma, seed, inelig=0.0, zero_share=0.0,
              k_outlier_channels=0, outlier_mult=20.0, table="shuffled", pool_pages=None,
              used_pages=None) -> Case:
    """Build a decode workload.

    ctx: int (every sequence) or a sequence of per-sequence lengths.
    table: "identity" (sequence b owns a contiguous run of pages), "shuffled"
    (a seeded permutation of the pool), or "subset" (``used_pages`` distinct
    pages drawn from a pool of ``pool_pages``).
    """
    rng = np.random.default_rng(seed)
    lens = np.full(B, ctx, dtype=np.int64) if np.isscalar(ctx) else np.asarray(ctx, dtype=np.int64)
    npages = (lens + PAGE - 1) // PAGE
    total = int(npages.sum())
    maxp = max(1, int(npages.max()) if B else 1)
    if table == "subset":
        P = int(pool_pages)
        assert total <= P
        ids = rng.choice(P, size=total, replace=False)
    else:
        P = total if pool_pages is None else int(pool_pages)
        ids = np.arange(total) if table == "identity" else rng.permutation(P)[:total]
    page_table = np.zeros((B, maxp), dtype=np.int32)
    pos = 0
    for b in range(B):
        page_table[b, : npages[b]] = ids[pos: pos + npages[b]]
        pos += npages[b]

    kspec = PoolSpec(P, Hkv, sigma, k_outlier_channels, outlier_mult, inelig, zero_share)
    vspec = PoolSpec(P, Hkv, sigma, 0, outlier_mult, inelig, zero_share)
    k_pool = _draw_pool(rng, kspec)
    v_pool = _draw_pool(rng, vspec)

    # Token slots past a sequence's end (in its last page) hold zeros.
    used_mask = np.zeros((P, PAGE), dtype=bool)
    for b in range(B):
        for p in range(npages[b]):
            n = min(PAGE, int(lens[b]) - p * PAGE)
            used_mask[page_table[b, p], :n] = True
    if table == "subset" or pool_pages is not None:
        # every page of an explicitly sized pool is live data
        used_mask[:] = True
    for pool in (k_pool, v_pool):
        pool.transpose(0, 2, 1, 3)[~used_mask] = 0
    # used blocks: [P][Hkv][16 tokens][2 blocks]
    ub = np.broadcast_to(used_mask[:, None, :, None], (P, Hkv, PAGE, HEAD_DIM // BLOCK))
    used_blocks = np.flatnonzero(ub.reshape(-1))
    chosen = {}
    for nm, pool in (("k", k_pool), ("v", v_pool)):
        chosen[nm] = _inject(rng, pool, used_blocks, inelig, zero_share)

    q = to_bf16_bits(rng.standard_normal(size=(B, Hq, HEAD_DIM), dtype=np.float32))
    meta = dict(seed=seed, sigma=sigma, inelig_target=inelig, zero_share=zero_share,
                k_outlier_channels=k_outlier_channels, used_blocks=int(used_blocks.size),
                forced_raw_k=int(chosen["k"].size), forced_raw_v=int(chosen["v"].size), table=table)
    return Case(name, q, k_pool, v_pool, page_table, lens.astype(np.int32), B, Hq, Hkv,
                1.0 / np.sqrt(HEAD_DIM), meta)


# The five benchmark workloads.  Index i is the i-th configuration of the
# benchmark list (0: tiny, 1: Llama-3.1-8B shape, 2: long context, 3: ragged
# serving batch, 4: codec pool + extreme context).
def config(i: int, *, scale_ctx: float = 1.0, inelig: float | None = None) -> Case:
    """Workload i at full size (scale_ctx < 1 shrinks the contexts for tests)."""
    def c(x):
        return max(PAGE, int(x * scale_ctx))
    if i == 0:
        return make_case("tiny: B=2 Hq=4 Hkv=1 ctx=512", B=2, Hq=4, Hkv=1, ctx=c(512), sigma=0.5,
                         inelig=0.02 if inelig is None else inelig, table="identity", seed=1000)
    if i == 1:
        return make_case("llama-3.1-8b: B=32 Hq=32 Hkv=8 ctx=4096", B=32, Hq=32, Hkv=8, ctx=c(4096),
                         sigma=0.7, k_outlier_channels=3, inelig=0.05 if inelig is None else inelig,
                         table="shuffled", seed=1001)
    if i == 2:
        # "same value distribution as config 1": read with 1-based numbering,
        # i.e. the tiny workload's lognormal(0, 0.5) and 2% raw blocks.
        return make_case("long: B=16 Hq=32 Hkv=8 ctx=32768", B=16, Hq=32, Hkv=8, ctx=c(32768), sigma=0.5,
                         inelig=0.02 if inelig is None else inelig, table="shuffled", seed=1002)
    if i == 3:
        rng = np.random.default_rng(31003)
        lens = rng.integers(1024, 16384 + 1, size=64)
        lens = np.maximum(1, (lens * scale_ctx).astype(np.int64))
        return make_case("ragged: B=64 Hq=32 Hkv=8 ctx~U[1024,16384]", B=64, Hq=32, Hkv=8, ctx=lens,
                         sigma=0.7, inelig=0.10 if inelig is None else inelig, zero_share=0.5,
                         table="shuffled", seed=1003)
    if i == 4:
        pool = max(2 * c(131072) * 4 // PAGE, int(65536 * scale_ctx))
        return make_case("extreme: B=4 Hq=32 Hkv=8 ctx=131072, 65536-page pool", B=4, Hq=32, Hkv=8,
                         ctx=c(131072), sigma=1.0, inelig=0.10 if inelig is None else inelig,
                         table="subset", pool_pages=pool, seed=1004)
    raise ValueError(i)


def codec_pool_sweep(fracs=(0.0, 0.10, 0.50, 1.0), num_pages: int = 65536, Hkv: int = 8, seed: int = 1004):
    """The codec-only workload at several raw-block shares: the K and V pools
    are drawn once (all blocks eligible) and each share is injected into a
    copy, with a generator seeded from (seed, share).  Yields (share, k, v)."""
    rng = np.random.default_rng(seed)
    spec = PoolSpec(num_pages, Hkv, 1.0)
    k0 = _draw_pool(rng, spec)
    v0 = _draw_pool(rng, spec)
    nb = k0.size // BLOCK
    allb = np.arange(nb, dtype=np.int64)
    for f in fracs:
        r = np.random.default_rng([seed, int(round(f * 1000))])
        k = k0.copy()
        v = v0.copy()
        _inject(r, k, allb, f, 0.0)
        _inject(r, v, allb, f, 0.0)
        yield f, k, v


def codec_pool(num_pages: int = 65536, Hkv: int = 8, inelig: float = 0.10, seed: int = 1004):
    """The codec-only workload: K and V pools of N(0,1) x lognormal(0,1)
    channel scales with an exact share of raw blocks (4 GiB at full size)."""
    rng = np.random.default_rng(seed)
    spec = PoolSpec(num_pages, Hkv, 1.0)
    k = _draw_pool(rng, spec)
    v = _draw_pool(rng, spec)
    nb = k.size // BLOCK
    allb = np.arange(nb, dtype=np.int64)
    _inject(rng, k, allb, inelig, 0.0)
    _inject(rng, v, allb, inelig, 0.0)
    return k, v

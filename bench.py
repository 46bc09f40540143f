"""Benchmark: fused decode attention over a compressed paged BF16 KV cache.

Default workload: Llama-3.1-8B-shaped decode attention, one layer: batch 32,
32 query / 8 KV heads, head_dim 128, 4096 tokens per sequence, 16-token pages
in a shuffled page table, ~5% raw blocks (the ZipFusion summary's "Llama three
point one eight-B at batch size thirty-two").

One step = one call of zf_decode_attention over the whole batch: one launch
of the fused attention kernel, whose last warp per sequence/head merges the
split results (the split counters are reset inside the kernel).  ``value`` is
compressed-KV GB/s (the bytes the method must read, divided by the device time
of a step); tokens/s at 32 layers, the raw-BF16 twin, the codec throughput,
the other benchmark workloads (``per_config``) and the capacity model are
extra fields.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (the path has no exchange step), one rank
per GPU; time is the max over ranks and value the sum of all ranks' bytes.
``--impl reference`` times the CPU oracle (decompress + fp64 attention) on a
bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
LAYERS = 32                      # Llama-3.1-8B depth, for tokens/s
METRIC = "compressed decode-attn HBM GB/s vs ~8 TB/s peak; tokens/s at B=32, ctx 4k"
KERNEL = "decode_attn_kernel<kFmtCompressed> (split merge fused in)"
META_BYTES_PER_CHUNK = 32 + 4 + 4    # base exponents, eligibility word, offset entry


# ------------------------------------------------------------- host helpers

def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The files the decode kernel is compiled from: its translation unit and the
# two device headers.  A traffic record stays valid while these are unchanged.
KERNEL_SOURCES = ("zf_attention.cu", "zf_device.cuh", "zf_internal.h")


def source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "decode_attention_zipfusion_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None, None
    if d.get("source_hash") != source_hash():
        return None, d.get("source_hash")
    return d, d.get("source_hash")


def chunk_bytes_from_elig(elig_words: np.ndarray) -> np.ndarray:
    """Payload bytes of each (page, kv head) chunk: 96 B per eligible block,
    128 B per raw block, 32 blocks per chunk (one eligibility word)."""
    pop = np.unpackbits(elig_words.view(np.uint8)).reshape(-1, 32).sum(1)
    return (32 * 128 - 32 * pop).astype(np.int64)


def algorithmic_bytes(case, k_elig, v_elig):
    """Bytes the compressed decode step must move: for every (sequence, kv
    head, page) of the batch its K and V payload extents plus per-chunk
    metadata, plus q, out, the page-table entries and seq_lens."""
    kb = chunk_bytes_from_elig(k_elig)
    vb = chunk_bytes_from_elig(v_elig)
    comp = 0
    raw_equiv = 0
    pages = 0
    for b in range(case.B):
        n = (int(case.seq_lens[b]) + 15) // 16
        ids = case.page_table[b, :n].astype(np.int64)
        chunks = (ids[:, None] * case.Hkv + np.arange(case.Hkv)[None, :]).reshape(-1)
        comp += int(kb[chunks].sum() + vb[chunks].sum()) + 2 * META_BYTES_PER_CHUNK * chunks.size
        raw_equiv += 2 * 4096 * chunks.size
        pages += n
    qo = 2 * case.B * case.Hq * 128 * 2
    small = 4 * pages + 4 * case.B
    return comp + qo + small, raw_equiv + qo + small, comp


class NvmlSampler:
    """SM clock, power and clock-event (throttle) reasons, sampled through NVML
    every ~0.5 ms by a host thread while the block runs (the timed region
    itself: it is only milliseconds long, too short for nvidia-smi's 20 ms
    sampling)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, index: int, period_s: float = 0.0005):
        self.index = index
        self.period = period_s
        self.rows = []  # (sm_mhz, power_w, reasons bitmask, host time)
        self.stop = threading.Event()
        self.thread = None
        self.nv = None
        self.max_mhz = None
        self.t_start = None  # the timed region, marked by the caller (host time)
        self.t_end = None

    def mark_start(self):
        self.t_start = time.perf_counter()

    def mark_end(self):
        self.t_end = time.perf_counter()

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.sample()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:
            self.nv = None
        return self

    def sample(self):
        nv = self.nv
        try:
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.rows.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                          nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0, int(reasons), time.perf_counter()))

    def _run(self):
        while not self.stop.is_set():
            try:
                self.sample()
            except Exception:
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        if self.nv is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self.sample()
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def window(self):
        """The samples of the timed region: those taken inside it, plus the
        last one before it and the first one after it (its edges); all
        samples when the region was not marked."""
        if self.t_start is None or self.t_end is None:
            return list(self.rows), len(self.rows)
        inside = [r for r in self.rows if self.t_start <= r[3] <= self.t_end]
        before = [r for r in self.rows if r[3] < self.t_start]
        after = [r for r in self.rows if r[3] > self.t_end]
        return before[-1:] + inside + after[:1], len(inside)

    def summary(self):
        rows, n_inside = self.window()
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"], "samples": 0,
                    "source": "NVML (unavailable)"}
        nv = self.nv
        names = sorted({n for r in rows for n, attr in self.REASONS
                        if hasattr(nv, attr) and r[2] & getattr(nv, attr)})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(r[0] for r in rows), "power_w_max": round(max(r[1] for r in rows), 1),
                "reasons": names, "samples": len(rows), "samples_in_timed_region": n_inside,
                "source": "NVML, every ~0.5 ms by a host thread started before the warm-up; the samples "
                          "inside the timed region and one at each of its edges"}


# ------------------------------------------------------- distributed plumbing

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(time_s: float, units: float, world: int):
    """Max of the timed region over ranks, sum of the work: whole-job rate."""
    if world <= 1:
        return time_s, units
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([time_s], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local):
    import torch
    import decode_attention_zipfusion_b200 as zf
    import zfsynth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    case = zfsynth.config(args.config)

    def up16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q = up16(case.q)
    k = up16(case.k_pool)
    v = up16(case.v_pool)
    pt = torch.from_numpy(case.page_table).to(dev)
    sl = torch.from_numpy(case.seq_lens).to(dev)
    kz = zf.compress(k)
    vz = zf.compress(v)
    torch.cuda.synchronize()
    ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, case.max_seq_len, dev)
    out = torch.empty((case.B, case.Hq, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((case.B, case.Hq), dtype=torch.float32, device=dev)
    k_elig = kz.elig.cpu().numpy().view(np.uint32)
    v_elig = vz.elig.cpu().numpy().view(np.uint32)
    alg_bytes, raw_equiv_bytes, kv_comp_bytes = algorithmic_bytes(case, k_elig, v_elig)
    n_raw = int(np.unpackbits(k_elig.view(np.uint8)).size - np.unpackbits(k_elig.view(np.uint8)).sum())

    def step_comp():
        zf.decode_attention(q, kz, vz, pt, sl, case.max_seq_len, num_pages=case.num_pages, Hkv=case.Hkv,
                            sm_scale=case.sm_scale, out=out, lse=lse, ws=ws)

    def step_raw():
        zf.decode_attention_raw(q, k, v, pt, sl, case.max_seq_len, sm_scale=case.sm_scale, out=out, lse=lse,
                                ws=ws)

    def timed(fn, steps, warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        s = torch.cuda.current_stream()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        barrier(world)
        return e0.elapsed_time(e1) / 1e3  # seconds

    # correctness guard: compressed and raw kernels agree bitwise
    step_comp()
    o_c = out.clone()
    l_c = lse.clone()
    step_raw()
    torch.cuda.synchronize()
    bitwise_equal = bool(torch.equal(o_c.view(torch.int16), out.view(torch.int16)) and torch.equal(l_c, lse))
    dev_err = zf.get_device_error(ws)

    # main timed region: W warm-up steps, then exactly K timed steps, with
    # the clocks sampled through NVML while the K steps run (the sampler starts
    # before the warm-up, so its start-up does not leave the GPU idle just
    # before the timed region)
    with NvmlSampler(local) as clk:
        for _ in range(args.warmup):
            step_comp()
        torch.cuda.synchronize()
        clk.mark_start()
        t = timed(step_comp, args.steps, 0)
        clk.mark_end()
    t_max, bytes_all = aggregate(t, float(alg_bytes) * args.steps, world)
    ms_per_step = t_max / args.steps * 1e3
    value = bytes_all / t_max / 1e9

    # per-launch distribution: one event between consecutive launches of the
    # same back-to-back loop (the stream never idles, so each gap is one launch)
    n_pl = max(50, min(500, args.steps))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_pl + 1)]
    torch.cuda.synchronize()
    evs[0].record()
    for i in range(n_pl):
        step_comp()
        evs[i + 1].record()
    torch.cuda.synchronize()
    per_launch = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(n_pl))

    def pct(p):
        return round(per_launch[min(n_pl - 1, int(p * n_pl))], 5)

    # extras (rank-local, not part of the headline)
    t_raw = timed(step_raw, max(10, args.steps // 4), 3)
    ms_raw = t_raw / max(10, args.steps // 4) * 1e3
    ms_comp_local = t / args.steps * 1e3

    # codec throughput on the same pools (K and V, compress then decompress)
    ncodec = max(5, min(50, args.steps // 10))
    kws = torch.empty(zf.lib().zf_compress_workspace_size(k.numel()), dtype=torch.uint8, device=dev)
    kz2 = zf.CompressedKV.empty(k.numel(), dev)
    dec = torch.empty(k.numel(), dtype=torch.bfloat16, device=dev)
    t_c = timed(lambda: zf.compress(k, out=kz2, ws=kws), ncodec, 3) / ncodec
    t_d = timed(lambda: zf.decompress(kz2, out=dec), ncodec, 3) / ncodec
    comp_units = kz2.units()
    nb = k.numel() // 64
    codec_out_bytes = comp_units * 16 + 4 * (nb + 1) + nb + 4 * ((nb + 31) // 32)
    compress_gbs = (2 * k.numel() + codec_out_bytes) / t_c / 1e9
    decompress_gbs = (2 * k.numel() + codec_out_bytes) / t_d / 1e9

    # end to end through the public API with host buffers
    q_h = q.cpu().pin_memory()
    pt_h = pt.cpu().pin_memory()
    sl_h = sl.cpu().pin_memory()
    out_h = torch.empty_like(out, device="cpu").pin_memory()
    ws_h = zf.decode_host_workspace(case.B, case.Hq, case.Hkv, pt.shape[1], case.max_seq_len, dev)

    def step_e2e():
        zf.decode_attention_host(q_h, kz, vz, pt_h, sl_h, case.max_seq_len, num_pages=case.num_pages,
                                 Hkv=case.Hkv, sm_scale=case.sm_scale, out=out_h, ws=ws_h)
        torch.cuda.current_stream().synchronize()

    ne2e = max(10, args.steps // 4)
    t_e2e = timed(step_e2e, ne2e, 3)
    t_e2e_max, e2e_bytes = aggregate(t_e2e, float(alg_bytes) * ne2e, world)
    h2d = q_h.numel() * 2 + pt_h.numel() * 4 + sl_h.numel() * 4
    d2h = out_h.numel() * 2

    # The same host-buffer call captured once in a CUDA graph (the copies in,
    # the kernel, the copy out) and replayed each step, with the same host
    # sync: what a serving loop that replays a captured step pays.
    # Rank-local (no collective, so a failed capture cannot desynchronise ranks).
    try:
        def host_call():
            zf.decode_attention_host(q_h, kz, vz, pt_h, sl_h, case.max_seq_len, num_pages=case.num_pages,
                                     Hkv=case.Hkv, sm_scale=case.sm_scale, out=out_h, ws=ws_h)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            host_call()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            host_call()

        def step_graph():
            graph.replay()
            torch.cuda.current_stream().synchronize()
        t_graph = timed_plain(step_graph, ne2e, 3)
        e2e_graph = {"value": round(float(alg_bytes) * ne2e / t_graph / 1e9, 2), "unit": "GB/s",
                     "ms_per_step": round(t_graph / ne2e * 1e3, 5),
                     "note": "rank-local; the zf_decode_attention_host call captured once in a CUDA graph and "
                             "replayed per step, with the same copies and host sync"}
        del graph
    except Exception as ex:  # report, do not fail the bench line
        e2e_graph = {"unavailable": f"{type(ex).__name__}: {str(ex)[:160]}"}

    # Where an end-to-end step's time goes: the same pieces as separate
    # stream operations, each bracketed by events (the host-buffer call does
    # them in one call), plus the host's wall time per step around them.
    q_d2, pt_d2, sl_d2 = torch.empty_like(q), torch.empty_like(pt), torch.empty_like(sl)
    nbd = max(10, min(200, args.steps))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nbd)]
    walls = []
    for i in range(nbd + 3):
        w0 = time.perf_counter()
        e = ev[i - 3] if i >= 3 else None
        if e:
            e[0].record()
        q_d2.copy_(q_h, non_blocking=True)
        pt_d2.copy_(pt_h, non_blocking=True)
        sl_d2.copy_(sl_h, non_blocking=True)
        if e:
            e[1].record()
        zf.decode_attention(q_d2, kz, vz, pt_d2, sl_d2, case.max_seq_len, num_pages=case.num_pages, Hkv=case.Hkv,
                            sm_scale=case.sm_scale, out=out, ws=ws)
        if e:
            e[2].record()
        out_h.copy_(out, non_blocking=True)
        if e:
            e[3].record()
        torch.cuda.current_stream().synchronize()
        if e:
            walls.append(time.perf_counter() - w0)
    med = lambda xs: float(np.median(xs))  # noqa: E731
    bd_h2d = med([a[0].elapsed_time(a[1]) for a in ev]) * 1e3
    bd_kernel = med([a[1].elapsed_time(a[2]) for a in ev]) * 1e3
    bd_d2h = med([a[2].elapsed_time(a[3]) for a in ev]) * 1e3
    bd_wall = med(walls) * 1e6
    e2e_breakdown = {"h2d_us": round(bd_h2d, 2), "kernel_us": round(bd_kernel, 2), "d2h_us": round(bd_d2h, 2),
                     "device_total_us": round(bd_h2d + bd_kernel + bd_d2h, 2), "host_wall_us": round(bd_wall, 2),
                     "host_only_us": round(bd_wall - (bd_h2d + bd_kernel + bd_d2h), 2),
                     "e2e_step_us": round(t_e2e / ne2e * 1e6, 2),
                     "note": "medians over steps of the same pieces as separate stream operations (pinned copies, "
                             "the kernel, the copy back, a host sync); host_only = wall time per step minus the "
                             "device time of its pieces (Python and ctypes calls, launch and sync latency)"}
    del q_d2, pt_d2, sl_d2

    # one call on an idle GPU (no back-to-back overlap with a previous call)
    iso = []
    for _ in range(20):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        step_comp()
        e1.record()
        torch.cuda.synchronize()
        iso.append(e0.elapsed_time(e1))
    isolated_ms = float(np.median(iso))

    # the lossy comparator of the method: the same attention over an FP8 E4M3
    # cache (one scale per pool from the pool's max magnitude)
    def pool_scale(bits):
        return max(float(np.abs((bits.astype(np.uint32) << 16).view(np.float32)).max()), 1e-30) / 448.0
    ks8, vs8 = pool_scale(case.k_pool), pool_scale(case.v_pool)
    k8 = zf.fp8_quantize(k, ks8)
    v8 = zf.fp8_quantize(v, vs8)
    out8 = torch.empty_like(out)

    def step_fp8():
        zf.decode_attention_fp8(q, k8, v8, ks8, vs8, pt, sl, case.max_seq_len, sm_scale=case.sm_scale, out=out8,
                                lse=lse, ws=ws)

    n8 = max(10, args.steps // 4)
    ms_fp8 = timed(step_fp8, n8, 3) / n8 * 1e3
    step_raw()
    step_fp8()
    torch.cuda.synchronize()
    exact = out.float()
    fp8_err = float(((out8.float() - exact).abs() / exact.abs().clamp_min(1.0)).max())
    fp8_bytes = raw_equiv_bytes - (raw_equiv_bytes - (alg_bytes - kv_comp_bytes)) // 2

    # the paged form (one extent per chunk, 8 B of table per chunk): decode
    # speed, storage, and the cost of appending each step's tokens
    pk, pv = zf.compress_paged(k), zf.compress_paged(v)
    out_pg = torch.empty_like(out)

    def step_paged():
        zf.decode_attention_paged(q, pk, pv, pt, sl, case.max_seq_len, num_pages=case.num_pages, Hkv=case.Hkv,
                                  sm_scale=case.sm_scale, out=out_pg, lse=lse, ws=ws)

    npg = max(10, args.steps // 4)
    ms_paged = timed(step_paged, npg, 3) / npg * 1e3
    step_raw()
    step_paged()
    torch.cuda.synchronize()
    paged_equal = bool(torch.equal(out_pg.view(torch.int16), out.view(torch.int16)))
    n_chunks = case.num_pages * case.Hkv
    paged_store = (pk.units() + pv.units()) * 16 + 2 * 8 * n_chunks
    flat_store = 2 * (kz.units() * 16 + 4 * (k.numel() // 64 + 1) + k.numel() // 64 + 4 * (k.numel() // 2048))
    raw_store = 2 * 2 * k.numel()
    # append: the first T tokens of every sequence, K and V, token by token
    T = 64
    pt_cpu = case.page_table
    tok_pages = torch.from_numpy(np.repeat(pt_cpu[:, :T // 16], 16, axis=1)).to(dev).long()  # page of token t
    kv_steps = [(k[tok_pages[:, t], :, t % 16, :].contiguous(), v[tok_pages[:, t], :, t % 16, :].contiguous())
                for t in range(T)]
    pos_steps = [torch.full((case.B,), t, dtype=torch.int32, device=dev) for t in range(T)]

    def build():
        aps = [zf.AppendPool(n_chunks, case.B, case.Hkv, packed_bytes=case.B * (T // 16) * case.Hkv * 4144,
                             device=dev) for _ in range(2)]
        return aps

    def time_appends(fused):
        aps = build()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for t in range(T):
            if fused:   # K and V in one launch
                zf.append_kv(aps[0], aps[1], kv_steps[t][0], kv_steps[t][1], pt, pos_steps[t])
            else:
                aps[0].append(kv_steps[t][0], pt, pos_steps[t])
                aps[1].append(kv_steps[t][1], pt, pos_steps[t])
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / T * 1e3, int(aps[0].err.item()) | int(aps[1].err.item())

    us_append_two, err_two = time_appends(False)
    us_append, err_one = time_appends(True)
    append_err = err_two | err_one

    peak, peak_kind = measured_peak()
    achieved = alg_bytes / (ms_comp_local / 1e3) / 1e9
    traffic_rec, _ = recorded_traffic()
    traffic = None
    if traffic_rec is not None and traffic_rec.get("workload") == case.name:
        traffic = traffic_rec.get("dram_bytes_per_launch")

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; N(0,1) x lognormal channel scales, K outlier channels, exact raw-block share)",
        "config": {"workload": case.name, "global_batch": case.B * world, "seq_len": case.max_seq_len,
                   "Hq": case.Hq, "Hkv": case.Hkv, "head_dim": 128, "page_tokens": 16,
                   "raw_block_share": round(n_raw / max(1, k_elig.size * 32), 4),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2 ({kv_comp_bytes / 1e6:.1f} MB compressed cache vs 126 MB L2), "
                         f"no flush"},
        "tokens_per_s": round(case.B * world / (ms_per_step / 1e3) / LAYERS, 1),
        "tokens_per_s_per_layer": round(case.B * world / (ms_per_step / 1e3), 1),
        "uncompressed_equiv_gbs": round(raw_equiv_bytes * world / (t_max / args.steps) / 1e9, 2),
        "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
        "compressed_kv_bytes": int(kv_comp_bytes),
        "raw_kv_bytes": int(raw_equiv_bytes - (alg_bytes - kv_comp_bytes)),
        "raw_twin": {"ms_per_step": round(ms_raw, 5),
                     "gbs": round(raw_equiv_bytes / (ms_raw / 1e3) / 1e9, 2),
                     "speedup_compressed_vs_raw": round(ms_raw / ms_comp_local, 4),
                     "bitwise_equal_outputs": bitwise_equal},
        "paged_format": {"ms_per_step": round(ms_paged, 5),
                         "speedup_vs_flat_compressed": round(ms_comp_local / ms_paged, 4),
                         "bitwise_equal_to_raw": paged_equal,
                         "storage_ratio": round(paged_store / raw_store, 4),
                         "flat_storage_ratio": round(flat_store / raw_store, 4),
                         "append_us_per_step_kv": round(us_append, 3),
                         "append_us_per_step_kv_two_launches": round(us_append_two, 3),
                         "append_device_error": append_err,
                         "append_note": f"one token per sequence, K and V in one launch (zf_append_paged_kv; "
                                        f"two_launches: one zf_append_paged call per pool), first {T} tokens, "
                                        f"from Python"},
        "fp8_comparator": {"ms_per_step": round(ms_fp8, 5), "kv_bytes": int((raw_equiv_bytes - (alg_bytes - kv_comp_bytes)) // 2),
                           "gbs": round(fp8_bytes / (ms_fp8 / 1e3) / 1e9, 2),
                           "speedup_vs_raw": round(ms_raw / ms_fp8, 4),
                           "speedup_vs_compressed": round(ms_comp_local / ms_fp8, 4),
                           "max_rel_err_vs_exact": round(fp8_err, 5),
                           "note": "E4M3 codes, one scale per pool; lossy, unlike the compressed cache "
                                   "(bitwise equal to the exact result)"},
        "codec": {"pool": "K pool of the workload", "values": int(k.numel()),
                  "compress_gbs": round(compress_gbs, 2), "decompress_gbs": round(decompress_gbs, 2),
                  "compress_ms": round(t_c * 1e3, 4), "decompress_ms": round(t_d * 1e3, 4)},
        "device_error_word": dev_err,
        "gpu": torch.cuda.get_device_name(dev),
        "kernel_source_hash": source_hash(),
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "traffic": traffic, "kernel": KERNEL,
                     "bytes_per_launch": int(alg_bytes),
                     "note": "duration = one call: one fused attention kernel launch (CUDA events on the launch stream)"},
        "e2e": {"value": round(e2e_bytes / t_e2e_max / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "one zf_decode_attention_host call per step (pinned H2D of q/page_table/seq_lens, the "
                        "fused kernel, D2H of out) and a host sync; the compressed KV cache is device-resident "
                        "state"},
        "e2e_graph": e2e_graph,
        "clocks": clk.summary(),
        "per_launch_ms": {"p10": pct(0.10), "p50": pct(0.50), "p90": pct(0.90), "launches": n_pl,
                          "isolated_call_ms": round(isolated_ms, 5),
                          "note": "rank-local, after the timed region; CUDA events between consecutive launches; "
                                  "isolated_call_ms: median of 20 single calls, each on an idle GPU, events recorded "
                                  "around the Python call (so it includes the host launch path)"},
        "e2e_breakdown": e2e_breakdown,
    }
    if world == 1 and not args.no_per_config:
        # every benchmark workload, then the codec sweep and the capacity
        # model (rank-local side measurements; the headline stays config 1)
        del kz2, dec, kws, k8, v8, pk, pv, kv_steps
        torch.cuda.empty_cache()
        per = {}
        for i in range(5):
            if i == args.config:
                per[str(i)] = {"workload": case.name, "ms_per_step": line["ms_per_step"],
                               "raw_twin_ms_per_step": line["raw_twin"]["ms_per_step"],
                               "compressed_kv_gbs": line["value"],
                               "uncompressed_equiv_gbs": line["uncompressed_equiv_gbs"],
                               "frac_of_measured_peak": round(line["value"] / peak, 4),
                               "frac_of_nominal_8tbs": round(line["value"] / NOMINAL_HBM_GBS, 4),
                               "tokens_per_s": line["tokens_per_s"],
                               "tokens_per_s_per_layer": line["tokens_per_s_per_layer"],
                               "speedup_compressed_vs_raw": line["raw_twin"]["speedup_compressed_vs_raw"],
                               "bitwise_equal_to_raw_twin": bitwise_equal, "device_error_word": dev_err,
                               "note": "the headline measurement above"}
            else:
                per[str(i)] = measure_workload(i, args.steps, dev, peak)
        per["codec_sweep_4gib"] = measure_codec_sweep(args.steps, dev)
        per["capacity_80gb"] = measure_capacity(args.kv_budget_gb, args.steps, dev)
        line["per_config"] = per
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ oracle timing

def oracle_pools(case):
    """The oracle's own compressed K/V pools (preparation, not timed)."""
    import oracle
    return oracle.compress(case.k_pool.reshape(-1)), oracle.compress(case.v_pool.reshape(-1))


def oracle_sample(case, seqs, pools, threads: int = 1):
    """Time the oracle's decode (decompress the sampled sequences' chunks,
    fp64 attention) for a subset of sequences; returns (seconds, bytes).
    With threads > 1 the sequences are shared out over a thread pool (the
    oracle's C calls release the GIL); the oracle itself is unchanged."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    kc, vc = pools
    k_dec = np.zeros_like(case.k_pool)
    v_dec = np.zeros_like(case.v_pool)

    def one(b):
        kb = 0
        n = (int(case.seq_lens[b]) + 15) // 16
        for pid in case.page_table[b, :n]:
            c0 = int(pid) * case.Hkv
            i0, i1 = c0 * 32, (c0 + case.Hkv) * 32
            k_dec[pid] = oracle.decompress(kc, i0, i1).reshape(case.Hkv, 16, 128)
            v_dec[pid] = oracle.decompress(vc, i0, i1).reshape(case.Hkv, 16, 128)
            kb += int(kc.offs[i1] - kc.offs[i0] + vc.offs[i1] - vc.offs[i0]) * 16
            kb += 2 * 40 * case.Hkv
        sel = slice(int(b), int(b) + 1)
        oracle.attention(case.q[sel], k_dec, v_dec, case.page_table[sel], case.seq_lens[sel], case.sm_scale)
        return kb

    t0 = time.perf_counter()
    if threads <= 1:
        kb = sum(one(b) for b in seqs)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            kb = sum(ex.map(one, list(seqs)))
    return time.perf_counter() - t0, kb


def host_cpu():
    """The host's CPU model (from /proc/cpuinfo) and logical core count."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_cpus": os.cpu_count()}


def cpu_baseline(case, budget_s=20.0):
    """The oracle on the host cores: all of them (a thread pool over
    sequences) and one, each on a bounded sample of the workload."""
    pools = oracle_pools(case)
    cores = os.cpu_count() or 1
    res = {}
    t_seq, _ = oracle_sample(case, np.array([0]), pools)  # calibration: one sequence, one thread
    for name, threads in (("all", cores), ("one", 1)):
        # as many sequences as fit half the budget; the whole batch again
        # while it still fits
        per = t_seq / min(threads, case.B)
        n = int(max(1, min(case.B, 0.5 * budget_s / max(per, 1e-3))))
        reps = max(1, min(20, int(0.5 * budget_s / max(per * n, 1e-3)))) if n == case.B else 1
        t = kb = 0
        for _ in range(reps):
            dt, db = oracle_sample(case, np.arange(n), pools, threads=threads)
            t += dt
            kb += db
        res[name] = (n, reps, t, kb, threads)
    n, reps, t, kb, threads = res["all"]
    n1, reps1, t1, kb1, _ = res["one"]
    return {"value": round(kb / t / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {case.B} sequences x {reps} (all {case.Hq} heads, {case.max_seq_len} tokens each): "
                      f"plain C decompress of their K/V chunks + fp64 attention, a thread pool of {threads} over "
                      f"sequences, {t:.2f} s",
            "single_core": {"value": round(kb1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "sample": f"{n1} of {case.B} sequences x {reps1}, one thread, {t1:.2f} s"},
            **host_cpu()}


def run_reference(args, world, rank):
    if rank != 0:
        return
    import zfsynth
    case = zfsynth.config(args.config)
    budget = 150.0
    cores = os.cpu_count() or 1
    pools = oracle_pools(case)
    per_seq, _ = oracle_sample(case, np.array([0]), pools)
    per_seq /= min(cores, case.B)
    n = int(max(1, min(case.B, budget / (args.steps + args.warmup) / max(per_seq, 1e-3))))
    seqs_all = np.arange(case.B)
    for i in range(args.warmup):
        oracle_sample(case, np.roll(seqs_all, -i * n)[:n], pools, threads=cores)
    tot_t = 0.0
    tot_b = 0
    for i in range(args.steps):
        t, kb = oracle_sample(case, np.roll(seqs_all, -i * n)[:n], pools, threads=cores)
        tot_t += t
        tot_b += kb
    value = tot_b / tot_t / 1e9
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": case.name, "global_batch": case.B, "seq_len": case.max_seq_len},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} of {case.B} sequences per step (plain C decompress + fp64 "
                                       f"attention, a thread pool of {cores} over sequences)", **host_cpu()},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def capacity_plan(budget_bytes: float, ratio: float, layers: int = LAYERS, Hkv: int = 8, ctx: int = 4096,
                  head_dim: int = 128):
    """Conversations of `ctx` tokens whose K and V caches (all `layers`) fit
    `budget_bytes`: raw BF16, and compressed at `ratio` (compressed bytes incl.
    metadata over raw bytes).  Returns (per-conversation raw bytes, B_raw,
    B_compressed)."""
    per_conv = layers * 2 * Hkv * ctx * head_dim * 2
    b_raw = int(budget_bytes // per_conv)
    b_comp = int(budget_bytes // (per_conv * ratio))
    return per_conv, b_raw, b_comp


def measure_capacity(kv_budget_gb: float, steps: int, dev):
    """'More Conversations per GPU': the Llama-3.1-8B shape (32 layers, 8 kv
    heads, 4096-token conversations) under a fixed KV budget.  The compression
    ratio is measured on the workload's own pools; then one layer's decode
    attention is timed at the raw batch (raw kernel) and at the compressed
    batch (compressed kernel)."""
    import torch
    import decode_attention_zipfusion_b200 as zf
    import zfsynth
    budget = kv_budget_gb * 1e9
    # ratio measured on the Llama-3.1-8B workload's distribution
    probe = zfsynth.config(1)
    comp_bytes = 0
    raw_bytes = 0
    for pool in (probe.k_pool, probe.v_pool):
        x = torch.from_numpy(np.ascontiguousarray(pool).reshape(-1).view(np.int16)).to(dev).view(torch.bfloat16)
        z = zf.compress(x)
        nb = x.numel() // 64
        comp_bytes += z.units() * 16 + 4 * (nb + 1) + nb + 4 * ((nb + 31) // 32)
        raw_bytes += 2 * x.numel()
        del x, z
    del probe
    ratio = comp_bytes / raw_bytes
    per_conv, b_raw, b_comp = capacity_plan(budget, ratio)
    case = zfsynth.make_case(f"capacity: B={b_comp} Hq=32 Hkv=8 ctx=4096", B=b_comp, Hq=32, Hkv=8, ctx=4096,
                             sigma=0.7, k_outlier_channels=3, inelig=0.05, table="shuffled", seed=1001)

    def up16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = up16(case.q), up16(case.k_pool), up16(case.v_pool)
    pt = torch.from_numpy(case.page_table).to(dev)
    sl = torch.from_numpy(case.seq_lens).to(dev)
    kz, vz = zf.compress(k), zf.compress(v)
    ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, case.max_seq_len, dev)
    n = max(10, steps)
    t_comp = timed_plain(lambda: zf.decode_attention(q, kz, vz, pt, sl, case.max_seq_len, num_pages=case.num_pages,
                                                     Hkv=case.Hkv, sm_scale=case.sm_scale, ws=ws), n, 3) / n
    # the raw cache at its own (smaller) batch: the first b_raw conversations
    q_r, pt_r, sl_r = q[:b_raw].contiguous(), pt[:b_raw].contiguous(), sl[:b_raw].contiguous()
    t_raw = timed_plain(lambda: zf.decode_attention_raw(q_r, k, v, pt_r, sl_r, case.max_seq_len,
                                                        sm_scale=case.sm_scale, ws=ws), n, 3) / n
    res = {"metric": "decode attention tokens/s per layer at a fixed KV budget (raw vs compressed)",
           "kv_budget_gb": kv_budget_gb, "layers": LAYERS, "ctx": 4096,
           "per_conversation_raw_bytes": per_conv, "compression_ratio_incl_metadata": round(ratio, 4),
           "conversations_raw": b_raw, "conversations_compressed": b_comp,
           "capacity_gain": round(b_comp / b_raw, 4),
           "raw": {"ms_per_step": round(t_raw * 1e3, 4), "tokens_per_s_per_layer": round(b_raw / t_raw, 1)},
           "compressed": {"ms_per_step": round(t_comp * 1e3, 4),
                          "tokens_per_s_per_layer": round(b_comp / t_comp, 1)},
           "attention_throughput_gain": round((b_comp / t_comp) / (b_raw / t_raw), 4),
           "data": "synthetic (seeded), the Llama-3.1-8B decode distribution with 5% raw blocks",
           "note": "attention only (one layer; GEMMs need weights and are out of scope)"}
    del q, k, v, kz, vz, ws
    torch.cuda.empty_cache()
    return res


def run_capacity(args):
    import torch
    print(json.dumps(measure_capacity(args.kv_budget_gb, args.steps, torch.device("cuda", 0))), flush=True)


def timed_plain(fn, steps, warmup):
    """Device time of `steps` back-to-back calls (CUDA events), seconds."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def measure_codec_sweep(steps: int, dev):
    """Codec throughput on the 4 GiB K+V pool at raw-block shares 0/10/50/100%:
    compress and decompress each pool, check the round trip bit for bit; one
    record per share (bytes read + written per second, averaged over K, V)."""
    import torch
    import decode_attention_zipfusion_b200 as zf
    import zfsynth
    n_rep = max(3, min(20, steps))
    out = []
    for f, k_np, v_np in zfsynth.codec_pool_sweep():
        res = {}
        for name, arr in (("K", k_np), ("V", v_np)):
            x = torch.from_numpy(arr.reshape(-1).view(np.int16)).to(dev).view(torch.bfloat16)
            n = x.numel()
            ws = torch.empty(zf.lib().zf_compress_workspace_size(n), dtype=torch.uint8, device=dev)
            z = zf.CompressedKV.empty(n, dev)
            y = torch.empty_like(x)
            t_c = timed_plain(lambda: zf.compress(x, out=z, ws=ws), n_rep, 2) / n_rep
            t_d = timed_plain(lambda: zf.decompress(z, out=y), n_rep, 2) / n_rep
            ok = bool(torch.equal(x.view(torch.int16), y.view(torch.int16)))
            nb = n // 64
            comp = z.units() * 16 + 4 * (nb + 1) + nb + 4 * ((nb + 31) // 32)
            res[name] = dict(compress_gbs=(2 * n + comp) / t_c / 1e9, decompress_gbs=(2 * n + comp) / t_d / 1e9,
                             ratio=comp / (2 * n), bitwise_roundtrip=ok, compress_ms=t_c * 1e3,
                             decompress_ms=t_d * 1e3)
            del x, z, y, ws
            torch.cuda.empty_cache()
        out.append({"raw_block_share": f, "unit": "GB/s", "steps": n_rep,
                    "compress_gbs": round((res["K"]["compress_gbs"] + res["V"]["compress_gbs"]) / 2, 2),
                    "decompress_gbs": round((res["K"]["decompress_gbs"] + res["V"]["decompress_gbs"]) / 2, 2),
                    "ratio_incl_metadata": round((res["K"]["ratio"] + res["V"]["ratio"]) / 2, 4),
                    "bitwise_roundtrip": res["K"]["bitwise_roundtrip"] and res["V"]["bitwise_roundtrip"],
                    "per_pool": {k2: {k3: round(v3, 4) if isinstance(v3, float) else v3 for k3, v3 in v2.items()}
                                 for k2, v2 in res.items()}})
    return out


def run_codec_sweep(args):
    """One JSON line per raw-block share (a side measurement, not the headline)."""
    import torch
    for rec in measure_codec_sweep(args.steps, torch.device("cuda", 0)):
        rec = {"metric": "codec GB/s (bytes read + written) on the 4 GiB K+V pool", **rec,
               "data": "synthetic (seeded; N(0,1) x lognormal(0,1) channel scales, exact raw-block share)"}
        print(json.dumps(rec), flush=True)


def measure_workload(index: int, steps: int, dev, peak: float):
    """One benchmark workload on one GPU: the compressed decode step and the
    raw-BF16 twin (device time of back-to-back calls), their outputs compared
    bit for bit, the device error word, and the roofline figures."""
    import torch
    import decode_attention_zipfusion_b200 as zf
    import zfsynth
    t_gen = time.perf_counter()
    case = zfsynth.config(index)
    t_gen = time.perf_counter() - t_gen

    def up16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = up16(case.q), up16(case.k_pool), up16(case.v_pool)
    pt = torch.from_numpy(case.page_table).to(dev)
    sl = torch.from_numpy(case.seq_lens).to(dev)
    kz, vz = zf.compress(k), zf.compress(v)
    ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, case.max_seq_len, dev)
    out = torch.empty((case.B, case.Hq, 128), dtype=torch.bfloat16, device=dev)
    out_r = torch.empty_like(out)
    lse = torch.empty((case.B, case.Hq), dtype=torch.float32, device=dev)
    lse_r = torch.empty_like(lse)
    k_elig = kz.elig.cpu().numpy().view(np.uint32)
    v_elig = vz.elig.cpu().numpy().view(np.uint32)
    alg, raw_equiv, kv_comp = algorithmic_bytes(case, k_elig, v_elig)

    def comp():
        zf.decode_attention(q, kz, vz, pt, sl, case.max_seq_len, num_pages=case.num_pages, Hkv=case.Hkv,
                            sm_scale=case.sm_scale, out=out, lse=lse, ws=ws)

    def raw():
        zf.decode_attention_raw(q, k, v, pt, sl, case.max_seq_len, sm_scale=case.sm_scale, out=out_r, lse=lse_r,
                                ws=ws)
    n = max(10, steps)
    t_c = timed_plain(comp, n, 3) / n
    t_r = timed_plain(raw, n, 3) / n
    comp()
    raw()
    torch.cuda.synchronize()
    equal = bool(torch.equal(out.view(torch.int16), out_r.view(torch.int16)) and torch.equal(lse, lse_r))
    err = zf.get_device_error(ws)
    gbs = alg / t_c / 1e9
    res = {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "max_seq_len": case.max_seq_len,
           "ms_per_step": round(t_c * 1e3, 5), "raw_twin_ms_per_step": round(t_r * 1e3, 5),
           "compressed_kv_gbs": round(gbs, 2),
           "uncompressed_equiv_gbs": round(raw_equiv / t_c / 1e9, 2),
           "frac_of_measured_peak": round(gbs / peak, 4), "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
           "tokens_per_s": round(case.B / t_c / LAYERS, 1), "tokens_per_s_per_layer": round(case.B / t_c, 1),
           "speedup_compressed_vs_raw": round(t_r / t_c, 4), "bitwise_equal_to_raw_twin": equal,
           "device_error_word": err, "bytes_per_step": int(alg), "compressed_kv_bytes": int(kv_comp),
           "raw_kv_bytes": int(raw_equiv - (alg - kv_comp)), "steps": n,
           "raw_block_share": round(case.meta["forced_raw_k"] / max(1, case.meta["used_blocks"]), 4),
           "input_generation_s": round(t_gen, 1)}
    del q, k, v, kz, vz, ws, out, out_r
    torch.cuda.empty_cache()
    return res


def run_one_kernel(args):
    """Time one decode kernel (compressed flat form, paged form, raw BF16 or
    FP8) on the workload, alone: the warm-up calls, then `steps` calls.  One
    JSON line; meant for profiling one kernel at a time."""
    import torch
    import decode_attention_zipfusion_b200 as zf
    import zfsynth
    dev = torch.device("cuda", 0)
    case = zfsynth.config(args.config)

    def up16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = up16(case.q), up16(case.k_pool), up16(case.v_pool)
    pt = torch.from_numpy(case.page_table).to(dev)
    sl = torch.from_numpy(case.seq_lens).to(dev)
    ws = zf.decode_workspace(case.B, case.Hq, case.Hkv, case.max_seq_len, dev)
    out = torch.empty((case.B, case.Hq, 128), dtype=torch.bfloat16, device=dev)
    kw = dict(sm_scale=case.sm_scale, out=out, ws=ws)
    if args.kernel == "compressed":
        kz, vz = zf.compress(k), zf.compress(v)
        fn = lambda: zf.decode_attention(q, kz, vz, pt, sl, case.max_seq_len, num_pages=case.num_pages,  # noqa: E731
                                         Hkv=case.Hkv, **kw)
    elif args.kernel == "paged":
        pk, pv = zf.compress_paged(k), zf.compress_paged(v)
        fn = lambda: zf.decode_attention_paged(q, pk, pv, pt, sl, case.max_seq_len, num_pages=case.num_pages,  # noqa: E731
                                               Hkv=case.Hkv, **kw)
    elif args.kernel == "raw":
        fn = lambda: zf.decode_attention_raw(q, k, v, pt, sl, case.max_seq_len, **kw)  # noqa: E731
    else:
        def pool_scale(bits):
            return max(float(np.abs((bits.astype(np.uint32) << 16).view(np.float32)).max()), 1e-30) / 448.0
        ks8, vs8 = pool_scale(case.k_pool), pool_scale(case.v_pool)
        k8, v8 = zf.fp8_quantize(k, ks8), zf.fp8_quantize(v, vs8)
        fn = lambda: zf.decode_attention_fp8(q, k8, v8, ks8, vs8, pt, sl, case.max_seq_len, **kw)  # noqa: E731
    torch.cuda.synchronize()
    t = timed_plain(fn, max(1, args.steps), args.warmup) / max(1, args.steps)
    print(json.dumps({"kernel": args.kernel, "workload": case.name, "ms_per_call": round(t * 1e3, 5),
                      "calls": max(1, args.steps), "warmup": args.warmup,
                      "device_error_word": zf.get_device_error(ws)}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads, the codec sweep and the capacity model in the JSON line")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--capacity", action="store_true",
                    help="conversations and attention tokens/s at a fixed KV budget, raw vs compressed (one GPU)")
    ap.add_argument("--kv-budget-gb", type=float, default=80.0)
    ap.add_argument("--codec-sweep", action="store_true",
                    help="codec throughput at raw-block shares 0/10/50/100%% on the 4 GiB pool (one GPU)")
    ap.add_argument("--kernel", choices=["compressed", "paged", "raw", "fp8"], default=None,
                    help="time only this decode kernel on the workload (for profiling one kernel); "
                         "the warm-up is not raised to 3 in this mode")
    args = ap.parse_args(argv)
    if args.kernel:
        run_one_kernel(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.codec_sweep:
        run_codec_sweep(args)
        return
    if args.capacity:
        run_capacity(args)
        return
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

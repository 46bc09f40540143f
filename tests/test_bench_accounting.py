"""Host logic of the bench.

* The algorithmic byte count (the numerator of the roofline's achieved
  bandwidth), checked against the oracle's own encoding: per used (page,
  kv head) chunk its K and V payload extents from the oracle's offset table,
  40 bytes of metadata per chunk and pool (32 base exponents, one
  eligibility word, one offset entry), and q, out, page-table entries and
  seq_lens once.
* The clock record: median SM clock, throttle reasons and the samples taken
  inside the timed window, from nvidia-smi rows.
"""
import numpy as np

import bench
import oracle
import zfsynth


def test_algorithmic_bytes_match_the_oracle_encoding():
    case = zfsynth.make_case("acct", B=4, Hq=8, Hkv=2, ctx=[300, 17, 0, 64], sigma=0.7, inelig=0.2,
                             k_outlier_channels=3, seed=501)
    kz = oracle.compress(case.k_pool.reshape(-1))
    vz = oracle.compress(case.v_pool.reshape(-1))
    comp_bytes, raw_bytes, kv_bytes = bench.algorithmic_bytes(case, kz.elig, vz.elig)

    kv = 0
    chunks = 0
    pages = 0
    for b in range(case.B):
        n = (int(case.seq_lens[b]) + 15) // 16
        pages += n
        for page in case.page_table[b, :n]:
            for h in range(case.Hkv):
                c = int(page) * case.Hkv + h
                for z in (kz, vz):
                    kv += (int(z.offs[32 * c + 32]) - int(z.offs[32 * c])) * 16 + 40
                chunks += 1
    small = 2 * case.B * case.Hq * 128 * 2 + 4 * pages + 4 * case.B
    assert kv_bytes == kv
    assert comp_bytes == kv + small
    assert raw_bytes == chunks * 2 * 4096 + small
    # every used block of a chunk is either 96 (eligible) or 128 (raw) bytes
    assert kv_bytes < chunks * 2 * (4096 + 40)


def test_chunk_bytes_from_eligibility_words():
    words = np.array([0, 0xFFFFFFFF, 1, 0x80000000, 0x0F0F0F0F], dtype=np.uint32)
    got = bench.chunk_bytes_from_elig(words)
    assert got.tolist() == [4096, 32 * 96, 4096 - 32, 4096 - 32, 4096 - 16 * 32]


def test_clock_summary_from_sampled_rows():
    """NVML samples (SM clock, power, clock-event reason mask) -> median clock,
    the device's max clock, the reasons seen, the sample count."""
    import types
    clk = bench.NvmlSampler(0)
    clk.nv = types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
                                   nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4,
                                   nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80)
    clk.max_mhz = 1965
    clk.rows = [(1965, 800.1, 0x0, 1.0), (1900, 990.0, 0x4, 2.0), (1950, 950.5, 0x0, 3.0), (1860, 1000.2, 0x4, 4.0)]
    s = clk.summary()
    assert s["sm_mhz"] == 1925.0 and s["sm_max_mhz"] == 1965 and s["sm_mhz_min"] == 1860
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 4 and s["power_w_max"] == 1000.2


def test_clock_summary_keeps_the_timed_window():
    """Samples before the warm-up ended or after the region are dropped, except
    the nearest one on each side (the region's edges)."""
    import types
    clk = bench.NvmlSampler(0)
    clk.nv = types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonSwPowerCap=0x4)
    clk.max_mhz = 1965
    clk.rows = [(1000, 100.0, 0x8, 1.0), (1500, 200.0, 0x0, 2.0), (1965, 600.0, 0x0, 3.5), (1950, 650.0, 0x4, 4.5),
                (1800, 300.0, 0x0, 6.0), (900, 90.0, 0x8, 7.0)]
    clk.t_start, clk.t_end = 3.0, 5.0
    s = clk.summary()
    assert s["samples"] == 4 and s["samples_in_timed_region"] == 2
    assert s["sm_mhz_min"] == 1500 and s["power_w_max"] == 650.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples():
    s = bench.NvmlSampler(0).summary()
    assert s["samples"] == 0 and s["reasons"] == ["no samples"]

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
    """nvidia-smi rows (clock, max clock, power, active mask, four reason
    flags) -> median clock, max, the reasons seen and the samples that fell
    inside the timed window."""
    clk = bench.ClockSampler(0)
    rows = [
        (1.00, ["1965", "1965", "800.1", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]),
        (1.02, ["1900", "1965", "990.0", "0x4", "Not Active", "Not Active", "Not Active", "Active"]),
        (1.04, ["1950", "1965", "950.5", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]),
        (1.06, ["[N/A]", "1965", "950.5", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]),
    ]
    clk.rows = list(rows)
    clk.window = (1.01, 1.05)
    s = clk.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 4 and s["samples_in_timed_region"] == 2


def test_clock_summary_without_samples():
    s = bench.ClockSampler(0).summary()
    assert s["samples"] == 0 and s["reasons"] == ["no samples"]

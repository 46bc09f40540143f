"""Exhaustive pin of the oracle's codec at block size 2: all 2^32 pairs of
bf16 bit patterns, checked for the lossless round trip, the eligibility
threshold (exponent spread <= 15), the base (the smaller exponent) and the
size (12 bits per value when eligible) by a threaded C harness linked to the
oracle library (tests/bruteforce_pairs.c).  The harness is also shown to
report failures, by running it on an oracle with a planted mistake."""
import os
import shutil
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.path.join(HERE, "_build")


def harness(lib_path: str, name: str) -> str:
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, name)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-pthread",
                           os.path.join(HERE, "bruteforce_pairs.c"), lib_path,
                           f"-Wl,-rpath,{os.path.dirname(lib_path)}", "-o", exe])
    return exe


def threads():
    return max(1, min(16, os.cpu_count() or 1))


@pytest.fixture(scope="module")
def gcc():
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")


def test_every_pair_of_bf16_patterns(gcc):
    exe = harness(oracle.build(), "bruteforce_pairs")
    res = subprocess.run([exe, str(threads())], capture_output=True, text=True, timeout=1200)
    assert res.returncode == 0 and res.stdout.strip() == "0", res.stdout + res.stderr


def test_harness_reports_a_planted_mistake(gcc):
    import test_oracle_mutants as tm
    exe = harness(tm.build_mutant("threshold_below_15"), "bruteforce_pairs_mutant")
    res = subprocess.run([exe, str(threads()), "512"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 1 and int(res.stdout.strip()) > 0

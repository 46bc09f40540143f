"""The C oracle under AddressSanitizer and UndefinedBehaviorSanitizer: a
driver (tests/oracle_sanitize.c) calls every oracle entry point on
exact-size heap buffers, checking the round trips as it goes."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_oracle_is_clean_under_asan_and_ubsan():
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "oracle_sanitize")
    cmd = ["gcc", "-O1", "-g", "-std=c11", "-Wall", "-Wextra", "-Werror", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=all", os.path.join(HERE, "oracle_sanitize.c"),
           os.path.join(ROOT, "oracle", "zf_oracle.c"), "-lm", "-o", exe]
    build = subprocess.run(cmd, capture_output=True, text=True)
    if build.returncode != 0 and "sanitize" in build.stderr and "cannot find" in build.stderr:
        pytest.skip("the C compiler has no sanitizer runtime")
    assert build.returncode == 0, build.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
    env.pop("LD_PRELOAD", None)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=300, env=env)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr

"""The C-ABI library loads without a GPU, exports every call include/zf.h
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import decode_attention_zipfusion_b200 as zf
from decode_attention_zipfusion_b200 import build as zbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zf.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zf_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    zbuild.build()
    return zf.lib()


def test_header_declares_the_four_named_calls():
    names = declared_functions()
    for f in ("zf_compress_kv", "zf_decompress_kv", "zf_decode_attention", "zf_decode_attention_raw"):
        assert f in names


def test_every_declared_symbol_is_exported(L):
    raw = ctypes.CDLL(zf.LIB_PATH)
    missing = [f for f in declared_functions() if not hasattr(raw, f)]
    assert not missing, missing


def test_host_only_queries(L):
    assert L.zf_version() >= 100
    assert L.zf_status_string(0) == b"ZF_OK"
    assert L.zf_status_string(6) == b"ZF_ERR_TIMEOUT"
    assert L.zf_compressed_bound(64 * 10) == 2 * 64 * 10
    assert L.zf_compressed_bound(63) == 0
    # 3073 blocks: 9 tiles of 384 blocks, one 8-byte scan state each after a 16-byte header
    assert L.zf_compress_workspace_size(64 * 1024 * 3 + 64) == 16 + 8 * 9
    a = L.zf_decode_workspace_size(32, 32, 8, 4096, 148)
    b = L.zf_decode_workspace_size(32, 32, 8, 4096, 74)
    assert a > b > 0
    assert L.zf_decode_workspace_size(-1, 32, 8, 4096, 148) == 0


def _attn(L, **kw):
    args = dict(q=16, k=None, v=None, num_pages=8, pt=16, maxp=4, sl=16, maxlen=64, B=2, Hq=8, Hkv=2, D=128,
                scale=0.088, out=16, lse=None, ws=256, wsb=1 << 20, stream=None)
    args.update(kw)
    kd = zf.CompressedDesc(16, 16, 16, 16, 8 * 2 * 2048, 1 << 20)
    return L.zf_decode_attention(args["q"], ctypes.byref(kd), ctypes.byref(kd), args["num_pages"], args["pt"],
                                 args["maxp"], args["sl"], args["maxlen"], args["B"], args["Hq"], args["Hkv"],
                                 args["D"], args["scale"], args["out"], args["lse"], args["ws"], args["wsb"],
                                 args["stream"])


def test_argument_errors_before_any_cuda_call(L):
    assert _attn(L, D=64) == 2                 # head_dim != 128
    assert _attn(L, Hq=6, Hkv=4) == 2          # Hq % Hkv
    assert _attn(L, Hq=32, Hkv=2) == 2         # group 16 > 8
    assert _attn(L, B=5000) == 2               # batch limit
    assert _attn(L, B=4097) == 2
    assert _attn(L, B=4096, Hq=64, Hkv=64) == 2   # 2^18 (sequence, kv head) segments > 2^17
    assert _attn(L, B=-1) == 1
    assert _attn(L, q=None) == 1
    assert _attn(L, q=8) == 1                  # misaligned q
    assert _attn(L, ws=128) == 1               # workspace must be 256-byte aligned
    assert _attn(L, scale=float("nan")) == 1
    assert _attn(L, B=0) == 0                  # nothing to do
    kd = zf.CompressedDesc(16, 16, 16, 16, 100, 1 << 20)   # n_values % 64
    assert L.zf_decompress_kv(ctypes.byref(kd), 16, None) == 1
    kd = zf.CompressedDesc(16, 16, 16, 16, 64 * 4, 100)
    assert L.zf_compress_kv(16, 64 * 4, ctypes.byref(kd), 256, 1024, None) == 3   # capacity < bound
    assert L.zf_compress_kv(16, 64 * 8, ctypes.byref(kd), 256, 1024, None) == 1   # n_values mismatch
    assert L.zf_clear_device_error(None, None) == 1


def test_product_has_no_cpu_fallback(monkeypatch, tmp_path):
    """Without the shared library the binding raises instead of computing."""
    monkeypatch.setattr(zf, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(zf, "_lib", None)
    with pytest.raises(ImportError):
        zf.lib()


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "decode_attention_zipfusion_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src and "zf_oracle" not in src


def test_host_buffer_entry_sizes_and_argument_errors(L):
    """zf_decode_attention_host: its workspace is the decode workspace plus
    256-byte aligned staging for q, the page table, seq_lens, out and lse;
    bad arguments are rejected before any copy or CUDA call."""
    def up(x):
        return (x + 255) // 256 * 256
    d = L.zf_decode_workspace_size(32, 32, 8, 4096, 148)
    want = up(up(up(up(up(d) + 32 * 32 * 256) + 32 * 256 * 4) + 32 * 4) + 32 * 32 * 256) + 32 * 32 * 4
    assert L.zf_decode_host_workspace_size(32, 32, 8, 256, 4096, 148) == want
    assert L.zf_decode_host_workspace_size(32, 32, 8, 0, 4096, 148) == 0
    assert L.zf_decode_host_workspace_size(-1, 32, 8, 256, 4096, 148) == 0

    def call(**kw):
        a = dict(q=16, kd=zf.CompressedDesc(16, 16, 16, 16, 8 * 2 * 2048, 1 << 20), num_pages=8, pt=16, maxp=4,
                 sl=16, maxlen=64, B=2, Hq=8, Hkv=2, D=128, scale=0.088, out=16, lse=None, ws=256, wsb=1 << 24)
        a.update(kw)
        return L.zf_decode_attention_host(a["q"], ctypes.byref(a["kd"]), ctypes.byref(a["kd"]), a["num_pages"],
                                          a["pt"], a["maxp"], a["sl"], a["maxlen"], a["B"], a["Hq"], a["Hkv"],
                                          a["D"], a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], None)
    assert call(D=64) == 2
    assert call(Hq=32, Hkv=2) == 2
    assert call(B=-1) == 1
    assert call(q=None) == 1
    assert call(out=None) == 1
    assert call(ws=None) == 1
    assert call(ws=128) == 1                     # workspace alignment
    assert call(kd=zf.CompressedDesc(16, 16, 16, 16, 4096, 1 << 20)) == 1   # pool size mismatch
    assert call(B=0) == 0


def test_bounded_wait_check_argument_errors(L):
    assert L.zf_check_bounded_wait(7, 256, 256, None) == 1      # no such mode
    assert L.zf_check_bounded_wait(-1, 256, 256, None) == 1
    assert L.zf_check_bounded_wait(0, None, 256, None) == 1
    assert L.zf_check_bounded_wait(0, 260, 256, None) == 1      # result must be 8-byte aligned
    assert L.zf_check_bounded_wait(0, 256, None, None) == 1


def test_header_and_library_from_plain_c(L):
    """A C11 program (-Wall -Wextra -Werror) includes zf.h, links libzf.so
    and gets the documented host-side answers without a GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_check")
    lib_dir = os.path.dirname(zf.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_check.c"),
                           "-L", lib_dir, "-lzf", f"-Wl,-rpath,{lib_dir}", "-o", exe])
    res = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr


def test_append_argument_errors(L):
    """zf_append_paged / zf_append_paged_kv reject bad pools and arguments on
    the host (the pointers below are never dereferenced)."""
    kd = zf.PagedDesc(1 << 12, 1 << 16, 16, 1 << 20)    # data, chunk_tab, num_chunks, capacity
    vd = zf.PagedDesc(1 << 24, 1 << 28, 16, 1 << 20)
    other = zf.PagedDesc(1 << 24, 1 << 28, 24, 1 << 20)
    B, Hkv = 2, 8

    def kv(k=kd, v=vd, B_=B, Hkv_=Hkv, kc=256, vc=512, kv_=1 << 8, vv=1 << 9):
        return L.zf_append_paged_kv(ctypes.byref(k), ctypes.byref(v), kv_, vv, 64, 4096, 128, B_, Hkv_, 0, 0,
                                    kc, vc, None, None)

    assert L.zf_append_paged(ctypes.byref(kd), 256, 64, 4096, 128, B, 3, 0, 256, None, None) == 1  # 16 % 3
    assert L.zf_append_paged(ctypes.byref(kd), 256, 64, 0, 128, B, Hkv, 0, 256, None, None) == 1   # no pages
    assert L.zf_append_paged(ctypes.byref(kd), 256, 64, 4096, 128, 0, Hkv, 0, 256, None, None) == 0  # B == 0
    assert kv(v=kd) == 1                 # the same pool twice
    assert kv(v=other) == 1              # different chunk counts
    assert kv(vc=256) == 1               # one cursor for both pools
    assert kv(Hkv_=0) == 1
    assert kv(kv_=0) == 1                # no K values
    assert kv(B_=0) == 0                 # nothing to do

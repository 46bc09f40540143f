"""The oracle's pins catch plausible mistakes.  Each case below plants one
mistake in a copy of the oracle's C source (a wrong threshold, a dropped
term, a wrong sign or index, a transposed operand, a swapped layout), builds
it with gcc, points the oracle at the broken build and runs every pin of
tests/test_oracle_*.py: at least one pin must fail for every planted mistake.
Only mistakes that keep every memory access of the oracle in bounds are
planted (a broken decoder never reads past its block)."""
import contextlib
import importlib
import inspect
import os
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
MUTANT_DIR = os.path.join(HERE, "_mutants")
PIN_MODULES = ("test_oracle_codec", "test_oracle_paged", "test_oracle_attention", "test_oracle_fp8")

# name -> [(text in zf_oracle.c, replacement), ...]; each text occurs once.
MUTANTS = {
    # codec: threshold, base, offsets, nibble layout, sign plane, decode, sizes
    "threshold_below_15": [("  int eligible = (emax - emin) <= 15;\n  *base_out",
                            "  int eligible = (emax - emin) < 15;\n  *base_out")],
    "base_is_block_max": [("*base_out = (uint8_t)emin;", "*base_out = (uint8_t)emax;")],
    "offset_without_base": [("int off_lo = exponent_field(w[k]) - emin;", "int off_lo = exponent_field(w[k]);")],
    "nibbles_swapped": [("out[n + k] = (uint8_t)(off_lo | (off_hi << 4));",
                         "out[n + k] = (uint8_t)(off_hi | (off_lo << 4));")],
    "high_nibble_wrong_value": [("int off_hi = exponent_field(w[k + n / 2]) - emin;",
                                 "int off_hi = exponent_field(w[k + 1]) - emin;")],
    "sign_of_own_value": [("sign_bit(w[partner])", "sign_bit(w[j])")],
    "decode_drops_the_addition": [("      e = base + off;", "      e = off;")],
    "raw_plane_minus_base": [("for (int j = 0; j < n; ++j) out[n + j] = (uint8_t)exponent_field(w[j]);",
                              "for (int j = 0; j < n; ++j) out[n + j] = (uint8_t)(exponent_field(w[j]) - emin);")],
    "eligible_block_raw_size": [("return eligible ? (int64_t)n * 12 / 8 : (int64_t)n * 2;",
                                 "return eligible ? (int64_t)n * 2 : (int64_t)n * 2;")],
    "offset_total_off_by_one": [("  offs[n_blocks] = (uint32_t)(pos / 16);",
                                 "  offs[n_blocks] = (uint32_t)(pos / 16 + 1);")],
    # paged form: header layout
    "paged_mask_bytes_reversed": [("out[32] = (uint8_t)(mask & 0xFF);", "out[32] = (uint8_t)(mask >> 24);"),
                                  ("out[35] = (uint8_t)(mask >> 24);", "out[35] = (uint8_t)(mask & 0xFF);")],
    "paged_bases_shifted": [("p += zfo_pack_block(src + (int64_t)i * 64, 64, out + p, &out[i], &el);",
                             "p += zfo_pack_block(src + (int64_t)i * 64, 64, out + p, &out[i + 1], &el);")],
    # attention: scale, grouping, layout, operands, normaliser, log, empty rows
    "attention_without_scale": [("s[t] = sm_scale * dot;", "s[t] = dot;")],
    "gqa_heads_interleaved": [("int hk = hq / group;", "int hk = hq % Hkv;")],
    "kv_layout_transposed": [("int64_t kv = ((pid * Hkv + hk) * page_size + t % page_size) * D;",
                              "int64_t kv = ((hk * num_pages + pid) * page_size + t % page_size) * D;")],
    "values_read_from_keys": [("o[d] += pt * kv_value(vsrc, vv + d);", "o[d] += pt * kv_value(ksrc, vv + d);")],
    "weights_not_normalised": [("double pt = exp(s[t] - m) / l;", "double pt = exp(s[t] - m);")],
    "normaliser_drops_first_token": [("for (int t = 0; t < len; ++t) l += exp(s[t] - m);",
                                      "for (int t = 1; t < len; ++t) l += exp(s[t] - m);")],
    "lse_in_base_2": [("lse[(int64_t)b * Hq + hq] = m + log(l);", "lse[(int64_t)b * Hq + hq] = m + log2(l);")],
    "empty_row_lse_zero": [("lse[(int64_t)b * Hq + hq] = -INFINITY;", "lse[(int64_t)b * Hq + hq] = 0.0;")],
    # FP8 E4M3
    "e4m3_bias_8": [("v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);", "v = (1.0 + m / 8.0) * ldexp(1.0, e - 8);")],
    "e4m3_subnormal_step": [("v = m * ldexp(1.0, -9);", "v = m * ldexp(1.0, -10);")],
    "e4m3_ties_away_from_even": [("((hi & 1) ? hi - 1 : hi)", "((hi & 1) ? hi : hi - 1)")],
    "e4m3_nan_saturates": [("if (isnan(x)) return 0x7F;", "if (isnan(x)) return 0x7E;")],
}


def build_mutant(name):
    src = open(oracle._SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    os.makedirs(MUTANT_DIR, exist_ok=True)
    c_path = os.path.join(MUTANT_DIR, f"zf_oracle_{name}.c")
    so_path = os.path.join(MUTANT_DIR, f"libzf_oracle_{name}.so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", so_path, c_path, "-lm"])
    return so_path


@contextlib.contextmanager
def oracle_built_from(so_path, monkeypatch):
    with monkeypatch.context() as m:
        m.setattr(oracle, "_LIB", so_path)
        m.setattr(oracle, "_lib", None)
        m.setattr(oracle, "build", lambda force=False: so_path)
        yield


def pins():
    """Every pin of the oracle test modules as (name, zero-argument call)."""
    out = []
    for mod_name in PIN_MODULES:
        mod = importlib.import_module(mod_name)
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            params = list(inspect.signature(fn).parameters)
            if not params:
                out.append((f"{mod_name}::{name}", fn))
                continue
            for mark in getattr(fn, "pytestmark", []):
                if mark.name == "parametrize" and len(params) == 1:
                    for value in mark.args[1]:
                        out.append((f"{mod_name}::{name}[{value}]", lambda fn=fn, value=value: fn(value)))
    return out


def test_the_pins_pass_on_the_real_oracle():
    for name, call in pins():
        call()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, monkeypatch):
    so_path = build_mutant(name)
    failed = []
    with oracle_built_from(so_path, monkeypatch):
        for pin, call in pins():
            try:
                call()
            except Exception:  # an assertion, or an error the mistake provokes
                failed.append(pin)
                break
    assert failed, f"planted mistake '{name}' passes every oracle pin"

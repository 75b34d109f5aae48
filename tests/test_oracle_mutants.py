"""Plausible mistakes planted in copies of the oracle (on the CPU) must each
trip at least one pin.  Each mutant is built from a copy of ``qsa_oracle.c``
with one textual change and checked in a child process."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qsa_oracle.c")

MUTANTS = {
    "visible from pos instead of pos+1": (
        "floor_div(pos + 1, QSA_RATIO)", "floor_div(pos, QSA_RATIO)"),
    "visible not clamped at zero": ("return v > 0 ? v : 0;", "return v;"),
    "position off by one": ("return seq_len - query_len + i;", "return seq_len - query_len + i + 1;"),
    "ReLU dropped": ("s += d > 0.0 ? d : 0.0;", "s += d;"),
    "absolute value instead of ReLU": ("s += d > 0.0 ? d : 0.0;", "s += d > 0.0 ? d : -d;"),
    "one head dropped": ("for (int h = 0; h < QSA_HEADS; ++h)", "for (int h = 0; h < QSA_HEADS - 1; ++h)"),
    "last feature dropped": ("for (int c = 0; c < QSA_DIM; ++c)", "for (int c = 0; c < QSA_DIM - 1; ++c)"),
    "every head reads head 0": ("const uint16_t *qh = q_row + h * q_stride_h;", "const uint16_t *qh = q_row;"),
    "scale dropped": ("return scale * s;", "return s;"),
    "page table ignored": ("int64_t logical_page = n / a->page_size;", "int64_t logical_page = 0;"),
    "rows and requests transposed": ("int64_t b = r / c->a.Q, i = r % c->a.Q;",
                                     "int64_t b = r % c->a.B, i = r / c->a.B;"),
    "prefill columns absolute": ("int64_t n = (int64_t)a->ks[t] + j;", "int64_t n = j;"),
    "prefill entries read row and column swapped": (
        "c->out[e] = prefill_entry(&c->a, c->tt[e], c->jj[e]);",
        "c->out[e] = prefill_entry(&c->a, c->jj[e], c->tt[e]);"),
    "prefill end not clipped to the interval": (
        "int64_t hi = a->ke[t] < a->Nk ? a->ke[t] : a->Nk;", "int64_t hi = a->Nk;"),
    "top-k ties to the higher column": ("return (a->j > b->j) - (a->j < b->j);",
                                        "return (a->j < b->j) - (a->j > b->j);"),
    "top-k selects masked blocks": ("if (!(v > -INFINITY)) continue;", "if (v != v) continue;"),
    "fp8 dequantisation scale dropped": ("k[e] = qsa_oracle_e4m3_to_double(k_row[e]) * k_scale;",
                                         "k[e] = qsa_oracle_e4m3_to_double(k_row[e]);"),
    "e4m3 exponent bias off by one": ("else v = ldexp(1.0 + m / 8.0, e - 7);",
                                      "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3 subnormals read as normals": ("if (e == 0) v = ldexp((double)m, -9);",
                                        "if (e == 0) v = ldexp(1.0 + m / 8.0, -7);"),
    "e4m3 sign ignored": ("return sign ? -v : v;", "return v;"),
    "fp16 read as bf16": ("return f16 ? f16_to_double(bits) : bf16_to_double(bits);",
                          "return bf16_to_double(bits);"),
    "fp16 exponent bias off by one": ("else mag = ldexp(1.0 + man / 1024.0, ex - 15);",
                                      "else mag = ldexp(1.0 + man / 1024.0, ex - 14);"),
    "fp16 subnormals flushed": ("else if (ex == 0) mag = ldexp((double)man, -24);",
                                "else if (ex == 0) mag = 0.0;"),
    "expansion open group starts one group late": (
        "for (int64_t j = 4 * vis; j <= p && n < width; ++j)",
        "for (int64_t j = 4 * vis + 4; j <= p && n < width; ++j)"),
    "expansion drops the last block token": ("for (int64_t r = 0; r < 4; ++r) dst[n++]",
                                             "for (int64_t r = 0; r < 3; ++r) dst[n++]"),
    "attention KV head by modulo": ("int64_t t = th / c->Hq, h = th % c->Hq, g = h / group;",
                                    "int64_t t = th / c->Hq, h = th % c->Hq, g = h % c->Hkv;"),
    "attention keeps future tokens": ("if (j < 0 || j > pos || j >= c->seq_lens[r]) continue;",
                                      "if (j < 0 || j >= c->seq_lens[r]) continue;"),
    "attention scale dropped": ("s[n] = c->scale * dot;", "s[n] = dot;"),
    "attention gate ignored": ("double gt = 1.0 / (1.0 + exp(-c->gate[th]));", "double gt = 1.0;"),
    "attention missing pages kept": ("if (page < 0 || page >= c->num_pages) return NULL;",
                                     "if (page < 0) page = 0;"),
    "top-k keeps the smallest": ("if (a->v > b->v) return -1;\n    if (a->v < b->v) return 1;",
                                 "if (a->v < b->v) return -1;\n    if (a->v > b->v) return 1;"),
}

CHILD = r"""
import json, sys
sys.path.insert(0, {tests!r}); sys.path.insert(0, {root!r})
import oracle, oracle_pins
result = {{}}
for name, lib in json.loads({libs!r}).items():
    o = oracle.Oracle(lib)
    tripped = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except AssertionError:
            tripped.append(pin.__name__)
    result[name] = tripped
print(json.dumps(result))
"""


@pytest.fixture(scope="module")
def tripped_by_mutant(tmp_path_factory):
    src = open(SRC).read()
    d = tmp_path_factory.mktemp("mutants")
    libs = {}
    for i, (name, (old, new)) in enumerate(sorted(MUTANTS.items())):
        assert src.count(old) == 1, f"mutation site not unique: {old!r}"
        mut = d / f"mutant{i}.c"
        mut.write_text(src.replace(old, new))
        lib = d / f"libmutant{i}.so"
        subprocess.run(["gcc", "-O1", "-std=c11", "-D_POSIX_C_SOURCE=200809L", "-fPIC",
                        "-shared", "-pthread", str(mut), "-o", str(lib), "-lm"], check=True)
        libs[name] = str(lib)
    code = CHILD.format(tests=os.path.join(ROOT, "tests"), root=ROOT, libs=json.dumps(libs))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tripped_by_mutant):
    assert tripped_by_mutant[name], f"no pin caught the mutant '{name}'"

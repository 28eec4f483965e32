"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that at least one pin in test_oracle.py catches each of them.  This shows
the pins constrain every step: bounds, page ranges, scores, selection and
attention."""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "slc_oracle.c")

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]

# (name, original text, replacement): each one must exist exactly once
MUTANTS = [
    ("score max->min", "acc += a > c ? a : c;", "acc += a < c ? a : c;"),
    ("score uses kmax twice", "double a = qd * lo[d], c = qd * hi[d];",
     "double a = qd * hi[d], c = qd * hi[d];"),
    ("score drops group sum", "for (int g = 0; g < group; g++) {\n                    const uint16_t *qh",
     "for (int g = 0; g < 1; g++) {\n                    const uint16_t *qh"),
    ("score wrong head index", "q + ((int64_t)b * hq + h * group + g) * dim;",
     "q + ((int64_t)b * hq + h + g) * dim;"),
    ("tie-break to higher page", "return (a->page > b->page) - (a->page < b->page);",
     "return (a->page < b->page) - (a->page > b->page);"),
    ("prefix rounds down", "int np = (prefix + PAGE - 1) / PAGE;", "int np = prefix / PAGE;"),
    ("window one page short", "ws = first / PAGE;", "ws = first / PAGE + 1;"),
    ("bounds read past length", "for (int t = 0; t < valid; t++) {", "for (int t = 0; t < PAGE; t++) {"),
    ("attention drops scale", "z[i] = scale * dot;", "z[i] = dot;"),
    ("attention unnormalised", "double p = z[i] / denom;", "double p = z[i];"),
    ("attention uses key as value",
     "const uint16_t *vt = v_cache + (((int64_t)phys * hkv + h) * PAGE + t % PAGE) * dim;",
     "const uint16_t *vt = k_cache + (((int64_t)phys * hkv + h) * PAGE + t % PAGE) * dim;"),
    ("selection keeps one too many", "int k = budget < m ? budget : m;",
     "int k = budget < m ? budget + 1 : m;"),
    ("sparse drops window pages", "for (int j = ws; j < n; j++)\n                    use[j] = 1;",
     "for (int j = ws + 1; j < n; j++)\n                    use[j] = 1;"),
    ("fp8 bounds round to nearest",
     "kmax8[base + d] = (uint8_t)oracle_fp8_round(kmax[base + d], 1);",
     "kmax8[base + d] = (uint8_t)oracle_fp8_round(kmax[base + d], kmax[base + d] - oracle_fp8_value(oracle_fp8_round(kmax[base + d], 0)) > oracle_fp8_value(oracle_fp8_round(kmax[base + d], 1)) - kmax[base + d]);"),
    ("fp8 rounding off by one code", "return lo < fp8_count ? fp8_table[lo].code : 0x7F;",
     "return lo + 1 < fp8_count ? fp8_table[lo + 1].code : 0x7F;"),
    ("top-delta gap strict", "const int near = smax - buf[i].score <= delta;",
     "const int near = smax - buf[i].score < delta;"),
    ("top-delta one page short of d", "const int in_top = i < d;", "const int in_top = i < d - 1;"),
    ("top-delta cap keeps the lowest pages", "if ((in_top || near) && k < cap)",
     "if (in_top || near)"),
]


def _run_pins():
    failed = []
    for t in PIN_TESTS:
        try:
            t()
        except Exception as e:  # an assertion, or a crash-free error
            failed.append(t.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: " + name
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(lib),
                           str(mutated), "-lm"])
    with oracle.use_library(str(lib)):
        failed = _run_pins()
    assert failed, "no pin caught the planted mistake: " + name


def test_unmutated_oracle_passes_all_pins():
    assert _run_pins() == []

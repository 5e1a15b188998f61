"""Plant plausible mistakes in a copy of the oracle and require that the pins
catch every one of them (the oracle's own source is left untouched)."""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "csa_oracle.c")

# (name, text in csa_oracle.c, replacement)
MUTANTS = [
    ("relu_dropped", "double relu = logit > 0.0 ? logit : 0.0;", "double relu = logit;"),
    ("relu_flipped", "double relu = logit > 0.0 ? logit : 0.0;", "double relu = logit < 0.0 ? -logit : 0.0;"),
    ("visibility_off_by_one", "return (s + 1) * (long long)m - 1 <= t;", "return (s + 1) * (long long)m <= t;"),
    ("visibility_start_token", "return (s + 1) * (long long)m - 1 <= t;", "return s * (long long)m <= t;"),
    ("tie_break_reversed", "if (a->index < b->index) return -1;\n    if (a->index > b->index) return 1;",
     "if (a->index < b->index) return 1;\n    if (a->index > b->index) return -1;"),
    ("sort_ascending", "if (a->score > b->score) return -1;\n    if (a->score < b->score) return 1;",
     "if (a->score > b->score) return 1;\n    if (a->score < b->score) return -1;"),
    ("q_transposed", "logit += qrow[(long long)h * d + j] * key[j];", "logit += qrow[(long long)j * H + h] * key[j];"),
    ("weight_wrong_head", "total += (double)wrow[h] * relu;", "total += (double)wrow[0] * relu;"),
    ("weight_dropped", "total += (double)wrow[h] * relu;", "total += relu;"),
    ("e4m3_bias", "v = ldexp(1.0 + (double)mant / 8.0, expo - 7);", "v = ldexp(1.0 + (double)mant / 8.0, expo - 8);"),
    ("e4m3_subnormal", "v = ldexp((double)mant / 8.0, 1 - 7);", "v = ldexp((double)mant / 8.0, -7);"),
    ("scale_ignored", "v = (double)k_scale[(long long)b * T + s] *", "v = 1.0 *"),
    ("gate_nonstrict", "if (mode == 1 && !(I > 0.0))", "if (mode == 1 && !(I >= 0.0))"),
    ("q_offset_ignored", "return i + q_offset;", "return i;"),
    ("pad_index", "out_idx[o] = -1;", "out_idx[o] = 0;"),
    ("keep_one_less", "long long keep = n < topk ? n : topk;", "long long keep = n < topk ? n : topk - 1;"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation target for {name} not found"
    mut = tmp_path / f"{name}.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-std=c99", "-shared", "-fPIC", "-o",
                           str(so), str(mut), "-lm"])
    return oracle.Oracle(str(so))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    orc = _build_mutant(tmp_path, name, old, new)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"

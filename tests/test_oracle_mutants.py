"""The oracle's pins catch plausible mistakes: each mutant below is a copy of
oracle.c with one mistake planted (a dropped term, a wrong sign, index,
offset, bias or tie order), compiled on its own; the oracle's CPU pins
(test_oracle, test_formats, test_schedule_oracle, test_topk_oracle) then run
against it in a child process, and at least one of them must fail. The
unchanged source, compiled the same way, must pass them (the control).

Every mistake is planted in the oracle, on the CPU; nothing here touches
the GPU or the CUDA library."""
import concurrent.futures
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle.py", "tests/test_formats.py", "tests/test_schedule_oracle.py",
        "tests/test_topk_oracle.py"]

# (name, text in oracle.c, replacement): the first occurrence is replaced
# (for the per-format point functions that is the FP8 one).
MUTANTS = [
    ("fp8 ReLU dropped", "double r = s * score;\n        if (r < 0.0) r = 0.0;",
     "double r = s * score;"),
    ("fp8 per-token scale dropped", "double r = s * score;", "double r = score;"),
    ("fp8 weight sign dropped", "sum += wh * r;", "sum += fabs(wh) * r;"),
    ("tolerance denominator signed", "a += fabs(wh) * r;", "a += wh * r;"),
    ("fp8 weights of draft 0 for every draft",
     "double wh = (double)w[((int64_t)b * next_n + n) * H + h];",
     "double wh = (double)w[((int64_t)b * next_n) * H + h];"),
    ("fp8 q of draft 0 for every draft",
     "const uint8_t* qrow = q + (((int64_t)b * next_n + n) * H + h) * D;",
     "const uint8_t* qrow = q + (((int64_t)b * next_n) * H + h) * D;"),
    ("fp8 token slot off by one", "int64_t slot = t % page_size;",
     "int64_t slot = (t + 1) % page_size;"),
    ("draft rule off by one", "int64_t c = ctx_b - next_n + 1 + n;",
     "int64_t c = ctx_b - next_n + n;"),
    ("masked elements written as 0", "o[t] = -INFINITY;", "o[t] = 0.0;"),
    ("e4m3 exponent bias", "v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);"),
    ("e4m3 subnormal scale", "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    ("e2m1 subnormal value", "v = 0.5 * m;", "v = 1.0 * m;"),
    ("bf16 bit position", "uint32_t u = (uint32_t)bits << 16;", "uint32_t u = (uint32_t)bits << 15;"),
    ("fp4 K nibble order", "uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);",
     "uint8_t code = (d % 2 == 0) ? (byte >> 4) : (byte & 0xF);"),
    ("fp4 K block-scale index", "double k = e2m1_value[code] * e4m3_value[srow[d / 16]];",
     "double k = e2m1_value[code] * e4m3_value[srow[(d / 16 + 1) % (D / 16)]];"),
    ("nvfp4 q nibble order", "uint8_t qc = (d % 2 == 0) ? (qb & 0xF) : (qb >> 4);",
     "uint8_t qc = (d % 2 == 0) ? (qb >> 4) : (qb & 0xF);"),
    ("nvfp4 q scaled by K's block scales",
     "double qv = e2m1_value[qc] * e4m3_value[qsc[d / 16]];",
     "double qv = e2m1_value[qc] * e4m3_value[srow[d / 16]];"),
    ("schedule without the remainder spread",
     "int64_t start = (int64_t)i * (U / S) + (i < U % S ? i : U % S);",
     "int64_t start = (int64_t)i * (U / S);"),
    ("schedule units rounded down", "U += (c + 255) / 256;", "U += c / 256;"),
    ("top-k ties to the higher token", "return (a->t > b->t) - (a->t < b->t);",
     "return (a->t < b->t) - (a->t > b->t);"),
    ("top-k padded with token 0", "o[i] = i < cbn ? items[i].t : -1;",
     "o[i] = i < cbn ? items[i].t : 0;"),
    ("top-k ignores the draft rule", "const int64_t cbn = draft_ctx(c, next_n, n);",
     "const int64_t cbn = c;"),
]


def _run_pins(lib_path):
    env = dict(os.environ, MQA_ORACLE_LIB=lib_path)
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider", "-k", "not generator"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-1500:]


def _build(tmp, name, src):
    d = os.path.join(tmp, name.replace(" ", "_").replace("'", ""))
    os.makedirs(d, exist_ok=True)
    c = os.path.join(d, "oracle.c")
    with open(c, "w") as f:
        f.write(src)
    return oracle_build.compile_to(c, os.path.join(d, "liboracle.so"))


@pytest.mark.slow
def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(oracle_build.SRC).read()
    jobs = [("control", src)]
    for name, old, new in MUTANTS:
        assert old in src, f"{name}: the text to mutate is not in oracle.c"
        mutated = src.replace(old, new, 1)
        assert mutated != src
        jobs.append((name, mutated))
    libs = [(name, _build(str(tmp_path), name, s)) for name, s in jobs]
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda nl: (nl[0],) + _run_pins(nl[1]), libs))
    rc0, out0 = results[0][1], results[0][2]
    assert rc0 == 0, "the unchanged oracle must pass its pins:\n" + out0
    survivors = [name for name, rc, _ in results[1:] if rc == 0]
    odd = [(name, rc) for name, rc, _ in results[1:] if rc not in (0, 1)]
    assert not odd, f"pins did not run cleanly against: {odd}"
    assert not survivors, f"planted mistakes no pin catches: {survivors}"

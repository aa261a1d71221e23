"""Mutation check of the oracle's pins.

Each mutant plants one plausible mistake in a copy of ``oracle/oracle.c`` (a
dropped term, a wrong sign, a wrong operand, an off-by-one, a wrong rounding
tie rule ...), builds it on the CPU, and reruns ``test_oracle_pins.py``
against it.  Every mutant must make at least one pin fail; a mutant that
survives means the pins leave that part of the oracle unchecked.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTANTS = [
    ("weight decay sign", "float d = g + t;", "float d = g - t;"),
    ("weight decay dropped", "float d = g + t;", "float d = g;"),
    ("weight decay on momentum", "float t = weight_decay * w_old;", "float t = weight_decay * v[j];"),
    ("momentum term dropped", "vn = u + d;", "vn = d;"),
    ("momentum on gradient", "float u = momentum * v[j];", "float u = momentum * d;"),
    ("update sign", "float wn = w_old - s;", "float wn = w_old + s;"),
    ("update uses d not v", "step = vn;", "step = d;"),
    ("unscale dropped", "return orc_widen16(g16) * inv_scale;", "return orc_widen16(g16);"),
    ("clip inverted", "g = g * coef;", "g = g / coef;"),
    ("clip coefficient inverted", "r->clip_coef = (float)((double)clip / r->norm);",
     "r->clip_coef = (float)(r->norm / (double)clip);"),
    ("clip threshold compares sumsq", "r->norm > (double)clip", "r->sumsq > (double)clip"),
    ("sum of |x| not x^2", "sumsq = sumsq + x * x;", "sumsq = sumsq + (x < 0 ? -x : x);"),
    ("no skip on overflow", "if (!r->found_inf) {", "if (1) {"),
    ("inf missed by check", "if (mag >= 0x7c00u) {", "if (mag > 0x7c00u) {"),
    ("subnormal bound", "else if (mag < 0x0400u)", "else if (mag <= 0x0400u)"),
    ("ties away from zero", "(rem == half && (m & 1u))", "(rem == half)"),
    ("truncation instead of rounding", "if (rem > half || (rem == half && (m & 1u)))", "if (0)"),
    ("subnormal binade of the narrowing", "int te = e > -14 ? e : -14;", "int te = e > -15 ? e : -15;"),
    ("overflow to largest finite", "return (uint16_t)(sign | 0x7c00u); /* |x| >= 2^16",
     "return (uint16_t)(sign | 0x7bffu); /* |x| >= 2^16"),
    ("subnormal widen exponent", "ldexpf((float)frac16, -24)", "ldexpf((float)frac16, -23)"),
    ("widen exponent bias", "((exp16 - 15u + 127u) << 23)", "((exp16 - 14u + 127u) << 23)"),
    ("growth off by one", "*clean_run >= cfg->growth_interval", "*clean_run > cfg->growth_interval"),
    ("backoff keeps counter", "float s = scale * cfg->backoff;\n        *clean_run = 0;",
     "float s = scale * cfg->backoff;"),
    ("growth by backoff", "float s = scale * cfg->growth;", "float s = scale * cfg->backoff;"),
    ("stale test inverted", "h_new == orc_rne16(w_old)", "h_new != orc_rne16(w_old)"),
    ("fp16 copy from old weight", "uint16_t h_new = orc_rne16(wn);", "uint16_t h_new = orc_rne16(w_old);"),
    ("histogram by fraction bits", "r->exp_hist[mag >> 10] += 1;", "r->exp_hist[mag & 31u] += 1;"),
    ("maximum includes inf/NaN", "            if (mag > max_mag)   /* bit patterns of magnitudes order like values */\n                max_mag = mag;\n",
     ""),
    ("direct scale without margin", "(double)margin * (double)max_abs", "(double)max_abs"),
    ("direct scale clamps swapped", "    if (s < min_scale)\n        s = min_scale;", "    if (s < min_scale)\n        s = max_scale;"),
    ("direct mode ignored", "    if (cfg->mode == ORC_SCALER_DIRECT) {", "    if (0) {"),
    ("direct mode zero max gives zero", "        return s > 0.0f ? s : scale;", "        return s;"),
    ("nesterov look-ahead dropped", "                step = d + m2;", "                step = vn;"),
    ("nesterov look-ahead on old v", "float m2 = momentum * vn;", "float m2 = momentum * v[j];"),
    ("adagrad without square", "float sq = d * d;", "float sq = d;"),
    ("adagrad without root", "float den = sqrtf(vn) + eps;", "float den = vn + eps;"),
    ("adagrad eps inside root", "float den = sqrtf(vn) + eps;", "float den = sqrtf(vn + eps);"),
    ("adagrad accumulates before decay", "            float sq = d * d;", "            float sq = g * g;"),
]


def _run_mutant(mutant, workdir):
    name, old, new = mutant
    with open(os.path.join(oracle_build.HERE, "oracle.c")) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
    d = os.path.join(workdir, "m%d" % MUTANTS.index(mutant))
    os.makedirs(d)
    with open(os.path.join(d, "oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    shutil.copy(os.path.join(oracle_build.HERE, "oracle.h"), d)
    so = os.path.join(d, "liboracle.so")
    subprocess.run(["gcc", *oracle_build.CFLAGS, os.path.join(d, "oracle.c"), "-o", so, "-lm"],
                   check=True, capture_output=True)
    env = dict(os.environ, ORACLE_LIB=so)
    out = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"),
                          "-x", "-q", "-p", "no:cacheprovider"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, out.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda m: _run_mutant(m, tmp), MUTANTS))
    survivors = [name for name, rc in results if rc == 0]
    assert survivors == [], f"mutants not caught by any pin: {survivors}"

"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory: a dropped term, a wrong constant, sign, index or
comparison), then runs the oracle's pin tests against that copy.  They must
fail.  The real oracle is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (id, text in ffd_oracle.c, replacement, which occurrence (0-based))
MUTANTS = [
    ("int4-scale-divisor", "float_to_bf16(amax / 7.0f)", "float_to_bf16(amax / 8.0f)", 0),
    ("int4-code-offset", "return u - 8;", "return u - 7;", 0),
    ("int4-code-clamp", "if (r > 7.0f) r = 7.0f;", "if (r > 6.0f) r = 6.0f;", 0),
    ("block-score-min-not-max", "if (dot > best) best = dot;",
     "if (best == INT64_MIN || dot < best) best = dot;", 0),
    ("topdelta-strict-compare", "int k = s[j] >= threshold;", "int k = s[j] > threshold;", 0),
    ("topdelta-no-running-update", "running = fmaxf(running, s[j]);", "(void)running;", 0),
    ("topdelta-split-stride", "split0 < nb; split0 += S)", "split0 < nb; split0 += S + 1)", 0),
    ("topdelta-no-group-union", "if (k) m[j / 32] |= 1u << (j % 32);",
     "if (k && h % G == 0) m[j / 32] |= 1u << (j % 32);", 0),
    ("pseudo-fixed-sink-only", "float pseudo = fmaxf(s[0], s[nb - 1]);", "float pseudo = s[0];", 1),
    ("pseudo-seeded-no-running-update", "running = fmaxf(running, s[j]);", "(void)running;", 1),
    ("query-fold-range", "float inv = 127.0f / a;", "float inv = 128.0f / a;", 0),
    ("attention-no-scale", "double scale = 1.0 / sqrt((double)D);", "double scale = 1.0;", 0),
    ("attention-denominator", "o[c] /= denom;", "o[c] /= denom + 1.0;", 0),
    ("attention-gqa-map",
     "      int g = h / G;\n      size_t row = (size_t)b * Hkv + g;\n      const uint16_t *qh",
     "      int g = h % Hkv;\n      size_t row = (size_t)b * Hkv + g;\n      const uint16_t *qh", 0),
    ("thumb-level-step", "(double)(254 * u - 381 + e) / 254.0", "(double)(256 * u - 381 + e) / 254.0", 0),
    ("thumb-score-offset", "(2 * thumb_code(tr, c) - 3)", "(2 * thumb_code(tr, c) - 2)", 0),
    ("thumb-residual-step", "nearbyintf(d * 254.0f)", "nearbyintf(d * 256.0f)", 0),
]


def _plant(src, old, new, nth):
    pos = -1
    for _ in range(nth + 1):
        pos = src.find(old, pos + 1)
        assert pos >= 0, f"mutation site not found: {old!r}"
    return src[:pos] + new + src[pos + len(old):]


def _run_pins(tmp_path, source):
    """The oracle's pin tests on a copy of the oracle built from `source`."""
    (tmp_path / "oracle").mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), tmp_path / "oracle")
    (tmp_path / "oracle" / "ffd_oracle.c").write_text(source)
    shutil.copytree(os.path.join(ROOT, "ffd_workloads"), tmp_path / "ffd_workloads",
                    ignore=shutil.ignore_patterns("__pycache__"))
    (tmp_path / "tests").mkdir()
    for name in ("conftest.py", "test_oracle.py", "test_oracle_tr.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), tmp_path / "tests")
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tmp_path / "tests" / "golden")
    env = dict(os.environ, PYTHONPATH=str(tmp_path), PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle.py", "tests/test_oracle_tr.py"],
                       cwd=tmp_path, env=env, capture_output=True, text=True, timeout=600)
    # the copy, not the repository's oracle, was loaded
    assert (tmp_path / "oracle" / "libffd_oracle.so").exists(), r.stdout[-2000:] + r.stderr[-2000:]
    return r


def test_unchanged_copy_passes(tmp_path):
    # the control: the harness itself does not make the pins fail
    with open(os.path.join(ROOT, "oracle", "ffd_oracle.c")) as f:
        r = _run_pins(tmp_path, f.read())
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("mid,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_a_planted_mistake(tmp_path, mid, old, new, nth):
    with open(os.path.join(ROOT, "oracle", "ffd_oracle.c")) as f:
        src = f.read()
    mutated = _plant(src, old, new, nth)
    assert mutated != src
    r = _run_pins(tmp_path, mutated)
    assert r.returncode == 1, f"{mid}: the pins did not catch it\n" + r.stdout[-3000:]

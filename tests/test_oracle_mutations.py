"""The oracle's pins have teeth: plausible mistakes planted in a copy of the C oracle
(on the CPU) must each be caught by at least one pin.

Each mutation rewrites one line of oracle/attn_oracle.c, builds the copy into a temporary
library, points the oracle's Python wrapper at it, and runs the pin suite
(test_oracle_pins.py) in a subprocess; the suite must fail. The unmutated copy must
pass, so the harness itself is checked too.
"""

from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
SRC = (ROOT / "oracle" / "attn_oracle.c").read_text()

MUTATIONS = {
    # the softmax without subtracting the row maximum (overflows for large logits)
    "no_max_subtraction": ("s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
    # causal test off by one (a row does not see its own key)
    "causal_off_by_one": ("nvis = last + 1;", "nvis = last;"),
    # LSE in log2 instead of natural log
    "lse_log2": ("*lse_out = m + log(l);", "*lse_out = m + log2(l);"),
    # interleaved instead of contiguous head groups
    "gqa_interleaved": ("const int g = h / group;", "const int g = h % Hkv;"),
    # weights not normalised
    "no_normalisation": ("s[j] /= l;", "s[j] /= 1.0;"),
    # key row read with the query's stride (transposed operand)
    "key_index": ("const uint16_t *krow = kh + j * (int64_t)d;",
                  "const uint16_t *krow = kh + (j % 2) * (int64_t)d;"),
    # the value of the wrong key
    "value_index": ("const uint16_t *vrow = vh + j * (int64_t)d;",
                    "const uint16_t *vrow = vh + (nvis - 1 - j) * (int64_t)d;"),
    # scale applied twice
    "scale_twice": ("s[j] = scale * acc;", "s[j] = scale * scale * acc;"),
    # global offsets ignored in the causal test
    "offsets_ignored": ("int64_t last = qpos - kv_off;", "int64_t last = qpos - kv_off * 0;"),
    # fully masked rows give LSE = 0 instead of -inf
    "empty_row_lse": ("*lse_out = -INFINITY;\n        return;", "*lse_out = 0.0;\n        return;"),
}


def _build(src: str, out: Path) -> Path:
    c = out / "attn_oracle.c"
    c.write_text(src)
    so = out / "liboracle.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                    str(c), "-lm"], check=True)
    return so


def _run_pins(so: Path) -> subprocess.CompletedProcess:
    # a tiny plugin loaded before the pins points the oracle wrapper at the copy
    code = (
        "import sys, ctypes, pytest\n"
        f"sys.path.insert(0, {str(ROOT)!r}); sys.path.insert(0, {str(ROOT / 'tests')!r})\n"
        "import oracle\n"
        f"oracle._LIB_PATH = __import__('pathlib').Path({str(so)!r})\n"
        "oracle.build = lambda force=False: oracle._LIB_PATH\n"
        "oracle._lib = None\n"
        f"sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider', "
        f"{str(ROOT / 'tests' / 'test_oracle_pins.py')!r}]))\n"
    )
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=600, env=dict(os.environ, OMP_NUM_THREADS="2"))


def test_unmutated_copy_passes(tmp_path):
    r = _run_pins(_build(SRC, tmp_path))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    assert SRC.count(old) == 1, f"mutation anchor not found once: {old!r}"
    r = _run_pins(_build(SRC.replace(old, new), tmp_path))
    assert r.returncode != 0, f"the pins did not catch mutation {name}"

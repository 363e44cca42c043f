"""The append kernel takes its two divisions without an IEEE divide, and the
stored scales and codes must not change for it ("KV cache quantization: what
FP8/INT8 K and V really give", "The quantization step": scale from the row's
range, codes from x / scale; codes and scales are compared bit for bit with the
oracle).

- The row scale amax / 448 (E4M3), amax / 57344 (E5M2) and (hi - lo) / 255
  (INT8) is a multiply by the rounded reciprocal and one correction on the exact
  FMA residual. Over every BF16 amax and every BF16 pair (hi, lo) this equals
  the IEEE quotient bit for bit.
- The code quotient x / s is the same correction with a per-row reciprocal of
  the BF16 scale s (Markstein's method), taken for s >= 2^-100; it may differ
  from the IEEE quotient in its last bit, but over every BF16 x with
  |x| <= 65536 s (the quotient range of all three formats, subnormal x
  included) the E4M3, E5M2 and rint codes are the IEEE quotient's.

A host C program enumerates all these cases; the last-bit differences of the
code quotient are counted too, so a rule that only ever reproduced the IEEE
quotient would show.
"""

import os
import re
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "native", "scale_division_check.c")
FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math"]   # every product and FMA as written


def _compile(src, exe):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    subprocess.run([gcc] + FLAGS + ["-o", exe, src, "-lm"], check=True)
    return exe


def _run(exe, mode, a, b):
    p = subprocess.run([exe, mode, hex(a), hex(b)], capture_output=True, text=True)
    m = re.search(r"checked (\d+) differ (\d+) mismatches (\d+)", p.stdout)
    assert m, p.stdout + p.stderr
    return p.returncode, p.stdout, tuple(int(v) for v in m.groups())


def _sliced(exe, mode, lo, hi):
    n = max(1, min(16, os.cpu_count() or 1))
    edges = [lo + (hi - lo) * i // n for i in range(n + 1)]
    with ThreadPoolExecutor(n) as ex:
        res = list(ex.map(lambda i: _run(exe, mode, edges[i], edges[i + 1]), range(n)))
    assert all(r[0] == 0 for r in res), "".join(r[1] for r in res if r[0])
    return [sum(r[2][j] for r in res) for j in range(3)]


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    return _compile(SRC, str(tmp_path_factory.mktemp("divcheck") / "scale_division_check"))


def test_row_scales_equal_the_ieee_quotient(checker):
    checked, _, bad = _sliced(checker, "scale", 0, 0x7F80)
    assert bad == 0
    assert checked > 2 * 0x7F80 + 0x7F80 * 0x7F80 // 2      # both constants + the INT8 ranges


def test_code_quotient_gives_ieee_codes_for_all_bf16_pairs(checker):
    checked, differ, bad = _sliced(checker, "quot", 0x0080, 0x7F80)
    assert bad == 0
    assert checked > 900_000_000
    assert differ > 0


def test_a_dropped_correction_is_caught(tmp_path):
    """Planted mistake on the host: the plain product RN(x RN(1/s)) without the
    residual correction changes codes, so the check has teeth."""
    src = open(SRC).read()
    planted = src.replace("const float q2 = fmaf(-e, r, q);",
                          "const float q2 = q; (void)e;")
    assert planted != src
    p = tmp_path / "planted.c"
    p.write_text(planted)
    exe = _compile(str(p), str(tmp_path / "planted"))
    rc, out, (_, _, bad) = _run(exe, "quot", 0x3C00, 0x3D00)
    assert rc == 1 and bad > 0, out


def test_a_plain_reciprocal_scale_is_caught(tmp_path):
    """Planted mistake: a scale taken as RN(a RN(1/c)) alone differs from the
    IEEE quotient for some BF16 amax."""
    src = open(SRC).read()
    planted = src.replace("return fmaf(fmaf(-q, c, a), r, q);", "return q;")
    assert planted != src
    p = tmp_path / "planted.c"
    p.write_text(planted)
    exe = _compile(str(p), str(tmp_path / "planted"))
    rc, out, (_, _, bad) = _run(exe, "scale", 0, 0x10)
    assert rc == 1 and bad > 0, out


def test_a_correction_that_loses_the_sign_of_zero_is_caught(tmp_path):
    """Planted mistake: the residual taken the other way round, e = fma(-q, s,
    x) and q2 = fma(e, r, q), turns x = -0 into +0, whose E4M3 / E5M2 code
    differs (0x00 against 0x80)."""
    src = open(SRC).read()
    planted = src.replace("const float e = fmaf(q, s, -x);", "const float e = fmaf(-q, s, x);")
    planted = planted.replace("const float q2 = fmaf(-e, r, q);", "const float q2 = fmaf(e, r, q);")
    assert planted != src
    p = tmp_path / "planted.c"
    p.write_text(planted)
    exe = _compile(str(p), str(tmp_path / "planted"))
    rc, out, (_, _, bad) = _run(exe, "quot", 0x3C00, 0x3C01)
    assert rc == 1 and bad > 0, out

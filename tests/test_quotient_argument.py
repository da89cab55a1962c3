"""The append kernel's quantize step reaches RN(v / s) without a division per
value (Markstein's correction step; see the quotient notes in csrc/append.cu).
This pins the arithmetic fact it relies on, in IEEE binary32 with
fused multiply-add on the host, for every bf16 significand against every
float significand of the scale (all 2^23), plus the patterns that stress a
reciprocal (all-ones, zero, the repeating 1/7 of amax / 448 scales).  A
negative control shows the check can fail."""
import os
import re
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker():
    d = tempfile.mkdtemp()
    exe = os.path.join(d, "quotient_check")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", os.path.join(HERE, "quotient_check.c"),
                    "-o", exe, "-lm"], check=True)
    return exe


def run(exe, first, count, stride, control=False):
    out = subprocess.run([exe, str(first), str(count), str(stride)] + (["c"] if control else []),
                         capture_output=True, text=True, check=True).stdout
    n, bad = map(int, re.match(r"n=(\d+) bad=(\d+)", out).groups())
    return n, bad


def test_corrected_product_is_the_ieee_quotient(checker):
    n, bad = run(checker, 0, 1 << 23, 1)                   # every float significand in [1, 2)
    assert n == 128 << 23 and bad == 0
    for m in (0x7FFFFF, 0x000000, 0x000001, 0x7FFFFE, 0x492492, 0x36DB6D, 0x5B6DB7, 0x12492):
        assert run(checker, m, 1, 1) == (128, 0)


def test_negative_control_uncorrected_product_differs(checker):
    n, bad = run(checker, 0, 1 << 12, 2039, control=True)
    assert bad > n // 20

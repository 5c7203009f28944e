"""The quantize kernel divides by the block scale with Markstein's method
(RN(1/d), then one fused-multiply-add correction) instead of a full
correctly rounded division.  This CPU test compiles tests/division_check.c
and runs it: over every finite fp16 and bf16 pair (w, c) with |w| <= c, for
the NF4 divisor c and the INT4-symmetric divisor RN(c/7), and over a seeded
sample of INT4-asymmetric divisors, the method's quotient equals RN(w/d)
wherever |w/d| >= 2^-6 and stays below 2^-5 (where every code and every
rint is the same) elsewhere.  About 4e9 pairs; a few seconds with OpenMP."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def test_markstein_quotient_decides_every_code_exhaustively(tmp_path):
    exe = tmp_path / "division_check"
    base = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", os.path.join(HERE, "division_check.c"),
            "-o", str(exe), "-lm"]
    try:
        subprocess.run(base[:1] + ["-fopenmp"] + base[1:], check=True, capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run(base, check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=1200)
    lines = r.stdout.strip().splitlines()
    assert r.returncode == 0, r.stdout + r.stderr
    assert len(lines) == 6
    for ln in lines:
        f = ln.split()
        assert int(f[3]) > 10_000_000 and f[5] == "0", ln

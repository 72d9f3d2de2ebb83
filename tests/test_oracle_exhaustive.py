"""Exhaustive pin of the oracle's E2M1 encoder: every fp32 value (NaN
excepted), both tie rules, against an independent brute-force nearest
search in C (tests/exhaustive_e2m1.c), about 10-30 s on the host cores."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def test_e2m1_encoder_exhaustive(orc, tmp_path):
    lib = orc.build()
    exe = str(tmp_path / "exhaustive_e2m1")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-o", exe,
                           os.path.join(HERE, "exhaustive_e2m1.c"), lib,
                           "-Wl,-rpath," + os.path.dirname(lib), "-lm"])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr

"""The quantizer kernels replace x / s by a reciprocal with one FMA correction; this
runs tests/quotient_check.c, which replays that sequence in IEEE host arithmetic for
every possible (amax, x) bf16 pair and both scale modes (about 2.1e9 quotients)."""
import os
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.slow
def test_quotient_shortcut_is_exact_for_every_bf16_pair():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "quotient_check")
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-o", exe, os.path.join(HERE, "quotient_check.c"),
                               "-lm"])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "ok" in out.stdout

"""The fused pass's short reciprocal and quotient, proven exact on the host.

The CUDA kernel does not call a full divide per NF4 block: it takes fl(1/a) for the
normalisation ("QLoRA", "How It Works": each block is scaled by its absmax) and fl(a/s) for the
8-bit code of the double-quantized constant (same section: the constants are quantized in
turn) with one Newton-Raphson correction on a fused multiply-add.  A small C program
(tests/division_check.c) replays that arithmetic with fmaf for every 16-bit value and every
pair of 16-bit values the kernel can meet, in both formats, and compares with the correctly
rounded IEEE reciprocal and quotient.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("div") / "division_check")
    subprocess.run([gcc, "-O2", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "division_check.c"), "-lm"], check=True)
    return exe


def _counts(out):
    w = out.split()
    return {w[i]: int(w[i + 1]) for i in (0, 2, 4, 6)} if len(w) >= 8 else {}


def test_short_reciprocal_and_quotient_are_exact(checker):
    r = subprocess.run([checker], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    words = r.stdout.split()
    assert words[0] == "recips" and words[4] == "quotients"
    assert int(words[1]) > 80_000 and int(words[3]) == 0   # every candidate reciprocal
    assert int(words[5]) > 600_000_000 and int(words[7]) == 0  # every pair a <= s


def test_division_check_catches_a_missing_correction(checker):
    """The check has teeth: the quotient without its correction step fails it."""
    r = subprocess.run([checker, "0"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 1
    assert int(r.stdout.split()[7]) > 0

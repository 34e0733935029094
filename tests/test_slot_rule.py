"""The fused pass's code lookup (slot curve + two tables) against the midpoint count.

The CUDA kernel decides each code with a cheap rule instead of counting midpoints (see
aqnf4_slot_tables in the header).  Here a small C program replays that rule in binary32 on
the host, with the library's tables, for every binary32 value near a midpoint or a slot
boundary and a strided sweep of the rest of [-1 - 2^-20, 1 + 2^-20], and compares with the
oracle's codebook: the code is the number of midpoints below v ("QLoRA", "How It Works").
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from quantized_lora_setup_b200 import aqnf4

HERE = os.path.dirname(os.path.abspath(__file__))


def _hex(a):
    return " ".join("%08x" % int(u) for u in np.asarray(a, np.float32).view(np.uint32))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("slot") / "slot_rule_check")
    subprocess.run([gcc, "-O2", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "slot_rule_check.c"), "-lm"], check=True)
    return exe


def _run(exe, curve, slot_mid, slot_level, mids, levels):
    feed = " ".join([_hex(curve), _hex(slot_mid), _hex(slot_level), _hex(mids), _hex(levels)])
    r = subprocess.run([exe], input=feed, capture_output=True, text=True, timeout=300)
    return r.returncode, r.stdout + r.stderr


def test_slot_tables_follow_the_codebook():
    curve, slot_mid, slot_level = aqnf4.aqnf4_slot_tables()
    levels, mids = oracle.codebook()
    assert slot_mid[0] == -np.inf and np.all(slot_mid[16:] == np.inf)
    assert np.array_equal(slot_mid[1:16].view(np.uint32), mids.view(np.uint32))
    assert np.array_equal(slot_level[1:17].view(np.uint32), levels.view(np.uint32))


def test_slot_rule_equals_the_midpoint_count(checker):
    curve, slot_mid, slot_level = aqnf4.aqnf4_slot_tables()
    levels, mids = oracle.codebook()
    rc, out = _run(checker, curve, slot_mid, slot_level, mids, levels)
    assert rc == 0, out
    assert "mismatches 0" in out
    assert int(out.split()[1]) > 50_000_000


def test_slot_check_catches_a_wrong_curve(checker):
    """The check itself has teeth: a curve with a shifted slot grid fails it."""
    curve, slot_mid, slot_level = aqnf4.aqnf4_slot_tables()
    levels, mids = oracle.codebook()
    bent = curve.copy()
    bent[0] *= np.float32(1.08)
    rc, out = _run(checker, bent, slot_mid, slot_level, mids, levels)
    assert rc == 1 and "mismatches 0" not in out

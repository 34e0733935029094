"""Host logic of bench.py that needs no GPU: the session command line, the algorithmic
byte counts its rooflines divide by."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_session_child_argv(bench):
    f = bench.session_child_argv
    assert f(["--sessions", "3", "--steps", "50", "--no-e2e"]) == ["--steps", "50", "--no-e2e",
                                                                   "--protocol"]
    assert f(["--sessions=3", "--protocol"]) == ["--protocol"]
    assert f([]) == ["--protocol"]


def test_dequant_alg_bytes(bench):
    # packed codes + 8-bit constants + fp32 DQ scales in, bf16 out
    n = 28672 * 8192
    nb = n // 64
    assert bench.dequant_alg_bytes(n) == n // 2 + nb + 4 * ((nb + 255) // 256) + 2 * n
    # a ragged tail: 100 elements = 2 blocks, 1 scale
    assert bench.dequant_alg_bytes(100) == 50 + 2 + 4 + 200


def _profile_commands():
    """Every `python bench.py ...` command line the profile summaries give (backslash
    continuations joined, inline-code backticks and trailing prose dropped)."""
    import glob
    import re
    cmds = []
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read().replace("\\\n", " ")
        for line in text.splitlines():
            for m in re.finditer(r"python bench\.py((?:\s+--?[\w-]+(?:[ =](?!--)[^\s`]+)?)*)", line):
                cmds.append((os.path.basename(path), m.group(1).split()))
    return cmds


def test_profile_commands_parse(bench, monkeypatch):
    """The commands the profiles record still parse with bench.py's own arguments."""
    cmds = _profile_commands()
    assert len(cmds) >= 5
    for name, argv in cmds:
        monkeypatch.setattr("sys.argv", ["bench.py"] + argv)
        bench.parse_args()  # exits on an unknown or malformed argument

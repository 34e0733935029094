"""Host logic of bench.py that needs no GPU: the session command line, the algorithmic
byte counts its rooflines divide by."""
import importlib.util
import json
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


def test_compact_summary_fits_the_line_tail(bench):
    """The summary that ends the JSON line keeps every headline figure in well under the
    1500 bytes of a line's tail."""
    rf = {"frac": 0.61234567, "achieved": 4000.0}
    wl = {"value": 3000.0, "layers_per_s": 40000.0, "roofline": rf}
    r = {"value": 3100.0, "layers_per_s": 54000.0, "roofline": rf,
         "workloads": {"14b": wl, "1.4b": wl},
         "dequant": {"shape": "28672x8192", "value": 5600.0, "roofline": rf},
         "dequant_sweep": {"points": [{"case": c, "frac": 0.5, "copy_frac": 0.6}
                                      for c in ("packed_1MB", "packed_8MB", "packed_16MB",
                                                "packed_1024MB")]},
         "nf4_linear": {"unit": "TFLOP/s", "tokens_4096": {"value": 1000.0,
                                                            "dequant_then_cublas": 1400.0},
                        "tokens_512": {"value": 800.0, "dequant_then_cublas": 700.0},
                        "tokens_128": {"value": 260.0, "dequant_then_cublas": 280.0}},
         "dq_score": {"roofline": rf}}
    s = bench.compact_summary(r)
    r["summary"] = s
    line = json.dumps(r)
    assert line.endswith(json.dumps(s) + "}")
    assert len(json.dumps(s)) < 1000
    for key in ("frac", "layers_per_s", "14b", "1.4b", "dequant", "gemm_tokens_4096",
                "gemm_tokens_512", "gemm_tokens_128", "dq_score_frac"):
        assert key in s
    assert s["dequant"]["packed_8MB"] == [0.5, 0.6]

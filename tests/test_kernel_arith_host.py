"""Host checks of the arithmetic rules inside the CUDA prologue that make its
codes and scales equal the oracle's bit for bit (the rules themselves are
stated in rotate_quant.cu): the constant-divisor Markstein quotient for the
row scale, and the checked reciprocal quantizer.  The rules are restated in
plain C (tests/host_c/quant_rules.c), compiled with gcc without contraction,
and compared with IEEE division and with rint of the correctly rounded
quotient.  No GPU, and nothing from the oracle or the CUDA sources."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is needed")
    exe = str(tmp_path_factory.mktemp("arith") / "quant_rules")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                           os.path.join(HERE, "host_c", "quant_rules.c"), "-lm"])
    return exe


def test_scale_division_and_checked_quantizer(checker):
    out = subprocess.run([checker, "97", "5000000"], capture_output=True, text=True, timeout=600)
    lines = dict(l.split(" ", 1) for l in out.stdout.strip().splitlines())
    checked, bad = map(int, lines["div"].split())
    cases, fast, bad_q = map(int, lines["quant"].split())
    assert checked > 40_000_000 and bad == 0
    assert cases > 4_000_000 and fast > cases // 4 and bad_q == 0
    assert out.returncode == 0


def test_the_checker_catches_a_wrong_rule(tmp_path):
    # A margin of zero (no guard for the rounding of the quotient) must let
    # wrong codes through on the int8 range; the test would be blind otherwise.
    if shutil.which("gcc") is None:
        pytest.skip("gcc is needed")
    src = open(os.path.join(HERE, "host_c", "quant_rules.c")).read()
    bad_src = src.replace("ldexpf(1.0f, -18) : ldexpf(1.0f, -14)", "0.0f : 0.0f")
    assert bad_src != src
    (tmp_path / "bad.c").write_text(bad_src)
    exe = str(tmp_path / "bad")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-o", exe, str(tmp_path / "bad.c"), "-lm"])
    out = subprocess.run([exe, "100003", "2000000"], capture_output=True, text=True, timeout=600)
    assert out.returncode == 1

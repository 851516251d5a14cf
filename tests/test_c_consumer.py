"""The C ABI from plain C: tests/c/abi_consumer.c includes include/convrot.h,
is compiled by gcc as strict C11 (-Wall -Wextra -Werror -pedantic), links
against libconvrot_b200.so and runs its host-side checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libdir():
    from rotation_quantized_bit_b200 import build
    return os.path.dirname(build.build())


def test_header_compiles_as_strict_c_and_links(tmp_path, libdir):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    exe = tmp_path / "abi_consumer"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
                           "-L", libdir, "-lconvrot_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"

"""Host-side checks of the bounds build (libm3_bounds.so: every kernel
compiled with M3_DEVICE_CHECKS, device-side index checks that record a
failure and skip the access instead of trapping): it exports the same ABI as
the normal build and says which build it is; the binding loads it under
M3_BOUNDS=1; and the range predicate every check uses, compiled for the host,
accepts exactly the in-range element ranges.  CPU-only."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "state_space_sequence_ssm_b200", "csrc")

from test_abi import declared_functions  # noqa: E402


@pytest.fixture(scope="module")
def bounds_lib():
    from state_space_sequence_ssm_b200 import build
    path = build.build(bounds=True)
    assert os.path.basename(path) == "libm3_bounds.so"
    return path


def test_bounds_build_exports_the_same_abi(bounds_lib):
    out = subprocess.run(["nm", "-D", "--defined-only", bounds_lib], capture_output=True, text=True).stdout
    assert set(re.findall(r"\bT (m3\w*)", out)) == set(declared_functions())
    und = subprocess.run(["nm", "-D", "--undefined-only", bounds_lib], capture_output=True, text=True).stdout
    assert not [l for l in und.splitlines() if "_ZN2m3" in l]
    lib = ctypes.CDLL(bounds_lib, mode=os.RTLD_NOW)
    assert lib.m3_device_checks() == 1
    assert lib.m3_version() == 103


def test_binding_loads_the_bounds_build_under_env():
    code = ("import state_space_sequence_ssm_b200 as m3, os; "
            "print(os.path.basename(m3.lib_path()), m3.device_checks())")
    env = dict(os.environ, M3_BOUNDS="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["libm3_bounds.so", "True"]
    env.pop("M3_BOUNDS")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["libm3.so", "False"]


PREDICATE_TEST = r"""
#include <climits>
#include <cstdio>
#include "dcheck.cuh"
using m3::dchk::in_range;
// compile-time cases
static_assert(in_range(0, 1, 1) && in_range(3, 4, 7) && in_range(0, 0, 0) && in_range(5, 0, 5), "inside");
static_assert(!in_range(-1, 1, 8) && !in_range(7, 2, 8) && !in_range(8, 1, 8) && !in_range(0, 9, 8), "outside");
static_assert(!in_range(0, -1, 8) && !in_range(0, 1, 0) && !in_range(6, 0, 5), "degenerate");
int main() {
    // no overflow: huge operands never wrap into "inside"
    int bad = 0;
    bad += in_range(LLONG_MAX, 2, LLONG_MAX);
    bad += in_range(LLONG_MAX - 1, 2, LLONG_MAX);
    bad += !in_range(LLONG_MAX - 2, 2, LLONG_MAX);
    bad += in_range(LLONG_MIN, 1, 10);
    bad += in_range(1, LLONG_MAX, 10);
    // exhaustive over small sizes against the plain definition
    for (long long n = 0; n <= 12; ++n)
        for (long long i = -3; i <= 15; ++i)
            for (long long c = -2; c <= 14; ++c) {
                bool want = c >= 0 && i >= 0 && i + c <= n;
                bad += in_range(i, c, n) != want;
            }
    std::printf("%d\n", bad);
    return bad != 0;
}
"""


def test_range_predicate_on_the_host(tmp_path):
    src = tmp_path / "pred.cpp"
    src.write_text(PREDICATE_TEST)
    exe = tmp_path / "pred"
    cuda_inc = "/usr/local/cuda/include"
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-w", f"-I{cuda_inc}", f"-I{CSRC}", f"-I{ROOT}/include",
                        str(src), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "0", r.stdout + r.stderr

"""Host code under AddressSanitizer and UndefinedBehaviorSanitizer (no GPU).

The oracle (tf_oracle.c) and the library's host code (argument checks, the
plan, the C ABI) are rebuilt with -fsanitize=address,undefined, and the
oracle's pins and the C-ABI argument tests run again in a child process that
preloads the sanitizer runtimes and loads those builds.  Any report (a heap
overflow, a use after free, an out-of-range shift, signed overflow) fails the
child, and with it this test.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OUT = os.path.join(ROOT, "_build", "asan")


def _runtime(name):
    path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                          text=True).stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


@pytest.mark.skipif(shutil.which("gcc") is None or shutil.which("nvcc") is None
                    and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs gcc and nvcc")
def test_oracle_pins_and_abi_checks_under_asan_and_ubsan():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not installed")
    import oracle
    from verify_paged_gqa_b200 import build
    os.makedirs(OUT, exist_ok=True)
    lib = build.build(sanitize=True)
    olib = oracle.compile_source(oracle._SRC, os.path.join(OUT, "libtforacle_asan.so"),
                                 sanitize=True)
    env = dict(os.environ,
               LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=0:protect_shadow_gap=0:abort_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1",
               TF_ORACLE_LIB=olib, TFPAGED_LIBRARY=lib)
    # the child checks that it runs on the sanitizer builds, then the tests
    probe = ("import oracle, verify_paged_gqa_b200 as t; oracle._load(); t.raw; "
             "maps = open('/proc/self/maps').read(); "
             f"assert {lib!r} in maps and {olib!r} in maps, 'sanitizer builds not loaded'")
    r = subprocess.run([sys.executable, "-c", probe], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py", "tests/test_abi_cpu.py"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert "runtime error" not in out and "AddressSanitizer" not in out, out[-4000:]

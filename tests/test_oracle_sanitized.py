"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

The oracle decides every parity test, so its own C must not read or write
outside the buffers it is given, on any input: tests/oracle_sanitize_main.c
drives it with exactly-sized heap blocks over round trips, short
capacities, truncated and bit-flipped containers and rewritten headers;
any sanitizer report or failed check ends the run with a non-zero status."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_oracle_is_memory_safe_under_sanitizers(tmp_path):
    exe = str(tmp_path / "oracle_sanitized")
    src = [os.path.join(ROOT, "oracle", "sz_oracle.c"), os.path.join(ROOT, "tests", "oracle_sanitize_main.c")]
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-g", "-Wall", "-Wextra", "-Werror",
                           "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer",
                           "-I", os.path.join(ROOT, "oracle"), "-o", exe] + src)
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-4000:]
    assert r.stdout.strip() == "ok"

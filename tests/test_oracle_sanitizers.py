"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

tests/oracle_sanitize_main.c drives every oracle entry point (routing with
dropped ids, activation quantisation, the layer in all five weight formats
with and without the shared expert, the router) on small seeded inputs; it is
compiled together with oracle/moe_oracle.c with -fsanitize=address,undefined
and -fno-sanitize-recover=all, so any out-of-bounds access, leak or undefined
operation fails the run.  CPU only.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_is_clean_under_asan_and_ubsan(tmp_path):
    exe = str(tmp_path / "oracle_sanitized")
    cmd = ["gcc", "-std=c11", "-O1", "-g", "-fno-omit-frame-pointer", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=all", "-ffp-contract=off", "-I", os.path.join(ROOT, "oracle"),
           os.path.join(HERE, "oracle_sanitize_main.c"), os.path.join(ROOT, "oracle", "moe_oracle.c"),
           "-lm", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "sanitized oracle run ok" in r.stdout

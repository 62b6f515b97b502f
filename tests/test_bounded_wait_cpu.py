"""The bounded poll behind every wait in the kernels, compiled for the host
and driven by a fake clock: with a limit of 0 it gives up at its first clock
check, it returns as soon as the condition holds, it gives up once the limit
has passed, and it gives up when another role raises the abort flag."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_experts_layer_logit_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "bounded_wait_check.cpp")


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("bw") / "bounded_wait_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, SRC, "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return {ln.split()[0]: (int(ln.split()[1]), int(ln.split()[2])) for ln in out.splitlines()}


def test_ready_at_once(results):
    assert results["ready_at_once"] == (1, 1)


def test_cap_zero_gives_up_at_the_first_clock_check(results):
    # one poll, then `every` more before the clock is read again
    assert results["cap0_never_ready"] == (0, 1 + 32)
    assert results["cap0_never_ready_every16"] == (0, 1 + 16)


def test_returns_when_ready_before_the_limit(results):
    assert results["ready_before_limit"] == (1, 501)


def test_limit_runs_out(results):
    ok, polls = results["limit_runs_out"]
    # the clock advances by one per check (every 32 polls): 101 checks after the first
    assert ok == 0 and polls == 1 + 32 * 101


def test_abort_flag_stops_the_wait(results):
    ok, polls = results["abort_flag"]
    assert ok == 0 and polls == 1 + 32 * 3   # the first check after the flag went up at poll 70

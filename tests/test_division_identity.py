"""The quantiser kernels divide by the group scale with a correctly rounded
reciprocal and one FMA residual correction instead of an IEEE division.  This
test restates that arithmetic in C on the host and checks that it yields the
same FP8 code as the IEEE quotient (encoded by the oracle) for every bf16 x with
|x| <= amax, over a stratified set of bf16 amax values (every amax whose scale is
near 2^-126 or 2^-64 plus every 9th one); FP8LIN_EXHAUSTIVE=1 checks all amax."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("div") / "division_identity")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                           os.path.join(HERE, "division_identity.c"),
                           os.path.join(ROOT, "oracle", "fp8_oracle.c"), "-lm", "-lpthread"])
    return exe


def test_fast_division_gives_ieee_codes(checker):
    stride = "1" if os.environ.get("FP8LIN_EXHAUSTIVE") == "1" else "9"
    r = subprocess.run([checker, stride], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "code_mismatches=0" in r.stdout


def test_delayed_scaling_division_gives_ieee_codes_and_clip_flags(tmp_path):
    """The delayed-scaling kernel divides by an arbitrary previous-step scale: for every
    bf16 x and scales of every binary exponent (8 significands each), its quotient must
    give the IEEE quotient's FP8 code and the same clipped flag (tests/division_delayed.c)."""
    exe = str(tmp_path / "division_delayed")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                           os.path.join(HERE, "division_delayed.c"),
                           os.path.join(ROOT, "oracle", "fp8_oracle.c"), "-lm", "-lpthread"])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("code_mismatches=0 clip_mismatches=0") == 2

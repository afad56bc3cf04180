"""The NVFP4 quantizers divide a block amax by 6 with an FMA-corrected product instead of an
IEEE division (the two-level scale of "NVIDIA developed a method to train neural networks in
4-bit precision", How it works: the per-16 scale is E4M3 of amax / 6 times the tensor scale).
The kernels are bit-exact with the oracle only if that quotient is correctly rounded for
every amax they can meet; this checks it exhaustively on the host, over every FP32 value the
fast path accepts, with the C library's correctly rounded fmaf."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _has_fma():
    try:
        with open("/proc/cpuinfo") as f:
            return " fma " in f.read()
    except OSError:
        return False


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_fma_division_by_six_is_correctly_rounded_for_every_fp32(tmp_path):
    exe = str(tmp_path / "div6")
    flags = ["-O2", "-ffp-contract=off"] + (["-mfma"] if _has_fma() else [])
    subprocess.run(["gcc", *flags, "-o", exe, os.path.join(HERE, "host", "div6_exhaustive.c"), "-lm"], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=900).stdout.split()
    bad, n = int(out[0]), int(out[1])
    assert n == 0x7F7FFFFF - 0x01000000 + 1
    assert bad == 0

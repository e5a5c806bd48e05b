"""Exhaustive pin of the oracle's E4M3 encoder (the OCP FP8 E4M3 format; the
pages' "FP8 dispatch" in "DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和
低延迟内核"): every binary32 bit pattern with |v| <= 480, both signs, against a
nearest-value search over the format's 127 finite magnitudes (tests/e4m3_sweep.c).
The range covers every rounding boundary, the subnormal binade, signed zeros and
the saturation band above 448.  About 2.3e9 values, spread over the host's cores.
"""
import os
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.slow
def test_e4m3_encoder_exhaustive_up_to_480(tmp_path):
    lib = oracle.build.build()
    exe = str(tmp_path / "e4m3_sweep")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                    os.path.join(HERE, "e4m3_sweep.c"), lib, "-o", exe,
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=1800)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    last = out.stdout.strip().splitlines()[-1]
    checked = int(last.split()[1])
    assert checked == 2 * (0x43F00000 + 1), last  # 480.0f is 0x43F00000

"""The converter's two encoders, checked on the CPU over their whole domain
(every BF16 block maximum x every BF16 value; about 10^9 pairs each): the
per-block multiplier and the product bracket it falls back to.

The GPU converter (csrc/quant.cu, verify_multiplier) encodes a block with
one multiply per element by a multiplier c it has checked on the 128 BF16
mantissas; tests/native/converter_multiplier_check.c repeats that choice in
FP32 and compares E4M3(RN(v * c)) with E4M3(RN(v / d)) for every v of every
block that takes a multiplier. The codes are the converter's definition
(FastVideo PR #1829, "Changes", converter bullet: W / s with s = amax / 448,
rounded to E4M3); the GPU tests then compare the kernel with the oracle."""
import os
import platform
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_multiplier_gives_the_quotient_codes_for_every_bf16_pair(tmp_path):
    exe = tmp_path / "check"
    # IEEE single precision with round to nearest and no fused multiply-add
    # (x86 would otherwise be free to use x87 extended precision)
    x86 = platform.machine().lower() in ("x86_64", "amd64", "i686", "i386")
    flags = ["-O2", "-ffp-contract=off"] + (["-msse2", "-mfpmath=sse"] if x86 else [])
    subprocess.run(["gcc", *flags, "-o", str(exe),
                    os.path.join(HERE, "native", "converter_multiplier_check.c"), "-lm",
                    "-lpthread"], check=True)
    threads = max(1, min(32, os.cpu_count() or 1))
    out = subprocess.run([str(exe), str(threads)], capture_output=True, text=True, timeout=900)
    line = out.stdout.strip().splitlines()[-1]
    f = dict(zip(line.split()[0::2], (int(v) for v in line.split()[1::2])))
    assert out.returncode == 0 and f["mismatches"] == 0, out.stdout
    # the product bracket: equal ends always give the quotient's code
    assert f["bracket_mismatches"] == 0 and f["bracket_pairs"] > 1.0e9, out.stdout
    assert 0 < f["straddles"] < 0.05 * f["bracket_pairs"]
    # every usable block maximum was tried, about 10^9 pairs compared
    assert f["blocks"] == 28064 and f["pairs"] > 9.8e8
    # most blocks take the multiplier (the rest keep the product bracket)
    assert f["rn"] + f["up"] + f["down"] > 0.9 * f["blocks"]

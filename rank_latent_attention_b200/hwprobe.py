"""Measure the sm_100a rates the kernels are designed around (needs a GPU).

    python -m rank_latent_attention_b200.hwprobe

Builds csrc/hwprobe.cu with nvcc into a temporary directory, runs it on the
current device and prints its JSON lines: MUFU ex2 throughput (fp32 and the
packed f16x2 / bf16x2 forms), fp32 and packed f32x2 FMA throughput,
exp2_poly3 throughput, tcgen05.mma rate (from one divergent thread and from
a warp under elect.sync; N = 64, 128, 256 with A in shared memory or TMEM),
and the mbarrier wake-up latency.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile

from .build import ARCH, CSRC, ROOT, _nvcc


def main() -> int:
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "hwprobe")
        cmd = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-o", exe,
               os.path.join(CSRC, "hwprobe.cu")]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            return 1
        return subprocess.run([exe]).returncode


if __name__ == "__main__":
    sys.exit(main())

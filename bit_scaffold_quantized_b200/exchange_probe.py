"""Build and run the exchange-latency probe (csrc/exchange_probe.cu) on the GPU.

    python -m bit_scaffold_quantized_b200.exchange_probe

Prints the device-timed cost of one grid-wide all-gather round of tagged words and of
one cluster all-to-all round by st.async, the two primitives whose latency bounds the
batch-1 token kernel's layer time.
"""
import os
import subprocess
import sys

from .build import CSRC, NVCC, PKG


def main():
    exe = os.path.join(PKG, "exchange_probe")
    src = os.path.join(CSRC, "exchange_probe.cu")
    if not os.path.exists(exe) or os.path.getmtime(exe) < os.path.getmtime(src):
        subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe, src], check=True)
    sys.exit(subprocess.run([exe]).returncode)


if __name__ == "__main__":
    main()

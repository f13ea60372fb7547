"""The few-token kernel's stream-K work split, checked on the CPU with the
kernel header's own host/device functions: a host program under
tests/host/ is compiled with nvcc (no GPU call) and run."""
import os
import subprocess

from bit_quantized_lora_blockwise_b200.build import ARCH, CSRC, ROOT, nvcc


def test_smallm_split_partitions_units(tmp_path):
    exe = tmp_path / "smallm_split_check"
    src = os.path.join(ROOT, "tests", "host", "smallm_split_check.cu")
    subprocess.check_call([nvcc(), *ARCH, "-O1", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                           "-o", str(exe), src], timeout=600)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0 and p.stdout.strip() == "ok", p.stdout + p.stderr

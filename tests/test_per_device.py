"""Per-device set-up bookkeeping of the CUDA library (kernel attributes and static scratch
addresses are per device): the host-only helper compiled with g++ and exercised on the CPU."""
import os
import subprocess
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_diffusion_decoding_denoising_b200", "csrc")


def test_per_device_once_bookkeeping():
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "per_device_check.cpp")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "per_device_check")
        subprocess.check_call(["g++", "-std=c++17", "-O1", "-pthread", "-I" + CSRC, src, "-o", exe])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


def test_every_init_function_is_per_device():
    """No one-shot process-wide flag guards a per-device set-up call any more."""
    import re
    for name in os.listdir(CSRC):
        if not name.endswith(".cu"):
            continue
        text = open(os.path.join(CSRC, name)).read()
        assert not re.search(r"static bool (done|attr)\b", text), name
        if "cudaFuncSetAttribute" in text or "cudaGetSymbolAddress" in text:
            assert "PerDeviceOnce" in text, name

"""Host-side exhaustive check of the kernels' register bit tricks (no GPU)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_diffusion_transformer_b200", "csrc")


def test_bit_tricks_match_naive_loops(tmp_path):
    exe = tmp_path / "host_bits_check"
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-I", CSRC, "-o", str(exe),
                           os.path.join(os.path.dirname(__file__), "host_bits_check.cpp")])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "OK" in out.stdout

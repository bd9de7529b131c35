"""Host-side checks of the quantizer's integer and floating-point arithmetic
(CPU only): fast division by the number of K groups, the FMA-based exact
quotient used instead of a per-element division (checked against IEEE
division on every bf16 (element, amax) pair), and the static quantizer's
quotient for caller-given scales (every bf16 magnitude against a sweep of
scales from the smallest subnormal to +inf)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fastdiv_and_exact_quotient(tmp_path):
    exe = tmp_path / "host_checks"
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    # the included kernel headers hold sm_100a device code (programmatic
    # launch, cache-hinted loads): compile their device side for that target
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    "-Xcompiler", "-fopenmp,-ffp-contract=off,-fno-fast-math",
                    "-I", os.path.join(ROOT, "fine_grained_fp8_token_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "host", "host_checks.cu"), "-lgomp"],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=900)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "quotient pairs:" in r.stdout and "mismatches: 0" in r.stdout
    assert "static quotient pairs:" in r.stdout

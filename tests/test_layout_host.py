"""Layout arithmetic shared by the kernels and the host, checked on the host.

tests/layout_check.cu includes the library's layout headers and checks, with
no kernel and no GPU, that the tiled weight layout (codes and scale atoms per
feature tile and K chunk) is a bijection with no gaps or overlaps, on the
2880-wide shapes and on ragged ones; that the padded form (two-MXFP8-term
layers) puts every code and scale byte where the weight tensor map's box of
the producer's part index finds it; and that the scale-atom byte formula is a
bijection onto the atoms."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def test_layout_arithmetic(tmp_path):
    exe = str(tmp_path / "layout_check")
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                           "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-o", exe,
                           os.path.join(ROOT, "tests", "layout_check.cu")])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr

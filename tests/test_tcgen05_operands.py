"""The tcgen05 attention kernel's operand layouts and descriptor encodings
against NVIDIA's CUTLASS/CuTe definitions (host programs, no GPU):

- its shared-memory tiles (Q, K, P K-major; V MN-major) equal CuTe's
  canonical 128-byte-swizzle UMMA layouts tiled in the kernel's order, so the
  strides its descriptors name are the ones CuTe would derive;
- its instruction and shared-memory descriptor encoders equal CUTLASS's
  bitfield unions filled with the same fields.

Skipped when nvcc or a vendored CUTLASS include tree is not available."""
import importlib.util
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.join(ROOT, "tests", "cutlass_checks")


def _cutlass_include():
    for pkg, rel in (("flashinfer", ("data", "cutlass", "include")), ("tilelang", ("3rdparty", "cutlass", "include"))):
        spec = importlib.util.find_spec(pkg)
        if spec and spec.origin:
            path = os.path.join(os.path.dirname(spec.origin), *rel)
            if os.path.exists(os.path.join(path, "cute", "arch", "mma_sm100_desc.hpp")):
                return path
    return None


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.parametrize("name,flags", [
    ("layout_check", ["-Wno-deprecated-gpu-targets"]),
    ("desc_check", ["-gencode", "arch=compute_100a,code=sm_100a", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "paged_kv_cache_333_b200", "csrc")]),
])
def test_tcgen05_operands_match_cutlass(tmp_path, name, flags):
    inc, nvcc = _cutlass_include(), _nvcc()
    if not inc or not nvcc:
        pytest.skip("nvcc or a CUTLASS include tree is not available")
    exe = str(tmp_path / name)
    subprocess.run([nvcc, "-std=c++17", "--expt-relaxed-constexpr", *flags, "-I", inc, "-o", exe,
                    os.path.join(HERE, name + ".cu")], check=True, timeout=600, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout
    assert "MISMATCH" not in r.stdout

"""The C ABI from a plain C program on the GPU: tests/c_gpu_parity.c
allocates with cudaMalloc, calls the relayouts, the reduce-scatter and the
all-gather on its own stream, and compares every result bit for bit with the
C oracle it links (no Python or torch on that path).  The compile step also
runs without a GPU."""
import os
import shutil
import subprocess

import pytest

from ragged_reduce_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_root():
    nvcc = shutil.which(os.environ.get("NVCC", "nvcc"))
    if not nvcc:
        pytest.skip("nvcc not on PATH (CUDA headers and libcudart not located)")
    return os.path.dirname(os.path.dirname(os.path.realpath(nvcc)))


def _build(tmp_path, name="c_gpu_parity"):
    import oracle
    cuda = _cuda_root()
    exe = str(tmp_path / name)
    lib_dir = os.path.dirname(_abi.LIB_PATH)
    oracle.load()  # builds the oracle library if it is missing or stale
    oracle_dir = os.path.dirname(oracle.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    os.path.join(ROOT, "tests", name + ".c"),
                    "-L", lib_dir, "-l:libh3rr.so", f"-Wl,-rpath,{lib_dir}",
                    "-L", oracle_dir, "-l:libh3oracle.so", f"-Wl,-rpath,{oracle_dir}",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe], check=True)
    return exe


def test_c_gpu_program_compiles(tmp_path):
    assert os.path.exists(_build(tmp_path))


@pytest.mark.gpu
def test_c_gpu_program_matches_oracle(tmp_path):
    out = subprocess.run([_build(tmp_path)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c gpu parity ok" in out.stdout


def test_c_device_reset_program_compiles(tmp_path):
    assert os.path.exists(_build(tmp_path, "c_device_reset"))


@pytest.mark.gpu
def test_calls_work_again_after_device_reset(tmp_path):
    """tests/c_device_reset.c: the bulk relayout (shared-memory opt-in) and
    the allocation-free staged relayout (static window address) before and
    after cudaDeviceReset, each against the C oracle."""
    out = subprocess.run([_build(tmp_path, "c_device_reset")], capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c device reset ok" in out.stdout

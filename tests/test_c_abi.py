"""The C ABI used from plain C, without Python in the loop: tests/c_abi/abi_client.c
is compiled with gcc against include/safedit.h and linked with libsafedit.so,
the CUDA runtime and the oracle library (test infrastructure).  On the CPU it
runs the host-side argument checks; on a GPU it also runs one SRSU attention
(plain, tail-balanced with a caller workspace and with the library's fixed
array, and with kept masks), one mask check and one SW-CFG call against the
oracle."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _client(tmp_path):
    from spatially_adaptive_dit_b200 import build
    from oracle import build_oracle
    build.build()
    build_oracle.build()
    pkg, orc = os.path.join(ROOT, "spatially_adaptive_dit_b200"), os.path.join(ROOT, "oracle")
    cudalib = os.path.join(CUDA, "lib64")
    exe = str(tmp_path / "abi_client")
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", os.path.join(ROOT, "tests", "c_abi", "abi_client.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", pkg, "-lsafedit", "-L", orc, "-loracle", "-L", cudalib, "-lcudart", "-lm",
           f"-Wl,-rpath,{pkg}:{orc}:{cudalib}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_client_builds_and_host_checks(tmp_path):
    exe = _client(tmp_path)
    r = subprocess.run([exe, "--abi"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi checks: ok" in r.stdout


@pytest.mark.gpu
def test_c_client_on_gpu(tmp_path):
    exe = _client(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c client ok" in r.stdout

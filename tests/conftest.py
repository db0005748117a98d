import os
import shutil
import subprocess
import sys
import warnings

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def host_build():
    """Compiler of the host-emulation drivers: build(d, exe_name, main_cpp,
    ubsan=True) compiles tests/host_emulation/<main_cpp> against the kernel
    header the test wrote into d, under AddressSanitizer (and UBSan unless
    ubsan=False), and returns (exe path, env for running it).  Without the
    sanitizer runtime it builds plainly at -O2 and says so."""
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    shim = os.path.join(ROOT, "tests", "host_emulation")

    def build(d, exe_name, main_cpp, ubsan=True):
        exe = d / exe_name
        base = ["-std=c++20", "-pthread", "-I", str(d), "-I", shim, "-o", str(exe), os.path.join(shim, main_cpp)]
        san = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all"] if ubsan else ["-fsanitize=address"]
        r = subprocess.run([cxx, "-O1", "-g"] + san + ["-fno-omit-frame-pointer"] + base, capture_output=True,
                           text=True)
        if r.returncode != 0:
            warnings.warn(f"{main_cpp}: built without sanitizers ({r.stderr.strip()[-200:]})")
            r = subprocess.run([cxx, "-O2"] + base, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-3000:]
        return exe, dict(os.environ, ASAN_OPTIONS="detect_leaks=0:abort_on_error=1")

    return build

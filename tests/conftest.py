import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_addoption(parser):
    parser.addoption("--runslow", action="store_true", default=False,
                     help="also run the exhaustive (slow) checks")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running; runs with --runslow")


def pytest_collection_modifyitems(config, items):
    if config.getoption("--runslow"):
        return
    skip = pytest.mark.skip(reason="exhaustive check: pass --runslow")
    for item in items:
        if "slow" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def pins_lib():
    """Test-only C helpers linked with the oracle (built with gcc here)."""
    import ctypes as C
    out_dir = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out_dir, exist_ok=True)
    so = os.path.join(out_dir, f"pins_{os.getpid()}.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-mf16c", "-msse4.1",
                    "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
                    os.path.join(ROOT, "tests", "csrc", "oracle_pins.c"),
                    os.path.join(ROOT, "oracle", "kvc_oracle.c"), "-o", so, "-lm"],
                   check=True)
    lib = C.CDLL(so)
    os.unlink(so)
    lib.pin_f16_directed.restype = C.c_uint64
    lib.pin_f16_directed.argtypes = [C.c_uint32, C.c_uint32, C.c_int,
                                     C.POINTER(C.c_uint32)]
    lib.pin_f16_directed_mt.restype = C.c_uint64
    lib.pin_f16_directed_mt.argtypes = [C.c_uint32, C.c_uint32, C.c_int, C.c_int,
                                        C.c_int, C.POINTER(C.c_uint32)]
    lib.map_f32_to_bf16.argtypes = [C.c_void_p, C.c_uint64, C.c_void_p]
    lib.map_f16_to_f32.argtypes = [C.c_void_p, C.c_uint64, C.c_void_p]
    return lib

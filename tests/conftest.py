import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU oracle case")


@pytest.fixture(scope="session")
def geometry_checker(tmp_path_factory):
    """Host build of tests/geometry_check.cu (the kernels' index arithmetic, csrc/geometry.cuh)."""
    exe = str(tmp_path_factory.mktemp("geom") / "geometry_check")
    subprocess.run(["nvcc", "-std=c++17", "-O1", "-x", "cu", "-I", os.path.join(ROOT, "sub_quadratic_two_squad_b200", "csrc"),
                    os.path.join(ROOT, "tests", "geometry_check.cu"), "-o", exe], check=True)
    return exe

import os
import sys

import pytest

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
for p in (ROOT, TESTS):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def _built_libs():
    """Build the generator and layer libraries once if they are missing (nvcc, seconds)."""
    import synth

    if not (os.path.exists(synth.HOST_LIB) and os.path.exists(synth.CUDA_LIB)):
        synth.build()
    lib = os.path.join(ROOT, "sparse_moe_expert_fp32_b200", "libmoe_b200.so")
    if not os.path.exists(lib):
        import subprocess

        subprocess.run([sys.executable, os.path.join(ROOT, "sparse_moe_expert_fp32_b200", "build.py")],
                       check=True)
    yield

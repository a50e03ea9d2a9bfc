import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    # build what the tests load (no-ops when up to date): the oracle and the
    # input generator with gcc, libgqa.so with nvcc
    import oracle
    import synth
    from kv_cache_02_b200 import build

    oracle.build()
    synth.build()
    build.build()

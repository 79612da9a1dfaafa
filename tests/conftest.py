import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size case (minutes)")
    # A fresh checkout has no built libraries (they are not committed): build them once,
    # as __graft_entry__.build() does, so that the package and the oracle import.
    if not os.path.exists(os.path.join(ROOT, "combine_moe_plan_03_b200", "libmoe.so")):
        import __graft_entry__
        __graft_entry__.build()

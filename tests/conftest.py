import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# In-tree libraries the tests load; a fresh checkout has none of them (they
# are build products), so the session builds whatever is missing first.
_LIBRARIES = [
    os.path.join(ROOT, "block_sparse_flashattention_ssa_b200", "libssa.so"),
    os.path.join(ROOT, "oracle", "liboracle.so"),
    os.path.join(ROOT, "synth", "libsynth.so"),
]


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    if not all(os.path.exists(p) for p in _LIBRARIES):
        import __graft_entry__

        __graft_entry__.build()

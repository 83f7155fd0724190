import atexit
import os
import shutil
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


# generated-kernel cubins of this session go to a temporary directory (the
# planner tests compile many plans; a persistent cache would only grow)
if "CGTP_JIT_CACHE" not in os.environ:
    _cache = tempfile.mkdtemp(prefix="cgtp_jit_")
    os.environ["CGTP_JIT_CACHE"] = _cache
    atexit.register(shutil.rmtree, _cache, True)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (runs on a B200)")

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


if os.environ.get("GQA_DECODE_CHECKED") == "1":
    import pytest

    @pytest.fixture(autouse=True)
    def _no_failed_index_check(request):
        """Under the checked build, every GPU test ends with no failed index
        check recorded."""
        yield
        if request.node.get_closest_marker("gpu") is None:
            return
        import torch
        if not torch.cuda.is_available():
            return
        import gqa_split_kv_decode_b200 as gk
        assert gk.checked_build()
        assert gk.bounds_report() is None, "an index check failed during this test"

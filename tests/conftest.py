import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(autouse=True)
def _workspace_error_word(request, monkeypatch):
    """Every workspace a GPU test hands to the library is checked afterwards:
    its error word must be clear (no expired bounded wait, no unexpected
    out-of-range mask value). Tests that expect a flag read and clear it."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import torch
    if not torch.cuda.is_available():
        yield
        return
    from kernelized_linear_attention_phi_b200 import binding
    made = []
    orig = binding.workspace

    def tracking(*a, **k):
        ws = orig(*a, **k)
        made.append(ws)
        return ws

    monkeypatch.setattr(binding, "workspace", tracking)
    yield
    for ws in made:
        status, flags = binding.la_last_error(ws)
        assert flags == 0, f"workspace error word {flags:#x} ({binding.STATUS_NAMES.get(status)})"

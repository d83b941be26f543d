import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")


@pytest.fixture
def golden():
    import json

    def load(name):
        with open(os.path.join(GOLDEN, name)) as f:
            return json.load(f)
    return load


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="needs a CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def assert_parity(got, ref, max_rel=1e-2, mean_abs=1e-3, what=""):
    """The floating-point bar: max|err| <= max_rel * max|ref| and mean|err| <= mean_abs."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mref = float(np.max(np.abs(ref)))
    assert err.max() <= max_rel * mref, f"{what}: max err {err.max():.3e} > {max_rel} * {mref:.3e}"
    assert err.mean() <= mean_abs, f"{what}: mean err {err.mean():.3e} > {mean_abs}"
    return float(err.max() / max(mref, 1e-300)), float(err.mean())

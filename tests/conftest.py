import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def read_block_pattern(path):
    """Parse a 'head block : key blocks' fixture into {(h, i): [j, ...]}."""
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split(":")
            h, i = (int(x) for x in lhs.split())
            rows[(h, i)] = [int(x) for x in rhs.split()]
    return rows


# ---------------------------------------------------------------- GPU helpers

# Parity bar against the fp64 oracle (bf16 outputs, unit-normal inputs).
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


def parity(got, want, max_tol=MAX_ABS_TOL, mean_tol=MEAN_ABS_TOL):
    """Compare a bf16/fp32 result (torch or numpy) with fp64 oracle values."""
    import numpy as np
    import torch

    if isinstance(got, torch.Tensor):
        got = got.detach().double().cpu().numpy()
    got = np.asarray(got, dtype=np.float64).reshape(np.shape(want))
    err = np.abs(got - np.asarray(want, dtype=np.float64))
    assert np.isfinite(got).all(), "non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= max_tol and mean <= mean_tol, f"max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


@pytest.fixture
def s2gpu():
    """The binding, with the device flags cleared before and checked after."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_heterogeneous_block_s2_b200 import s2attn

    s2attn.set_wait_timeout_ns(500_000_000)
    s2attn.device_status(reset=True)
    yield s2attn
    rc, flags = s2attn.device_status(reset=True)
    s2attn.set_wait_timeout_ns(2_000_000_000)
    assert rc == 0, f"device flags {flags:#x} after test"

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


# Achieved errors of the GPU parity checks; written as JSON lines to the file named by the
# SD_PARITY_LOG environment variable at the end of the session (nothing is written without it).
PARITY_RECORDS = []


def record_parity(name, **values):
    PARITY_RECORDS.append(dict(name=name, **{k: float(v) for k, v in values.items()}))


def pytest_sessionfinish(session, exitstatus):
    path = os.environ.get("SD_PARITY_LOG")
    if path and PARITY_RECORDS:
        import json
        with open(path, "w") as f:
            for r in PARITY_RECORDS:
                f.write(json.dumps(r) + "\n")


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device for -m gpu tests; fails (never skips) when there is none."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    from unet_latent_attention_b200 import build
    build.build()
    return torch.device("cuda:0")


def max_abs_mean_abs(a, b):
    import numpy as np
    d = np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


def rel_err(gpu, ref):
    """Norm-wise relative error max|gpu - ref| / max|ref|."""
    import numpy as np
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-300))

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def load_golden(name):
    """Parse a tests/golden/*.txt fixture: '# ' comments, '[section]' headers,
    whitespace-separated numbers (inf/-inf allowed)."""
    import numpy as np

    sections, cur = {}, None
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("[") and line.endswith("]"):
                cur = line[1:-1]
                sections[cur] = []
                continue
            sections[cur].append([float(x) for x in line.split()])
    return {k: np.array(v, dtype=np.float64) for k, v in sections.items()}

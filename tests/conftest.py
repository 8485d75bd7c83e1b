import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # temporary files of the tests (tmp_path) stay inside the repository
    if not config.option.basetemp:
        config.option.basetemp = str(ROOT / ".pytest_tmp")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) where no device exists, so the CPU
    # suite can run with or without the marker filter.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def rel_l2(x, ref):
    """||x - ref|| / max(||ref||, 1e-30) over the whole array."""
    import numpy as np
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def max_rel_l2_per_slice(x, ref, slice_axes):
    """Tolerance measure: the worst relative L2 error over (sequence, head) slices.

    ``slice_axes`` are the axes that index slices; the others are reduced.
    """
    import numpy as np
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    other = tuple(a for a in range(x.ndim) if a not in slice_axes)
    num = np.sqrt(((x - ref) ** 2).sum(axis=other))
    den = np.maximum(np.sqrt((ref ** 2).sum(axis=other)), 1e-30)
    return float((num / den).max())


def max_rel_l2_per_window(x, ref, window=64):
    """Worst relative L2 error over token windows of one sequence.

    ``x`` and ``ref`` are [tokens, heads, dv] for ONE sequence, tokens counted
    from the sequence start.  Each (window, head) block of ``window`` tokens
    (the last one ragged) is compared on its own, so an error confined to one
    chunk is not diluted by the rest of a long sequence.
    """
    import numpy as np
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    T = x.shape[0]
    worst = 0.0
    for a in range(0, T, window):
        d = x[a:a + window] - ref[a:a + window]
        num = np.sqrt((d ** 2).sum(axis=(0, 2)))
        den = np.maximum(np.sqrt((ref[a:a + window] ** 2).sum(axis=(0, 2))), 1e-30)
        worst = max(worst, float((num / den).max()))
    return worst

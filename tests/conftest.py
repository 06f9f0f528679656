import json
import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # Without a GPU, tests marked gpu are skipped rather than failing on import.
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


def pytest_terminal_summary(terminalreporter):
    """Decision and boundary-event counts of the named parity checks."""
    mod = sys.modules.get("_parity")
    recs = getattr(mod, "RECORDS", None)
    if not recs:
        return
    terminalreporter.write_sep("-", "parity decisions and boundary events")
    for r in recs:
        terminalreporter.write_line(f"{r['check']}: {r['decisions']} decisions, {r['boundary_events']} boundary events")
    out = os.environ.get("UNO_PARITY_EVENTS")
    if out:
        Path(out).write_text(json.dumps(recs, indent=1) + "\n")

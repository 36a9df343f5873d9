import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """The 1-ulp bf16 flips the parity checks counted, and how often the mailbox
    consumer met unwritten slots in the concurrent rounds (GPU runs only)."""
    race = sys.modules.get("test_gpu_mailbox_race")
    waits = getattr(race, "WAITS", None) if race else None
    if waits:
        terminalreporter.write_line("mailbox rounds with producers running: " + "; ".join(
            f"{c}: {w} of {n} slot groups first read unwritten" for c, w, n in waits))
    mod = sys.modules.get("_parity")
    flips = getattr(mod, "FLIPS", None) if mod else None
    if not flips:
        return
    total = sum(f for _, f, _ in flips)
    elems = sum(n for _, _, n in flips)
    worst = max(flips, key=lambda t: t[1] / max(t[2], 1))
    terminalreporter.write_line(
        f"bf16 ulp checks: {len(flips)} arrays, {total} one-ulp flips in {elems} elements "
        f"({total / max(elems, 1):.2e}); largest share {worst[1]}/{worst[2]} in {worst[0]}")

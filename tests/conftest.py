import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


# Fitted-map gains and the output bars each parity case applied (filled by the GPU parity tests,
# printed at the end of the run so that every relaxation of a bar is visible).
_PARITY_LOG = pytest.StashKey[list]()


@pytest.fixture(scope="session")
def parity_log(request):
    return request.config.stash.setdefault(_PARITY_LOG, [])


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    rows = config.stash.get(_PARITY_LOG, [])
    if not rows:
        return
    terminalreporter.write_sep("-", "end-to-end output bars: fitted-map gain and the bar applied per head")
    terminalreporter.write_line(f"{'case':34s} {'head':>4s} {'gain_inf':>9s} {'gain_2':>8s} {'e2e bar':>11s} "
                                f"{'quality slack':>13s} {'err gpu':>9s} {'err oracle':>10s}")
    for r in rows:
        terminalreporter.write_line(f"{r['case'][:34]:34s} {r['head']:4d} {r['gain_inf']:9.3f} {r['gain_2']:8.3f} "
                                    f"{r['e2e']:>11s} {r['slack']:13.2e} {r['e_gpu']:9.4f} {r['e_orc']:10.4f}")

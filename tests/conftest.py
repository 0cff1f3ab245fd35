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
    terminalreporter.write_line("e2e max-abs / rel-L2: the corrected output against the oracle's, whatever bar applied "
                                "(the flat bar: 2e-2 / 1e-2 bf16, 1e-4 fp32); err: mean error against exact rows")
    terminalreporter.write_line(f"{'case':34s} {'head':>4s} {'gain_inf':>9s} {'gain_2':>8s} {'e2e bar':>11s} "
                                f"{'e2e max-abs':>11s} {'e2e rel-L2':>10s} {'slack':>9s} {'err gpu':>9s} "
                                f"{'err oracle':>10s}")
    for r in rows:
        terminalreporter.write_line(f"{r['case'][:34]:34s} {r['head']:4d} {r['gain_inf']:9.3f} {r['gain_2']:8.3f} "
                                    f"{r['e2e']:>11s} {r['e2e_abs']:11.3e} {r['e2e_rl2']:10.3e} {r['slack']:9.2e} "
                                    f"{r['e_gpu']:9.4f} {r['e_orc']:10.4f}")

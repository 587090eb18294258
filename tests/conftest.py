import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def synth_mod():
    import synth
    synth.build()
    return synth


# Parity records: counts and errors the GPU parity tests measured (exempt mask
# rows per configuration, rows compared, error maxima), printed in the terminal
# summary so that a quiet run still reports them.
_PARITY_RECORDS = []


@pytest.fixture
def parity_record():
    def add(what, **fields):
        _PARITY_RECORDS.append((what, fields))
    return add


def pytest_terminal_summary(terminalreporter):
    if not _PARITY_RECORDS:
        return
    terminalreporter.section("parity records")
    for what, fields in _PARITY_RECORDS:
        body = ", ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}"
                         for k, v in fields.items())
        terminalreporter.write_line(f"{what}: {body}")

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)

_ORACLE_POOL = None


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU oracle run")


def pytest_collection_finish(session):
    """Start the oracle's long trajectories in worker processes once the selected tests
    are known, before any of them touches the GPU (see tests/oracle_jobs.py)."""
    global _ORACLE_POOL
    if session.config.option.collectonly:
        return
    if any("oracle_refs" in getattr(item, "fixturenames", ()) for item in session.items):
        from oracle_jobs import OraclePool
        _ORACLE_POOL = OraclePool()


def pytest_sessionfinish(session, exitstatus):
    if _ORACLE_POOL is not None:
        _ORACLE_POOL.shutdown()


@pytest.fixture(scope="session")
def oracle_refs():
    global _ORACLE_POOL
    if _ORACLE_POOL is None:
        from oracle_jobs import OraclePool
        _ORACLE_POOL = OraclePool()
    return _ORACLE_POOL

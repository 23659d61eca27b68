import pathlib
import sys

ROOT = pathlib.Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionstart(session):
    # tests/test_oracle_mutations.py runs the pins in a child process with a mistake
    # planted in the oracle (in memory only)
    import os
    index = os.environ.get("HRA_ORACLE_MUTATION")
    if index is not None:
        import oracle_mutations
        oracle_mutations.apply(int(index))

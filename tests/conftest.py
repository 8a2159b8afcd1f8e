import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _library_is_stale() -> bool:
    pkg = os.path.join(ROOT, "hierarchical_sparse_attention_zha_b200")
    lib = os.path.join(pkg, "libzha.so")
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    srcs = [os.path.join(pkg, "csrc", f) for f in os.listdir(os.path.join(pkg, "csrc"))]
    srcs.append(os.path.join(ROOT, "include", "zha.h"))
    return any(os.path.getmtime(s) > t for s in srcs)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")
    if _library_is_stale():
        from hierarchical_sparse_attention_zha_b200 import build
        build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


# Tie report: every parity case that compares kept sets with the oracle records
# its RouteReport here; the counts are printed at the end of the session (also
# under -q), so a run's log says how many disagreements were ties.
_PARITY_ROWS: list = []


@pytest.fixture(scope="session")
def parity_log():
    def record(case: str, report) -> None:
        _PARITY_ROWS.append((case, report.summary()))
    return record


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not _PARITY_ROWS:
        return
    tr = terminalreporter
    tr.section("route parity vs oracle (ties within 1e-5 are counted, not failed)")
    tot = {"heads": 0, "levels_compared": 0, "ties": 0, "hard": 0}
    for case, s in _PARITY_ROWS:
        tr.write_line(f"{case}: heads {s['heads']} levels {s['levels_compared']} ties {s['ties']} "
                      f"hard {s['hard']} exact-heads {s['exact_heads']}")
        for k in tot:
            tot[k] += s[k]
    tr.write_line(f"TOTAL: heads {tot['heads']} levels {tot['levels_compared']} ties {tot['ties']} "
                  f"hard {tot['hard']}")

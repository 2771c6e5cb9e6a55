import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


# workloads whose full-size outputs the summary lists
_SUMMARY_PREFIXES = ("tiny_f32", "detr_encoder_f32", "detr_decoder_bf16", "encoder_1024_bf16",
                     "stress_1080p_k8_bf16", "bf16 grad_value", "fused bf16 grad_value", "no-alloc")


def pytest_terminal_summary(terminalreporter):
    """Normwise and elementwise errors of the full-size parity checks of
    this run (both metrics of tests/gpu_util.py assert_close)."""
    gu = sys.modules.get("tests.gpu_util")
    recs = [r for r in getattr(gu, "RECORDS", []) if r[0].startswith(_SUMMARY_PREFIXES)]
    if not recs:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity against the oracle: normwise / elementwise error")
    for what, e, ee in recs:
        tr.write_line(f"{what:60s} {e:9.2e} {ee:9.2e}")

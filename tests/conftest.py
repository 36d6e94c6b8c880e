import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle


# Attention parity records of the GPU tests: case -> max abs error, max rel error (over
# |oracle| >= 1e-3), worst error / bound ratio and elements compared.  With
# PAGEDKV_PARITY_OUT set, the session writes them there as JSON.
PARITY = {}


def record_parity(what, max_abs, max_rel, worst_ratio, n):
    key = what or "case"
    k, i = key, 1
    while k in PARITY:
        i += 1
        k = "%s #%d" % (key, i)
    PARITY[k] = {"max_abs": max_abs, "max_rel": max_rel, "worst_err_over_bound": worst_ratio,
                 "elements": n}


def pytest_sessionfinish(session, exitstatus):
    out = os.environ.get("PAGEDKV_PARITY_OUT")
    if out and PARITY:
        d = os.path.dirname(out)
        if d:
            os.makedirs(d, exist_ok=True)
        rec = {"bound": "|gpu - oracle| <= 2e-3 + 1e-2 |oracle| per element",
               "cases": len(PARITY),
               "max_abs_over_all": max(v["max_abs"] for v in PARITY.values()),
               "max_rel_over_all": max(v["max_rel"] for v in PARITY.values()),
               "worst_err_over_bound_over_all": max(v["worst_err_over_bound"]
                                                    for v in PARITY.values()),
               "per_case": PARITY}
        with open(out, "w") as f:
            json.dump(rec, f, indent=1, sort_keys=True)

"""Shared helpers of the GPU parity tests: tolerances and input subsetting."""
import json
import os

import numpy as np

from workloads import subset_users  # noqa: F401  (re-exported for the tests)

# Acceptance bars: fp32 max abs error; bf16 max abs relative to max|ref| and
# the mean relative error sum|g - r| / sum|r|.
F32_MAX_ABS = 1e-4
BF16_MAX_REL = 1e-2
BF16_MEAN_REL = 2e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    return {
        "max_abs": float(diff.max()) if diff.size else 0.0,
        "max_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "mean_rel": float(diff.sum() / max(np.abs(ref).sum(), 1e-300)),
    }


def assert_parity(got, ref, dtype, what=""):
    e = errors(got, ref)
    _log(what, e)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    if dtype == "f32":
        assert e["max_abs"] <= F32_MAX_ABS, f"{what}: {e}"
    else:
        assert e["max_abs"] <= BF16_MAX_REL * e["max_ref"], f"{what}: {e}"
        assert e["mean_rel"] <= BF16_MEAN_REL, f"{what}: {e}"
    return e


def _log(what, e):
    path = os.environ.get("REST_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], "what": what,
                                **e}) + "\n")

"""Shared helpers of the GPU parity tests: tolerances and input subsetting."""
import json
import os

import numpy as np

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


def subset_users(inp: dict, users, with_requests=True) -> dict:
    """The inputs of a subset of users (and their requests), re-packed."""
    users = list(users)
    cu = inp["cu_seqlens"]
    rows = np.concatenate([np.arange(cu[u], cu[u + 1]) for u in users])
    new_cu = np.zeros(len(users) + 1, dtype=np.int32)
    new_cu[1:] = np.cumsum([cu[u + 1] - cu[u] for u in users])
    out = dict(inp, x=inp["x"][rows], ts=inp["ts"][rows], cu_seqlens=new_cu)
    if with_requests:
        ru, rc, cc = inp["req_user"], inp["req_cutoff"], inp["cu_cands"]
        keep = [r for r in range(len(ru)) if ru[r] in users]
        remap = {u: i for i, u in enumerate(users)}
        cand_rows = np.concatenate([np.arange(cc[r], cc[r + 1]) for r in keep]) if keep else np.zeros(0, int)
        ncs = [cc[r + 1] - cc[r] for r in keep]
        new_cc = np.zeros(len(keep) + 1, dtype=np.int32)
        new_cc[1:] = np.cumsum(ncs)
        out.update(req_user=np.array([remap[ru[r]] for r in keep], dtype=np.int32),
                   req_cutoff=np.array([rc[r] for r in keep], dtype=np.int32), cu_cands=new_cc,
                   z=inp["z"][cand_rows], _cand_rows=cand_rows)
    out["_rows"] = rows
    return out


def _log(what, e):
    path = os.environ.get("REST_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], "what": what,
                                **e}) + "\n")

"""The C-ABI library loads, exports what include/rest.h declares, and rejects
invalid arguments on the host before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import shared_prefix_behavior_b200 as R
import workloads as W
from tests.conftest import gpu_available

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rest.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rest_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "rest_encoder_attn" in names and "rest_cross_decode" in names and "rest_rank_request" in names
    lib = ctypes.CDLL(R.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(R.EXPORTS) <= set(names)


def test_static_ws_size_matches_the_header():
    src = open(os.path.join(ROOT, "include", "rest.h")).read()
    m = re.search(r"#define REST_STATIC_WS_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", src)
    assert m, "REST_STATIC_WS_BYTES not found in rest.h"
    assert R.STATIC_WS_BYTES == int(m.group(1)) * int(m.group(2)) * int(m.group(3))


def test_status_strings():
    for code in range(9):
        assert R.library().rest_status_string(code)
    assert R.library().rest_status_string(0) == b"ok"


FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host


def _heads(taus, d, base=10000.0):
    taus = np.asarray(taus, dtype=np.int64)
    return taus, R.Heads(d, len(taus), d // len(taus), taus.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), base)


def _batch(cu):
    cu = np.asarray(cu, dtype=np.int32)
    return cu, R.Batch(len(cu) - 1, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))


def _layer(d, dff=0, gates=0):
    return R.EncLayer(FAKE, FAKE, FAKE if dff else None, FAKE if dff else None, FAKE, FAKE, FAKE, FAKE, 0.1, 0.1, dff,
                      gates)


def _enc(dt=R.REST_BF16, taus=(0, 0, 1, 64), d=64, cu=(0, 10, 30), layers=None, l_switch=0, x=FAKE, ts=FAKE,
         out=FAKE, ws=FAKE, ws_bytes=1 << 40, base=10000.0):
    t, hs = _heads(taus, d, base)
    c, b = _batch(cu)
    if layers is None:
        layers = [_layer(d, 192)]
    arr = (R.EncLayer * max(1, len(layers)))(*layers)
    return R.library().rest_encoder_attn(dt, ctypes.byref(hs), ctypes.byref(b), x, ts, arr, len(layers), l_switch,
                                         out, ws, ws_bytes, None, None)


def _reqs(u, c, cc):
    u, c, cc = (np.asarray(a, dtype=np.int32) for a in (u, c, cc))
    P = ctypes.POINTER(ctypes.c_int32)
    return (u, c, cc), R.Requests(len(u), u.ctypes.data_as(P), c.ctypes.data_as(P), cc.ctypes.data_as(P))


def _dec_call(dt=R.REST_BF16, cu=(0, 10, 30), req=((0, 1), (10, 5), (0, 4, 6)), K=3, d=64, ws_bytes=1 << 40,
              wq=FAKE):
    t, hs = _heads((0, 0, 1, 64), d)
    c, b = _batch(cu)
    keep, rq = _reqs(*req)
    dp = R.DecParams(K, wq, FAKE, FAKE)
    return R.library().rest_cross_decode(dt, ctypes.byref(hs), ctypes.byref(b), FAKE, ctypes.byref(rq), FAKE,
                                         ctypes.byref(dp), FAKE, FAKE, ws_bytes, None, None)


INVALID, UNSUPPORTED, WORKSPACE, NO_DEVICE = 1, 3, 6, 7


@pytest.mark.parametrize("kw,code", [
    (dict(d=60), INVALID),                       # d != n_heads * head_dim
    (dict(taus=(0, 0, -1, 64)), INVALID),        # negative granularity
    (dict(taus=(0, 0, 0)), INVALID),             # 64 / 3 heads
    (dict(dt=7), INVALID),
    (dict(cu=(1, 10)), INVALID),                 # cu_seqlens[0] != 0
    (dict(cu=(0, 10, 5)), INVALID),              # decreasing
    (dict(l_switch=2), INVALID),                 # l_switch > n_layers
    (dict(x=FAKE + 4), INVALID),                 # misaligned
    (dict(ts=None), INVALID),
    (dict(layers=[_layer(64, 100)]), INVALID),   # d_ff not a multiple of 64
    (dict(layers=[_layer(64, 192, 3)]), INVALID),  # no such gate variant
    (dict(base=-1.0), INVALID),
    (dict(d=4 * 24, taus=(0, 0, 1, 64)), UNSUPPORTED),  # head_dim 24
    (dict(ws_bytes=1000), WORKSPACE),
    (dict(ws=None), WORKSPACE),
])
def test_encoder_rejects_invalid_arguments(kw, code):
    assert _enc(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(req=((0, 2), (10, 5), (0, 4, 6))), INVALID),   # user out of range
    (dict(req=((0, 1), (11, 5), (0, 4, 6))), INVALID),   # cutoff > L_u
    (dict(req=((0, 1), (0, 5), (0, 4, 6))), INVALID),    # cutoff 0
    (dict(req=((0, 1), (10, 5), (0, 4, 3))), INVALID),   # cu_cands decreasing
    (dict(req=((0, 1), (10, 5), (1, 4, 6))), INVALID),   # cu_cands[0] != 0
    (dict(K=0), INVALID),
    (dict(K=9), INVALID),
    (dict(wq=None), INVALID),
    (dict(ws_bytes=16), WORKSPACE),
])
def test_decoder_rejects_invalid_arguments(kw, code):
    assert _dec_call(**kw) == code


def test_empty_work_is_a_successful_noop():
    assert _enc(cu=(0,)) == 0                           # no users
    assert _enc(cu=(0, 0, 0)) == 0                      # users without tokens
    assert _dec_call(req=((0, 1), (10, 5), (0, 0, 0))) == 0   # no candidates
    assert _dec_call(req=((), (), (0,))) == 0            # no requests


@pytest.mark.skipif(gpu_available(), reason="checks the no-GPU status")
def test_valid_call_without_gpu_reports_no_device():
    assert _enc() == NO_DEVICE
    assert _dec_call() == NO_DEVICE


def test_workspace_size_grows_with_the_batch():
    for i in (0, 1, 4):
        w = W.workload(i)
        cu = np.concatenate([[0], np.cumsum(w.lengths)]).astype(np.int32)
        cc = np.concatenate([[0], np.cumsum(w.req_ncand)]).astype(np.int32)
        nb = R.workspace_size(R.REST_BF16 if w.dtype == "bf16" else R.REST_F32, w.taus, w.d, cu, (),
                              (w.req_user, w.req_cutoff, cc), 3)
        e = 2 if w.dtype == "bf16" else 4
        assert nb >= w.total_cands * 3 * w.d * (2 * e + 4)


def test_rank_request_host_validation():
    t, hs = _heads((0, 0, 1, 64), 64)
    c, b = _batch((0, 10, 30))
    keep, rq = _reqs((0, 1), (10, 21), (0, 4, 6))   # cutoff 21 > 20
    arr = (R.EncLayer * 1)(_layer(64, 192))
    dp = R.DecParams(3, FAKE, FAKE, FAKE)
    st = R.library().rest_rank_request(R.REST_BF16, ctypes.byref(hs), ctypes.byref(b), FAKE, FAKE, arr, 1, 0,
                                       ctypes.byref(rq), FAKE, ctypes.byref(dp), FAKE, FAKE, FAKE, 1 << 40, None, None)
    assert st == INVALID


def _score_call(dt=R.REST_BF16, d=256, K=3, n=5, d_ff=704, z=FAKE, y=FAKE, f=FAKE, score=FAKE, ws=FAKE,
                ws_bytes=1 << 30, null_params=False, w13=FAKE):
    sp = R.ScoreParams(w13, FAKE, FAKE, FAKE, FAKE, 0.5, d_ff)
    return R.library().rest_score_head(dt, d, K, n, z, y, None if null_params else ctypes.byref(sp), f, score, ws,
                                       ws_bytes, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=0), 1), (dict(d=2048), 1), (dict(d=100), 1), (dict(K=0), 1), (dict(K=9), 1), (dict(n=-1), 1),
    (dict(d_ff=0), 1), (dict(d_ff=100), 1), (dict(dt=7), 1), (dict(null_params=True), 1), (dict(z=None), 1),
    (dict(y=FAKE + 4), 1), (dict(f=None), 1), (dict(score=None), 1), (dict(w13=None), 1),
    (dict(ws=None), 6), (dict(ws_bytes=100), 6),
])
def test_score_head_rejects_invalid_arguments(kw, code):
    assert _score_call(**kw) == code


def test_score_head_workspace_and_empty_batch():
    out = ctypes.c_size_t(0)
    assert R.library().rest_score_workspace_size(R.REST_BF16, 256, 3, 1000, 704, ctypes.byref(out)) == 0
    assert out.value >= 1000 * 3 * (256 + 704) * 2
    assert _score_call(n=0, z=None, y=None, f=None, score=None, ws=None) == 0  # nothing to do


@pytest.mark.skipif(gpu_available(), reason="the no-device status needs a host without a GPU")
def test_score_head_without_gpu_reports_no_device():
    assert _score_call() == 7


# ------------------------------------------------------------ append-only cache

def _append(cu=(0, 4, 6), cap=(16, 8), length=(10, 2), rows=None, t_first=(100, 200), t_last=(150, 250),
            n_layers=1, kv=FAKE, h=None, x=FAKE, ws_bytes=1 << 40, no_cache=False):
    t, hs = _heads((0, 0, 1, 64), 64)
    c, b = _batch(cu)
    layers = [_layer(64, 192) for _ in range(n_layers)]
    arr = (R.EncLayer * max(1, n_layers))(*layers)
    capv = np.asarray(cap, dtype=np.int64)
    cu_cap = np.zeros(len(capv) + 1, dtype=np.int32)
    cu_cap[1:] = np.cumsum(capv)
    ln = np.asarray(length, dtype=np.int32)
    tf, tl = np.asarray(t_first, dtype=np.int64), np.asarray(t_last, dtype=np.int64)
    kp = (ctypes.c_void_p * max(1, n_layers))(*([kv] * n_layers))
    P32, P64 = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    cache = R.KVCacheStruct(kp, kp, h, int(cu_cap[-1]) if rows is None else rows, cu_cap.ctypes.data_as(P32),
                            ln.ctypes.data_as(P32), tf.ctypes.data_as(P64), tl.ctypes.data_as(P64))
    return R.library().rest_encoder_append(R.REST_BF16, ctypes.byref(hs), ctypes.byref(b), x, FAKE, arr, n_layers,
                                           0, None if no_cache else ctypes.byref(cache), FAKE, FAKE, ws_bytes,
                                           None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(no_cache=True), INVALID),
    (dict(length=(13, 2)), INVALID),             # 13 cached + 4 new > 16 rows
    (dict(length=(10, 7)), INVALID),             # 7 + 2 > 8
    (dict(length=(-1, 2)), INVALID),
    (dict(rows=20), INVALID),                    # regions end past the arrays
    (dict(cap=(16, -2)), INVALID),               # decreasing region bounds
    (dict(t_first=(200, 200)), INVALID),         # first timestamp after the last
    (dict(kv=None), INVALID),                    # a layer without cache arrays
    (dict(kv=FAKE + 8), INVALID),                # misaligned cache array
    (dict(h=FAKE + 4), INVALID),
    (dict(x=FAKE + 2), INVALID),
    (dict(ws_bytes=64), WORKSPACE),
])
def test_append_rejects_invalid_arguments(kw, code):
    assert _append(**kw) == code


def test_append_of_no_tokens_is_a_noop_and_workspace_is_sized():
    assert _append(cu=(0, 0, 0)) == 0
    w = W.workload(1)
    small = R.append_workspace_size(R.REST_BF16, w.taus, w.d, [0, 64, 128], [])
    big = R.append_workspace_size(R.REST_BF16, w.taus, w.d, [0, 4096, 8192], [])
    assert 0 < small < big


@pytest.mark.skipif(gpu_available(), reason="the no-device status needs a host without a GPU")
def test_append_without_gpu_reports_no_device():
    assert _append() == NO_DEVICE


def test_cache_bookkeeping_counts_appended_tokens():
    import torch
    c = R.KVCache([10, 5], n_layers=2, d=64, dtype=torch.float32, device="cpu")
    assert c.rows == 15 and list(c.cu_cap) == [0, 10, 15] and len(c.k) == 2 and c.h is not None
    c.advance([0, 3, 3], np.array([7, 9, 9]))
    assert list(c.len) == [3, 0] and c.t_first[0] == 7 and c.t_last[0] == 9
    c.advance([0, 1, 3], np.array([12, 40, 41]))
    assert list(c.len) == [4, 2] and c.t_first[0] == 7 and c.t_last[0] == 12
    assert c.t_first[1] == 40 and c.t_last[1] == 41


# ------------------------------------------------------------ attention core (training)

def _core(fn="fwd", cu=(0, 10, 30), ptr=FAKE, bad=None, ws_bytes=1 << 40, dt=R.REST_BF16):
    t, hs = _heads((0, 0, 1, 64), 64)
    c, b = _batch(cu)
    lib = R.library()
    # forward: q k v o o_lo lse; backward: q k v o o_lo lse d_o dq dk dv (o_lo may be NULL, not misaligned)
    n = 6 if fn == "fwd" else 10
    args = [ptr] * n
    if bad is not None:
        args[bad] = FAKE + 8 if bad % 2 or bad == 4 else None
    f = lib.rest_attn_forward if fn == "fwd" else lib.rest_attn_backward
    return f(dt, ctypes.byref(hs), ctypes.byref(b), *args, FAKE, ws_bytes, None, None)


@pytest.mark.parametrize("fn,bad", [("fwd", i) for i in range(6)] + [("bwd", i) for i in range(10)])
def test_attention_core_rejects_missing_or_misaligned_pointers(fn, bad):
    assert _core(fn, bad=bad) == INVALID


def test_attention_core_low_part_only_with_bf16():
    assert _core("fwd", dt=R.REST_F32) == INVALID  # o_lo given to an fp32 call


def test_attention_core_workspace_empty_and_no_device():
    assert _core("fwd", ws_bytes=16) == WORKSPACE and _core("bwd", ws_bytes=16) == WORKSPACE
    assert _core("fwd", cu=(0, 0)) == 0 and _core("bwd", cu=(0,)) == 0
    assert _core("fwd", cu=(0, 5, 3)) == INVALID
    assert 0 < R.attn_workspace_size(R.REST_BF16, 8, 32, [0, 64]) < R.attn_workspace_size(R.REST_BF16, 8, 32, [0, 4096])
    if not gpu_available():
        assert _core("fwd") == NO_DEVICE and _core("bwd") == NO_DEVICE


def test_selftest_rejects_invalid_arguments():
    lib = R.library()
    assert lib.rest_selftest_wait_timeout(0, 10**7, FAKE, None) == INVALID       # no CTA
    assert lib.rest_selftest_wait_timeout(2000, 10**7, FAKE, None) == INVALID    # too many
    assert lib.rest_selftest_wait_timeout(4, 10, FAKE, None) == INVALID          # limit too short
    assert lib.rest_selftest_wait_timeout(4, 10**7, None, None) == INVALID       # no status word
    if not gpu_available():
        assert lib.rest_selftest_wait_timeout(4, 10**7, FAKE, None) == NO_DEVICE

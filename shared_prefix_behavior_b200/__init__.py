"""Python binding of the ReST ranking-forward library (librest_b200.so).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels. PyTorch provides device memory and the current stream. There is
no CPU fallback: if the library is missing, importing this package raises.

Entry points (same names as the C ABI in include/rest.h):

* ``rotation_table``  -- rotation index and cos/sin table (ReST §3.2.2, eq. 5)
* ``encoder_attn``    -- encoder T (§3.2, eqs. 3-6)
* ``cross_decode``    -- projection-free, token-specific cross decoder C (§3.3, eqs. 7-8)
* ``rank_request``    -- shared-prefix serving: T once, C for every candidate (§3.5)
* ``encoder_append``  -- T on tokens appended to cached histories (``KVCache``)
* ``score_head``      -- decoder block and candidate score (§3.3.2, eq. 8)
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int, c_int32, c_int64, c_longlong, c_size_t, c_void_p
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librest_b200.so")

REST_F32, REST_BF16 = 0, 1
# attention-sublayer gates (rest_gates): value + output (the DGA layer), output only, Q/K/V + output
GATES = {"vo": 0, "o": 1, "qkvo": 2}
STATUS = {0: "REST_OK", 1: "REST_ERR_INVALID_ARG", 2: "REST_ERR_UNSORTED_TIME", 3: "REST_ERR_UNSUPPORTED",
          4: "REST_ERR_CUDA", 5: "REST_ERR_TIMEOUT", 6: "REST_ERR_WORKSPACE", 7: "REST_ERR_NO_DEVICE",
          8: "REST_ERR_RANGE"}
EXPORTS = ("rest_workspace_size", "rest_rotation_table", "rest_encoder_attn", "rest_cross_decode",
           "rest_rank_request", "rest_status_string", "rest_launch_count", "rest_profile_begin",
           "rest_profile_end", "rest_cross_decode_static_ws", "rest_score_workspace_size", "rest_score_head",
           "rest_append_workspace_size", "rest_encoder_append", "rest_attn_workspace_size", "rest_attn_forward",
           "rest_attn_backward", "rest_selftest_wait_timeout", "rest_static_ws_bytes")


class RestError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib.rest_status_string(status).decode()})")
        self.status = status


class Heads(ctypes.Structure):
    _fields_ = [("d", c_int), ("n_heads", c_int), ("head_dim", c_int), ("tau", POINTER(c_int64)),
                ("rope_base", c_double)]


class Batch(ctypes.Structure):
    _fields_ = [("n_users", c_int), ("cu_seqlens", POINTER(c_int32))]


class EncLayer(ctypes.Structure):
    _fields_ = [("w_qkvgg", c_void_p), ("w_o", c_void_p), ("w_ffn13", c_void_p), ("w_ffn2", c_void_p),
                ("ln_attn_g", c_void_p), ("ln_attn_b", c_void_p), ("ln_ffn_g", c_void_p), ("ln_ffn_b", c_void_p),
                ("alpha_attn", c_float), ("alpha_ffn", c_float), ("d_ff", c_int), ("gates", c_int)]


class DecParams(ctypes.Structure):
    _fields_ = [("K", c_int), ("w_q", c_void_p), ("w_go", c_void_p), ("w_o", c_void_p)]


class ScoreParams(ctypes.Structure):
    _fields_ = [("w_ffn13", c_void_p), ("w_ffn2", c_void_p), ("ln_g", c_void_p), ("ln_b", c_void_p),
                ("w_s", c_void_p), ("b_s", c_float), ("d_ff", c_int)]


class Requests(ctypes.Structure):
    _fields_ = [("n_req", c_int), ("req_user", POINTER(c_int32)), ("req_cutoff", POINTER(c_int32)),
                ("cu_cands", POINTER(c_int32))]


class KVCacheStruct(ctypes.Structure):
    _fields_ = [("k", POINTER(c_void_p)), ("v", POINTER(c_void_p)), ("h", c_void_p), ("rows", c_longlong),
                ("cu_cap", POINTER(c_int32)), ("len", POINTER(c_int32)), ("t_first", POINTER(c_int64)),
                ("t_last", POINTER(c_int64))]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", c_int), ("ms", c_double), ("flops", c_double),
                ("bytes", c_double)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python shared_prefix_behavior_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    lib.rest_workspace_size.argtypes = [c_int, POINTER(Heads), POINTER(Batch), POINTER(EncLayer), c_int,
                                        POINTER(Requests), c_int, POINTER(c_size_t)]
    lib.rest_rotation_table.argtypes = [POINTER(Heads), POINTER(Batch), P, P, P, P, P, c_size_t, P, P]
    lib.rest_encoder_attn.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, P, POINTER(EncLayer), c_int, c_int,
                                      P, P, c_size_t, P, P]
    lib.rest_cross_decode.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, POINTER(Requests), P,
                                      POINTER(DecParams), P, P, c_size_t, P, P]
    lib.rest_cross_decode_static_ws.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, POINTER(Requests), P,
                                                POINTER(DecParams), P, P, P]
    lib.rest_rank_request.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, P, POINTER(EncLayer), c_int, c_int,
                                      POINTER(Requests), P, POINTER(DecParams), P, P, P, c_size_t, P, P]
    lib.rest_score_workspace_size.argtypes = [c_int, c_int, c_int, c_longlong, c_int, POINTER(c_size_t)]
    lib.rest_score_head.argtypes = [c_int, c_int, c_int, c_longlong, P, P, POINTER(ScoreParams), P, P, P, c_size_t,
                                    P, P]
    lib.rest_append_workspace_size.argtypes = [c_int, POINTER(Heads), POINTER(Batch), POINTER(EncLayer), c_int,
                                               POINTER(c_size_t)]
    lib.rest_encoder_append.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, P, POINTER(EncLayer), c_int, c_int,
                                        POINTER(KVCacheStruct), P, P, c_size_t, P, P]
    lib.rest_attn_workspace_size.argtypes = [c_int, POINTER(Heads), POINTER(Batch), POINTER(c_size_t)]
    lib.rest_attn_forward.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, P, P, P, P, P, P, c_size_t, P, P]
    lib.rest_attn_backward.argtypes = [c_int, POINTER(Heads), POINTER(Batch), P, P, P, P, P, P, P, P, P, P, P,
                                       c_size_t, P, P]
    lib.rest_selftest_wait_timeout.argtypes = [c_int, c_longlong, P, P]
    for name in ("rest_selftest_wait_timeout", "rest_workspace_size", "rest_rotation_table", "rest_encoder_attn",
                 "rest_cross_decode",
                 "rest_rank_request", "rest_cross_decode_static_ws", "rest_score_workspace_size", "rest_score_head",
                 "rest_append_workspace_size", "rest_encoder_append", "rest_attn_workspace_size",
                 "rest_attn_forward", "rest_attn_backward"):
        getattr(lib, name).restype = c_int
    lib.rest_status_string.argtypes = [c_int]
    lib.rest_status_string.restype = ctypes.c_char_p
    lib.rest_launch_count.argtypes = [c_int]
    lib.rest_launch_count.restype = c_longlong
    lib.rest_profile_begin.argtypes = []
    lib.rest_profile_begin.restype = None
    lib.rest_profile_end.argtypes = [POINTER(KernelStat), c_int]
    lib.rest_profile_end.restype = c_int
    lib.rest_static_ws_bytes.argtypes = []
    lib.rest_static_ws_bytes.restype = c_size_t
    return lib


_lib = _load()
# the scratch array of rest_cross_decode_static_ws, as the library was built
STATIC_WS_BYTES = int(_lib.rest_static_ws_bytes())


def library() -> ctypes.CDLL:
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise RestError(status, where)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class _Host:
    """Keeps the host arrays of one call alive and builds the ABI structs."""

    def __init__(self, taus, d, rope_base, cu_seqlens, reqs=None):
        self.taus = np.ascontiguousarray(np.asarray(taus, dtype=np.int64))
        n_heads = len(self.taus)
        self.heads = Heads(d, n_heads, d // n_heads, self.taus.ctypes.data_as(POINTER(c_int64)), float(rope_base))
        self.cu = _i32(cu_seqlens)
        self.batch = Batch(len(self.cu) - 1, self.cu.ctypes.data_as(POINTER(c_int32)))
        self.reqs = None
        if reqs is not None:
            self.ru, self.rc, self.cc = _i32(reqs[0]), _i32(reqs[1]), _i32(reqs[2])
            self.reqs = Requests(len(self.ru), self.ru.ctypes.data_as(POINTER(c_int32)),
                                 self.rc.ctypes.data_as(POINTER(c_int32)), self.cc.ctypes.data_as(POINTER(c_int32)))


def _enc_layers(layers: Sequence[dict]):
    arr = (EncLayer * max(1, len(layers)))()
    for i, L in enumerate(layers):
        ffn = L.get("w_ffn13") is not None
        arr[i] = EncLayer(_ptr(L["w_qkvgg"]), _ptr(L["w_o"]), _ptr(L["w_ffn13"]) if ffn else None,
                          _ptr(L["w_ffn2"]) if ffn else None, _ptr(L["ln_attn_g"]), _ptr(L["ln_attn_b"]),
                          _ptr(L["ln_ffn_g"]), _ptr(L["ln_ffn_b"]), float(L["alpha_attn"]), float(L["alpha_ffn"]),
                          int(L["w_ffn13"].shape[1] // 2) if ffn else 0, GATES[L.get("gates", "vo")])
    return arr


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return REST_BF16
    if t.dtype == torch.float32:
        return REST_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def workspace_size(dtype: int, taus, d: int, cu_seqlens, layers: Sequence[dict] = (), reqs=None, K: int = 3,
                   rope_base: float = 10000.0) -> int:
    h = _Host(taus, d, rope_base, cu_seqlens, reqs)
    arr = _enc_layers(layers)
    out = c_size_t(0)
    _check(_lib.rest_workspace_size(dtype, ctypes.byref(h.heads), ctypes.byref(h.batch), arr, len(layers),
                                    ctypes.byref(h.reqs) if h.reqs is not None else None, K, ctypes.byref(out)),
           "rest_workspace_size")
    return out.value


def _workspace(nbytes: int, device):
    import torch
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


_ERR_WORDS = {}


def _err_word(device, stream=None):
    """The device status word for calls on (device, stream): one per pair, kept
    for the process; every library call clears it on its stream before its
    first kernel, so concurrent calls on different streams never share one."""
    import torch
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device(dev.type, torch.cuda.current_device())
    key = (dev, _stream(stream))
    w = _ERR_WORDS.get(key)
    if w is None:
        w = _ERR_WORDS[key] = torch.zeros(1, dtype=torch.int32, device=dev)
    return w


def check_device_error(err) -> None:
    """Synchronize and raise if a kernel reported an error in the status word."""
    code = int(err.item())
    if code != 0:
        err.zero_()  # the word is kept for later calls: leave it clear even for one that enqueues nothing
        raise RestError(code, "device")


def rotation_table(ts, cu_seqlens, taus, head_dim: int, rope_base: float = 10000.0, stream=None, check=True):
    """Rotation index [T, H] int64 and cos/sin tables [T, H, head_dim/2] fp32 (ReST §3.2.2, eq. 5)."""
    import torch
    dev = ts.device
    H = len(taus)
    T = ts.shape[0]
    h = _Host(taus, H * head_dim, rope_base, cu_seqlens)
    idx = torch.empty((T, H), dtype=torch.int64, device=dev)
    cos = torch.empty((T, H, head_dim // 2), dtype=torch.float32, device=dev)
    sin = torch.empty_like(cos)
    nb = workspace_size(REST_F32, taus, H * head_dim, cu_seqlens, rope_base=rope_base)
    ws, err = _workspace(nb, dev), _err_word(dev, stream)
    _check(_lib.rest_rotation_table(ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(ts), _ptr(idx), _ptr(cos),
                                    _ptr(sin), _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "rest_rotation_table")
    if check:
        check_device_error(err)
    return idx, cos, sin


def encoder_attn(x, ts, cu_seqlens, taus, layers: Sequence[dict], l_switch: int, rope_base: float = 10000.0,
                 h_out=None, ws=None, stream=None, check=True):
    """Encoder T over packed histories: returns H [T, d] in x's dtype (ReST §3.2)."""
    import torch
    dev, d = x.device, x.shape[1]
    dt = _dtype_code(x)
    h = _Host(taus, d, rope_base, cu_seqlens)
    arr = _enc_layers(layers)
    if h_out is None:
        h_out = torch.empty_like(x)
    if ws is None:
        ws = _workspace(workspace_size(dt, taus, d, cu_seqlens, layers, rope_base=rope_base), dev)
    err = _err_word(dev, stream)
    _check(_lib.rest_encoder_attn(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(x), _ptr(ts), arr,
                                  len(layers), l_switch, _ptr(h_out), _ptr(ws), ws.numel(), _ptr(err),
                                  _stream(stream)), "rest_encoder_attn")
    if check:
        check_device_error(err)
    return h_out


def _dec(dec: dict) -> DecParams:
    return DecParams(int(dec["w_q"].shape[0]), _ptr(dec["w_q"]), _ptr(dec["w_go"]), _ptr(dec["w_o"]))


def cross_decode(hmem, cu_seqlens, taus, reqs, z, dec: dict, rope_base: float = 10000.0, y_out=None, ws=None,
                 stream=None, check=True):
    """Cross decoder C: y [N, K, d] fp32 for every candidate of every request (ReST §3.3).

    ``reqs`` = (req_user, req_cutoff, cu_cands) host integer arrays.
    """
    import torch
    dev, d = hmem.device, hmem.shape[1]
    dt = _dtype_code(hmem)
    h = _Host(taus, d, rope_base, cu_seqlens, reqs)
    dp = _dec(dec)
    if y_out is None:
        y_out = torch.empty(z.shape, dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(workspace_size(dt, taus, d, cu_seqlens, (), reqs, dp.K, rope_base), dev)
    err = _err_word(dev, stream)
    _check(_lib.rest_cross_decode(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(hmem), ctypes.byref(h.reqs),
                                  _ptr(z), ctypes.byref(dp), _ptr(y_out), _ptr(ws), ws.numel(), _ptr(err),
                                  _stream(stream)), "rest_cross_decode")
    if check:
        check_device_error(err)
    return y_out


def cross_decode_static_ws(hmem, cu_seqlens, taus, reqs, z, dec: dict, rope_base: float = 10000.0, y_out=None,
                           stream=None, check=True, err=None):
    """``cross_decode`` for callers that cannot allocate device memory.

    The decoder's scratch lives in the library's own fixed device array of
    STATIC_WS_BYTES bytes instead of a caller workspace; batches that need
    more raise RestError(REST_ERR_WORKSPACE). Calls share that array, so
    calls that overlap on the GPU race; order them on one stream. A device's
    first call loads the array (one with no candidates does only that).
    (This wrapper itself allocates y_out and the status word with torch when
    they are not given; a caller that cannot allocate passes its own.)
    """
    import torch
    dev, d = hmem.device, hmem.shape[1]
    dt = _dtype_code(hmem)
    h = _Host(taus, d, rope_base, cu_seqlens, reqs)
    dp = _dec(dec)
    if y_out is None:
        y_out = torch.empty(z.shape, dtype=torch.float32, device=dev)
    if err is None:
        err = _err_word(dev, stream)
    _check(_lib.rest_cross_decode_static_ws(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(hmem),
                                            ctypes.byref(h.reqs), _ptr(z), ctypes.byref(dp), _ptr(y_out), _ptr(err),
                                            _stream(stream)), "rest_cross_decode_static_ws")
    if check:
        check_device_error(err)
    return y_out


def rank_request(x, ts, cu_seqlens, taus, layers: Sequence[dict], l_switch: int, reqs, z, dec: dict,
                 rope_base: float = 10000.0, h_out=None, y_out=None, ws=None, stream=None, check=True):
    """Shared-prefix serving: H = T(x) once, then C for every candidate. Returns (H, y) (ReST §3.5)."""
    import torch
    dev, d = x.device, x.shape[1]
    dt = _dtype_code(x)
    h = _Host(taus, d, rope_base, cu_seqlens, reqs)
    arr = _enc_layers(layers)
    dp = _dec(dec)
    if h_out is None:
        h_out = torch.empty_like(x)
    if y_out is None:
        y_out = torch.empty(z.shape, dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(workspace_size(dt, taus, d, cu_seqlens, layers, reqs, dp.K, rope_base), dev)
    err = _err_word(dev, stream)
    _check(_lib.rest_rank_request(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(x), _ptr(ts), arr,
                                  len(layers), l_switch, ctypes.byref(h.reqs), _ptr(z), ctypes.byref(dp), _ptr(h_out),
                                  _ptr(y_out), _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "rest_rank_request")
    if check:
        check_device_error(err)
    return h_out, y_out


class KVCache:
    """An append-only encoder cache: per layer the rotated keys and gated values
    of every cached token, and the cached tokens' rows of H, in zero-filled
    device arrays of ``capacity[u]`` rows per user; plus the host bookkeeping
    the C ABI reads (cached length, first and last timestamp per user)."""

    def __init__(self, capacity, n_layers: int, d: int, dtype, device, keep_h: bool = True):
        import torch
        cap = _i32(capacity)
        self.n_users = len(cap)
        self.cu_cap = np.zeros(self.n_users + 1, dtype=np.int32)
        self.cu_cap[1:] = np.cumsum(cap)
        self.rows = int(self.cu_cap[-1])
        shape = (max(1, self.rows), d)
        self.k = [torch.zeros(shape, dtype=dtype, device=device) for _ in range(n_layers)]
        self.v = [torch.zeros(shape, dtype=dtype, device=device) for _ in range(n_layers)]
        self.h = torch.zeros(shape, dtype=dtype, device=device) if keep_h else None
        self.len = np.zeros(self.n_users, dtype=np.int32)
        self.t_first = np.zeros(self.n_users, dtype=np.int64)
        self.t_last = np.zeros(self.n_users, dtype=np.int64)

    def struct(self):
        """The rest_kv_cache view; the returned tuple keeps its host arrays alive."""
        kp = (c_void_p * max(1, len(self.k)))(*[t.data_ptr() for t in self.k])
        vp = (c_void_p * max(1, len(self.v)))(*[t.data_ptr() for t in self.v])
        st = KVCacheStruct(kp, vp, _ptr(self.h), self.rows, self.cu_cap.ctypes.data_as(POINTER(c_int32)),
                           self.len.ctypes.data_as(POINTER(c_int32)), self.t_first.ctypes.data_as(POINTER(c_int64)),
                           self.t_last.ctypes.data_as(POINTER(c_int64)))
        return st, (kp, vp)

    def advance(self, cu_new, ts_host) -> None:
        """Record an append of the tokens packed by cu_new with host timestamps ts_host."""
        cu = _i32(cu_new)
        ts = np.asarray(ts_host, dtype=np.int64)
        for u in range(self.n_users):
            s, e = int(cu[u]), int(cu[u + 1])
            if e == s:
                continue
            if self.len[u] == 0:
                self.t_first[u] = ts[s]
            self.t_last[u] = ts[e - 1]
            self.len[u] += e - s

    def batch(self):
        """(cu_seqlens, cutoff limit) for decoding against the cached H: the
        regions' bounds serve as rest_cross_decode's batch."""
        return self.cu_cap.copy(), self.len.copy()


def append_workspace_size(dtype: int, taus, d: int, cu_new, layers: Sequence[dict] = (),
                          rope_base: float = 10000.0) -> int:
    h = _Host(taus, d, rope_base, cu_new)
    arr = _enc_layers(layers)
    out = c_size_t(0)
    _check(_lib.rest_append_workspace_size(dtype, ctypes.byref(h.heads), ctypes.byref(h.batch), arr, len(layers),
                                           ctypes.byref(out)), "rest_append_workspace_size")
    return out.value


def encoder_append(x, ts, cu_new, taus, layers: Sequence[dict], l_switch: int, cache: KVCache,
                   rope_base: float = 10000.0, ts_host=None, advance: bool = True, h_out=None, ws=None,
                   stream=None, check=True):
    """Encoder T on tokens appended to the histories in ``cache``: returns the
    new rows of H [T_new, d] and writes the new keys, values (and H) into the
    cache. With ``advance`` the cache's bookkeeping then counts the new tokens
    (their host timestamps: ``ts_host``, else copied from ``ts``)."""
    import torch
    dev, d = x.device, x.shape[1]
    dt = _dtype_code(x)
    h = _Host(taus, d, rope_base, cu_new)
    arr = _enc_layers(layers)
    if h_out is None:
        h_out = torch.empty_like(x)
    if ws is None:
        ws = _workspace(append_workspace_size(dt, taus, d, cu_new, layers, rope_base), dev)
    cst, keep = cache.struct()
    err = _err_word(dev, stream)
    _check(_lib.rest_encoder_append(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(x), _ptr(ts), arr,
                                    len(layers), l_switch, ctypes.byref(cst), _ptr(h_out), _ptr(ws), ws.numel(),
                                    _ptr(err), _stream(stream)), "rest_encoder_append")
    del keep
    if check:
        check_device_error(err)
    if advance:
        cache.advance(cu_new, ts.cpu().numpy() if ts_host is None else ts_host)
    return h_out


def attn_workspace_size(dtype: int, n_heads: int, head_dim: int, cu_seqlens) -> int:
    h = _Host(np.zeros(n_heads, dtype=np.int64), n_heads * head_dim, 10000.0, cu_seqlens)
    out = c_size_t(0)
    _check(_lib.rest_attn_workspace_size(dtype, ctypes.byref(h.heads), ctypes.byref(h.batch), ctypes.byref(out)),
           "rest_attn_workspace_size")
    return out.value


def attn_forward(q, k, v, cu_seqlens, n_heads: int, o=None, o_lo=None, lse=None, ws=None, stream=None,
                 check=True):
    """Causal attention core for training (ULT, §3.5): returns (O [T, d] in
    q's dtype, O's bf16 low part (bf16 calls; None in fp32), lse [T, n_heads]
    fp32)."""
    import torch
    dev, (T, d) = q.device, q.shape
    dt = _dtype_code(q)
    h = _Host(np.zeros(n_heads, dtype=np.int64), d, 10000.0, cu_seqlens)
    if o is None:
        o = torch.empty_like(q)
    if o_lo is None and dt == REST_BF16:
        o_lo = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, n_heads), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(attn_workspace_size(dt, n_heads, d // n_heads, cu_seqlens), dev)
    err = _err_word(dev, stream)
    _check(_lib.rest_attn_forward(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(o), _ptr(o_lo), _ptr(lse), _ptr(ws), ws.numel(), _ptr(err),
                                  _stream(stream)), "rest_attn_forward")
    if check:
        check_device_error(err)
    return o, o_lo, lse


def attn_backward(q, k, v, o, o_lo, lse, d_o, cu_seqlens, n_heads: int, dq=None, dk=None, dv=None, ws=None,
                  stream=None, check=True):
    """Gradients (dq, dk, dv), fp32 [T, d], of the attention core from dO."""
    import torch
    dev, (T, d) = q.device, q.shape
    dt = _dtype_code(q)
    h = _Host(np.zeros(n_heads, dtype=np.int64), d, 10000.0, cu_seqlens)
    dq = torch.empty((T, d), dtype=torch.float32, device=dev) if dq is None else dq
    dk = torch.empty((T, d), dtype=torch.float32, device=dev) if dk is None else dk
    dv = torch.empty((T, d), dtype=torch.float32, device=dev) if dv is None else dv
    if ws is None:
        ws = _workspace(attn_workspace_size(dt, n_heads, d // n_heads, cu_seqlens), dev)
    err = _err_word(dev, stream)
    _check(_lib.rest_attn_backward(dt, ctypes.byref(h.heads), ctypes.byref(h.batch), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(o), _ptr(o_lo), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv),
                                   _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "rest_attn_backward")
    if check:
        check_device_error(err)
    return dq, dk, dv


def selftest_wait_timeout(device, n_ctas: int = 148, limit_cycles: int = 20_000_000, stream=None) -> int:
    """Runs the failure-detection self-test and returns the status word it left
    (REST_ERR_TIMEOUT, 5, when detection works)."""
    import torch
    err = torch.zeros(1, dtype=torch.int32, device=device)
    _check(_lib.rest_selftest_wait_timeout(n_ctas, limit_cycles, _ptr(err), _stream(stream)),
           "rest_selftest_wait_timeout")
    return int(err.item())


def launch_count(reset: bool = False) -> int:
    """Kernel launches the library enqueued on this thread (since the last reset)."""
    return int(_lib.rest_launch_count(1 if reset else 0))


def profile_begin() -> None:
    """Start bracketing every library launch of this thread with CUDA events."""
    _lib.rest_profile_begin()


def profile_end() -> List[dict]:
    """Stop profiling; per kernel name: launches, ms, algorithmic flops and bytes."""
    buf = (KernelStat * 64)()
    n = _lib.rest_profile_end(buf, 64)
    return [{"name": buf[i].name.decode(), "launches": buf[i].launches, "ms": buf[i].ms, "flops": buf[i].flops,
             "bytes": buf[i].bytes} for i in range(min(n, 64))]


def score_workspace_size(dtype: int, d: int, K: int, n_cands: int, d_ff: int) -> int:
    out = c_size_t(0)
    _check(_lib.rest_score_workspace_size(dtype, d, K, n_cands, d_ff, ctypes.byref(out)), "rest_score_workspace_size")
    return out.value


def score_head(z, y, sp: dict, f_out=None, score_out=None, ws=None, stream=None, check=True):
    """Decoder block and candidate score (ReST §3.3.2 eq. 8): returns (f [N, K, d]
    fp32, score [N] fp32) from the query tokens z and the decoder output y."""
    import torch
    dev = z.device
    N, K, d = z.shape
    dt = _dtype_code(z)
    d_ff = int(sp["w_ffn2"].shape[1])
    if f_out is None:
        f_out = torch.empty((N, K, d), dtype=torch.float32, device=dev)
    if score_out is None:
        score_out = torch.empty((N,), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(score_workspace_size(dt, d, K, N, d_ff), dev)
    params = ScoreParams(_ptr(sp["w_ffn13"]), _ptr(sp["w_ffn2"]), _ptr(sp["ln_g"]), _ptr(sp["ln_b"]),
                         _ptr(sp["w_s"]), float(sp["b_s"]), d_ff)
    err = _err_word(dev, stream)
    _check(_lib.rest_score_head(dt, d, K, N, _ptr(z), _ptr(y), ctypes.byref(params), _ptr(f_out), _ptr(score_out),
                                _ptr(ws), ws.numel(), _ptr(err), _stream(stream)), "rest_score_head")
    if check:
        check_device_error(err)
    return f_out, score_out


def to_device(inp: dict, device) -> dict:
    """Move one batch of host inputs (numpy) to device tensors of the batch's dtype."""
    import torch
    wdt = torch.bfloat16 if inp["dtype"] == "bf16" else torch.float32

    def dev(a, dtype=wdt):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)

    layers = []
    for L in inp["layers"]:
        layers.append({
            "w_qkvgg": dev(L["w_qkvgg"]), "w_o": dev(L["w_o"]), "w_ffn13": dev(L["w_ffn13"]),
            "w_ffn2": dev(L["w_ffn2"]), "alpha_attn": L["alpha_attn"], "alpha_ffn": L["alpha_ffn"],
            "gates": L.get("gates", "vo"),
            **{k: dev(L[k], torch.float32) for k in ("ln_attn_g", "ln_attn_b", "ln_ffn_g", "ln_ffn_b")},
        })
    return {
        "x": dev(inp["x"]), "ts": dev(inp["ts"], torch.int64), "z": dev(inp["z"]),
        "dec": {k: dev(v) for k, v in inp["dec"].items()}, "layers": layers,
        "score": ({"w_ffn13": dev(inp["score"]["w_ffn13"]), "w_ffn2": dev(inp["score"]["w_ffn2"]),
                   **{k: dev(inp["score"][k], torch.float32) for k in ("ln_g", "ln_b", "w_s")},
                   "b_s": float(inp["score"]["b_s"])} if "score" in inp else None),
        "cu_seqlens": np.asarray(inp["cu_seqlens"], dtype=np.int32), "taus": np.asarray(inp["taus"]),
        "l_switch": int(inp["l_switch"]), "rope_base": float(inp["rope_base"]),
        "reqs": (np.asarray(inp["req_user"], np.int32), np.asarray(inp["req_cutoff"], np.int32),
                 np.asarray(inp["cu_cands"], np.int32)),
        "dtype": inp["dtype"],
    }

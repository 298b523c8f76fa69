"""Seeded synthetic workloads for the ReST ranking forward.

This module only draws inputs: shapes, packed index arrays, timestamps,
features and weights. It holds none of the method's arithmetic (no buckets,
rotations, norms, attention). Both the fp64 oracle and the CUDA path read
what it produces.

The five workloads follow the shapes of the ReST paper's serving setting
("From Language to Behavior", ReST reading, §3.5 shared-prefix serving and
§5.3 scaling axes: sequence length up to 16k, width d in {128, 256, 512}).
The pages' industrial data is confidential and their public datasets are not
available, so every value is synthetic:

* features and candidate query tokens ~ N(0, 1);
* every weight matrix ~ N(0, 1/d);
* timestamps: t0 = 1.7e9 s, gaps = max(1, floor(exp(N(ln 600, 2^2)))) s;
* LayerNorm gamma = 1, beta = 0 unless ``ln_affine`` asks for random ones.

bf16 workloads round every value to bf16 (round-to-nearest-even) and keep the
rounded value in float32 storage, so both sides see identical numbers.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

T0_SECONDS = 1_700_000_000
ONE_YEAR_SECONDS = 31_536_000

# Granularities in seconds, the power of two nearest in log2 to each named
# unit: second, minute, hour, day, week, quarter, year.
GRANULARITY_SECONDS = {
    "second": 1,
    "minute": 1 << 6,
    "hour": 1 << 12,
    "day": 1 << 16,
    "week": 1 << 19,
    "quarter": 1 << 23,
    "year": 1 << 25,
}
SEVEN_LEVELS = [GRANULARITY_SECONDS[k] for k in
                ("second", "minute", "hour", "day", "week", "quarter", "year")]


def ffn_width(d: int) -> int:
    """LLaMA-style SwiGLU width: 8d/3 rounded up to a multiple of 64."""
    return 64 * ((8 * d + 191) // 192)


def head_taus(n_heads: int, n_rope: int, levels: List[int]) -> np.ndarray:
    """Per-head granularity: RoPE heads (0) first, then the time heads.

    Time head i of m takes levels[round(i * (len(levels)-1) / (m-1))], which
    keeps the finest and the coarsest level.
    """
    m = n_heads - n_rope
    taus = [0] * n_rope
    for i in range(m):
        pos = 0.0 if m == 1 else i * (len(levels) - 1) / (m - 1)
        taus.append(levels[int(math.floor(pos + 0.5))])
    return np.asarray(taus, dtype=np.int64)


@dataclasses.dataclass
class Workload:
    name: str
    dtype: str                      # "f32" or "bf16"
    lengths: List[int]              # L_u per user
    d: int
    n_heads: int
    head_dim: int
    taus: np.ndarray                # int64 [n_heads]
    n_layers: int
    alpha_attn: float
    alpha_ffn: float
    d_ff: int                       # 0 = attention-only layers
    l_switch: int
    req_user: List[int]
    req_cutoff: List[int]
    req_ncand: List[int]
    K: int = 3
    rope_base: float = 10000.0
    duplicate_frac: float = 0.0     # share of positions i>=1 copying token i-1
    span_seconds: Optional[int] = None  # rescale each history to this span
    gates: str = "vo"               # attention gates: "vo" (DGA), "o" or "qkvo" (ablation variants)

    @property
    def n_users(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def n_req(self) -> int:
        return len(self.req_user)

    @property
    def total_cands(self) -> int:
        return int(sum(self.req_ncand))

    @property
    def max_len(self) -> int:
        return int(max(self.lengths)) if self.lengths else 0


def _full_requests(lengths, ncand):
    n = len(lengths)
    return list(range(n)), list(lengths), [ncand] * n


def workload(idx: int) -> Workload:
    """The five named workloads (0 = tiny fp32 ... 4 = ragged shared-prefix)."""
    if idx == 0:
        lengths = [64]
        u, c, n = _full_requests(lengths, 8)
        return Workload("tiny-f32-L64-d64", "f32", lengths, 64, 4, 16,
                        head_taus(4, 2, [GRANULARITY_SECONDS[k] for k in ("minute", "hour", "day")]),
                        1, 0.01, 0.01, ffn_width(64), 0, u, c, n)
    if idx == 1:
        lengths = [1024] * 32
        u, c, n = _full_requests(lengths, 128)
        return Workload("bf16-32x1024-d256-4L-N128", "bf16", lengths, 256, 8, 32,
                        head_taus(8, 4, SEVEN_LEVELS), 4, 0.1, 0.1, ffn_width(256), 1, u, c, n)
    if idx == 2:
        lengths = [4096] * 8
        u, c, n = _full_requests(lengths, 256)
        return Workload("bf16-8x4096-d512-2L-N256-dup5", "bf16", lengths, 512, 8, 64,
                        head_taus(8, 4, SEVEN_LEVELS), 2, 0.01, 0.01, ffn_width(512), 0, u, c, n,
                        duplicate_frac=0.05)
    if idx == 3:
        lengths = [16384] * 2
        u, c, n = _full_requests(lengths, 512)
        return Workload("bf16-2x16384-d512-1L-N512-1y", "bf16", lengths, 512, 8, 64,
                        head_taus(8, 4, SEVEN_LEVELS), 1, 0.01, 0.01, ffn_width(512), 0, u, c, n,
                        span_seconds=ONE_YEAR_SECONDS)
    if idx == 4:
        return ragged_workload(seed=1004)
    raise ValueError(f"no workload {idx}")


def ragged_workload(seed: int, n_users: int = 64, d: int = 256, n_heads: int = 8,
                    min_len: int = 128, max_len: int = 16384, median_len: float = 2048.0,
                    min_cands: int = 64, max_cands: int = 1024, max_cutoffs: int = 4,
                    n_layers: int = 1) -> Workload:
    """Ragged padding-free batch with 1-4 request cutoffs per user.

    L_u = clip(round(exp(N(ln median_len, 1))), min_len, max_len); the last
    cutoff is L_u and the others are uniform integers in [min_len, L_u];
    candidates per request are uniform in [min_cands, max_cands].
    """
    rng = np.random.default_rng(seed)
    lengths, ru, rc, rn = [], [], [], []
    for u in range(n_users):
        L = int(np.clip(np.round(np.exp(rng.normal(math.log(median_len), 1.0))), min_len, max_len))
        lengths.append(L)
        R = int(rng.integers(1, max_cutoffs + 1))
        cuts = [L] + [int(rng.integers(min(min_len, L), L + 1)) for _ in range(R - 1)]
        for c in sorted(cuts):
            ru.append(u)
            rc.append(c)
            rn.append(int(rng.integers(min_cands, max_cands + 1)))
    hd = d // n_heads
    return Workload(f"bf16-ragged{n_users}-d{d}", "bf16", lengths, d, n_heads, hd,
                    head_taus(n_heads, n_heads // 2, SEVEN_LEVELS), n_layers, 0.01, 0.01,
                    ffn_width(d), n_layers // 4, ru, rc, rn)


def small_workload(dtype: str = "bf16", lengths=(300, 129, 64), d: int = 128, n_heads: int = 4,
                   n_rope: Optional[int] = None, n_layers: int = 2, l_switch: int = 1,
                   requests=None, ncand: int = 20, alpha: float = 0.1, ffn: bool = True,
                   levels=None, K: int = 3, duplicate_frac: float = 0.05,
                   name: str = "small", gates: str = "vo") -> Workload:
    """A small ragged workload for parity tests (several tiles and a ragged tail).

    ``requests`` is a list of (user, cutoff, n_candidates); by default every
    user has one request at its full length with ``ncand`` candidates.
    """
    lengths = list(lengths)
    if n_rope is None:
        n_rope = n_heads // 2
    if requests is None:
        requests = [(u, L, ncand) for u, L in enumerate(lengths)]
    return Workload(f"{name}-{dtype}-d{d}", dtype, lengths, d, n_heads, d // n_heads,
                    head_taus(n_heads, n_rope, levels or SEVEN_LEVELS), n_layers, alpha, alpha,
                    ffn_width(d) if ffn else 0, l_switch,
                    [r[0] for r in requests], [r[1] for r in requests], [r[2] for r in requests],
                    K=K, duplicate_frac=duplicate_frac, gates=gates)


# --------------------------------------------------------------------------
# value generation
# --------------------------------------------------------------------------

def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest-even on the float32 bits) and return float32."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32).reshape(f.shape)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def draw_timestamps(rng, L: int, span_seconds: Optional[int] = None) -> np.ndarray:
    gaps = np.maximum(1.0, np.floor(np.exp(rng.normal(math.log(600.0), 2.0, size=max(L - 1, 0)))))
    if span_seconds is not None and L > 1:
        gaps = np.maximum(1.0, np.round(gaps * (span_seconds / gaps.sum())))
    t = np.empty(L, dtype=np.int64)
    if L:
        t[0] = T0_SECONDS
        t[1:] = T0_SECONDS + np.cumsum(gaps.astype(np.int64))
    return t


def make_inputs(w: Workload, seed: int, ln_affine: bool = False) -> dict:
    """Draw every input array of a workload. Deterministic in (w, seed)."""
    rng = np.random.default_rng(seed)
    d, T = w.d, w.total_tokens
    cu = np.zeros(w.n_users + 1, dtype=np.int32)
    cu[1:] = np.cumsum(w.lengths)
    x = rng.standard_normal((T, d))
    ts = np.empty(T, dtype=np.int64)
    for u, L in enumerate(w.lengths):
        s = int(cu[u])
        ts[s:s + L] = draw_timestamps(rng, L, w.span_seconds)
        if w.duplicate_frac > 0 and L > 1:
            ndup = int(round(w.duplicate_frac * (L - 1)))
            pos = np.sort(rng.choice(np.arange(1, L), size=ndup, replace=False))
            for p in pos:               # copy the previous click: features and time
                x[s + p] = x[s + p - 1]
                ts[s + p] = ts[s + p - 1]
    sd = 1.0 / math.sqrt(d)
    layers = []
    for _ in range(w.n_layers):
        lay = {
            "w_qkvgg": _store(rng.standard_normal((d, {"vo": 5, "o": 4, "qkvo": 7}[w.gates] * d)) * sd, w.dtype),
            "gates": w.gates,
            "w_o": _store(rng.standard_normal((d, d)) * sd, w.dtype),
            "w_ffn13": _store(rng.standard_normal((d, 2 * w.d_ff)) * sd, w.dtype) if w.d_ff else None,
            "w_ffn2": _store(rng.standard_normal((w.d_ff, d)) * sd, w.dtype) if w.d_ff else None,
            "alpha_attn": w.alpha_attn,
            "alpha_ffn": w.alpha_ffn,
        }
        for name in ("ln_attn", "ln_ffn"):
            if ln_affine:
                lay[name + "_g"] = (1.0 + 0.2 * rng.standard_normal(d)).astype(np.float32)
                lay[name + "_b"] = (0.1 * rng.standard_normal(d)).astype(np.float32)
            else:
                lay[name + "_g"] = np.ones(d, dtype=np.float32)
                lay[name + "_b"] = np.zeros(d, dtype=np.float32)
        layers.append(lay)
    dec = {
        "w_q": _store(rng.standard_normal((w.K, d, d)) * sd, w.dtype),
        "w_go": _store(rng.standard_normal((w.K, d, d)) * sd, w.dtype),
        "w_o": _store(rng.standard_normal((d, d)) * sd, w.dtype),
    }
    cu_c = np.zeros(w.n_req + 1, dtype=np.int32)
    cu_c[1:] = np.cumsum(w.req_ncand)
    z = _store(rng.standard_normal((w.total_cands, w.K, d)), w.dtype)
    # decoder block FFN and score readout: drawn after every array above, which stay as they were
    dff = ffn_width(d)
    score = {
        "w_ffn13": _store(rng.standard_normal((w.K, d, 2 * dff)) * sd, w.dtype),
        "w_ffn2": _store(rng.standard_normal((w.K, dff, d)) * sd, w.dtype),
        "ln_g": np.ones((w.K, d), dtype=np.float32),
        "ln_b": np.zeros((w.K, d), dtype=np.float32),
        "w_s": (rng.standard_normal(d) * sd).astype(np.float32),
        "b_s": 0.25,
    }
    if ln_affine:
        score["ln_g"] = (1.0 + 0.2 * rng.standard_normal((w.K, d))).astype(np.float32)
        score["ln_b"] = (0.1 * rng.standard_normal((w.K, d))).astype(np.float32)
    return {
        "x": _store(x, w.dtype),
        "ts": ts,
        "cu_seqlens": cu,
        "taus": w.taus.copy(),
        "layers": layers,
        "l_switch": w.l_switch,
        "dec": dec,
        "score": score,
        "z": z,
        "req_user": np.asarray(w.req_user, dtype=np.int32),
        "req_cutoff": np.asarray(w.req_cutoff, dtype=np.int32),
        "cu_cands": cu_c,
        "rope_base": w.rope_base,
        "dtype": w.dtype,
    }


def make_memory(w: Workload, seed: int) -> np.ndarray:
    """A synthetic encoder output H ~ N(0,1) [T, d], for testing the decoder alone."""
    rng = np.random.default_rng(seed + 7919)
    return _store(rng.standard_normal((w.total_tokens, w.d)), w.dtype)


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


def tile_workload(w: Workload, n: int) -> Workload:
    """The workload's users and requests repeated n times (one global batch)."""
    if n == 1:
        return w
    U = w.n_users
    return dataclasses.replace(
        w, name=f"{w.name}x{n}", lengths=list(w.lengths) * n,
        req_user=[u + i * U for i in range(n) for u in w.req_user],
        req_cutoff=list(w.req_cutoff) * n, req_ncand=list(w.req_ncand) * n)

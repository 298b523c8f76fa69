"""fp64 CPU oracle of the ReST encode-once / decode-many ranking forward.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain statement of what
the CUDA path must compute. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the library never does, and the
library shares no code with it.

Every function follows the ReST paper as read on the page "From Language to
Behavior" (paper-archivist close reading of arXiv 2609.01240); the section
and equation numbers below are that page's. Where the page leaves a detail
open the reading taken is stated in the docstring (the same readings are
fixed in the repository's written specification).

Everything is float64; inputs (bf16 or fp32 values) are upcast exactly.
Matrix products use numpy's matmul as a library primitive; there is no
fusion or reordering beyond the definitions.

Pins (tests/test_oracle_pins.py): every public function is checked against
something other than itself -- a literal loop implementation with explicit
rotation matrices (oracle/brute.py) on tiny inputs, torch's fp64
scaled_dot_product_attention and layer_norm, closed forms (first causal row,
cutoff 1, alpha 0), and the invariants the page states (relative position and
relative time, eq. 14; causality; candidate permutation; shared-prefix
reuse, §3.5).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

LN_EPS = 1e-5


class UnsortedTimestamps(ValueError):
    pass


# --------------------------------------------------------------------------
# §3.2.2: rotation index (RoPE position or RoTE time bucket) and angles
# --------------------------------------------------------------------------

def rotation_index(ts: np.ndarray, cu_seqlens: np.ndarray, taus: np.ndarray,
                   time_origin: Optional[Sequence[int]] = None,
                   pos_offset: int = 0) -> np.ndarray:
    """Per (token, head) rotation index, int64 [T, n_heads].

    §3.2.2: RoPE heads (tau_h = 0) use the ordinal position; RoTE heads use
    the bucket b_i = floor((t_i - t_1) / tau_h), t_1 the first timestamp of
    the user's sequence. Reading: positions are 0-based within each user.

    ``time_origin`` (per user) replaces t_1 and ``pos_offset`` shifts every
    position; both exist only so the tests can check the invariances of
    eq. 14 and are not part of the method.
    """
    ts = np.asarray(ts, dtype=np.int64)
    T = ts.shape[0]
    H = len(taus)
    idx = np.zeros((T, H), dtype=np.int64)
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        if e <= s:
            continue
        t = ts[s:e]
        if np.any(t[1:] < t[:-1]):
            raise UnsortedTimestamps(f"user {u}: timestamps decrease")
        origin = t[0] if time_origin is None else np.int64(time_origin[u])
        rel = t - origin                                    # exact int64
        for h, tau in enumerate(taus):
            if tau == 0:
                idx[s:e, h] = np.arange(e - s, dtype=np.int64) + pos_offset
            else:
                idx[s:e, h] = np.floor_divide(rel, np.int64(tau))
    return idx


def frequencies(head_dim: int, rope_base: float) -> np.ndarray:
    """theta_j = base^(-2j/d_h), j = 0..d_h/2-1 (RoPE's schedule; §3.2.2 says
    RoPE and RoTE share one rotation mechanism, so RoTE heads use it too)."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(rope_base), -2.0 * j / head_dim)


def rotation_angles(idx: np.ndarray, head_dim: int, rope_base: float,
                    angle_scale: float = 1.0) -> np.ndarray:
    """phi[i, h, j] = idx[i, h] * theta_j in fp64 (eq. 5's R_Theta(idx)).

    ``angle_scale`` = 0 turns every rotation into the identity (test knob).
    """
    return idx.astype(np.float64)[:, :, None] * frequencies(head_dim, rope_base)[None, None, :] * angle_scale


def rotate(v: np.ndarray, phi: np.ndarray) -> np.ndarray:
    """Apply the block-diagonal R_Theta per head to rows of v [T, H*d_h].

    Reading: 2x2 blocks on the column pairs (2j, 2j+1) of each head,
    (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
    """
    T, H, half = phi.shape
    x = v.reshape(T, H, half, 2)
    a, b = x[..., 0], x[..., 1]
    c, s = np.cos(phi), np.sin(phi)
    out = np.empty_like(x)
    out[..., 0] = a * c - b * s
    out[..., 1] = a * s + b * c
    return out.reshape(T, H * half * 2)


# --------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------

def sigmoid(z: np.ndarray) -> np.ndarray:
    """Bounded sigmoid gate (§3.2.1: sigmoid instead of HSTU's SiLU gate)."""
    return 1.0 / (1.0 + np.exp(-z))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z), the SwiGLU activation of the LLaMA block (§3.2)."""
    return z * sigmoid(z)


def layer_norm(v: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """LN over the last axis with the biased variance (eq. 6's LN)."""
    mu = v.mean(axis=-1, keepdims=True)
    var = ((v - mu) ** 2).mean(axis=-1, keepdims=True)
    return (v - mu) / np.sqrt(var + eps) * g.astype(np.float64) + b.astype(np.float64)


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Row softmax with the row maximum subtracted; -inf entries give 0."""
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    return E / E.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# §3.2.1: Dual-Gated Attention
# --------------------------------------------------------------------------

def causal_attention_probs(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """P = softmax(q k^T * scale + M_causal) for one sequence and one head (eq. 3)."""
    L = q.shape[0]
    S = (q @ k.T) * scale
    S[np.triu_indices(L, 1)] = -np.inf
    return softmax_rows(S)


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# Column blocks of the attention projection weight for each choice of gates:
# the DGA layer (value and output gates, eqs. 3-4) and the two variants of the
# page's gated-attention ablation (output gate alone; Q, K, V and output).
GATE_BLOCKS = {"vo": ("q", "k", "v", "gv", "go"),
               "o": ("q", "k", "v", "go"),
               "qkvo": ("q", "k", "v", "gv", "go", "gq", "gk")}


def dga_sublayer(y: np.ndarray, phi: np.ndarray, cu_seqlens: np.ndarray, layer: dict,
                 n_heads: int, gates: bool = True, row_chunk: int = 2048,
                 kv_out: Optional[list] = None) -> np.ndarray:
    """Eqs. 3-5: (Attention(R q, R k, sigmoid(y W_gv) * y W_V) * sigmoid(y W_go)) W_o.

    Readings: no biases; the gates are full d x d projections applied
    elementwise; head h owns columns h*d_h..(h+1)*d_h-1; the score scale is
    1/sqrt(d_h) (eq. 7's multi-head form; eq. 3 is written single-head).
    ``layer["gates"]`` picks the gates ("vo" when absent, see GATE_BLOCKS);
    with Q and K gates, the gated projections are what eq. 5 rotates, so the
    scores keep eq. 14's dependence on the index difference alone.
    ``gates=False`` replaces every sigmoid by 1 (test knob). When ``kv_out``
    is a list, the rotated keys R k and the gated values V' of every row (the
    operands later queries attend to) are appended to it as a pair.
    """
    T, d = y.shape
    hd = d // n_heads
    W = _f64(layer["w_qkvgg"])
    names = GATE_BLOCKS[layer.get("gates", "vo")]
    P = y @ W
    blk = {n: P[:, i * d:(i + 1) * d] for i, n in enumerate(names)}
    Q, Kx, V = blk["q"], blk["k"], blk["v"]
    if gates and "gq" in blk:
        Q = Q * sigmoid(blk["gq"])
        Kx = Kx * sigmoid(blk["gk"])
    Vg = V * sigmoid(blk["gv"]) if gates and "gv" in blk else V
    Go = blk["go"]
    Qr, Kr = rotate(Q, phi), rotate(Kx, phi)
    if kv_out is not None:
        kv_out.append((Kr, Vg))
    O = np.zeros((T, d))
    scale = 1.0 / math.sqrt(hd)
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        L = e - s
        for h in range(n_heads):
            cols = slice(h * hd, (h + 1) * hd)
            q, k, v = Qr[s:e, cols], Kr[s:e, cols], Vg[s:e, cols]
            for r0 in range(0, L, row_chunk):
                r1 = min(L, r0 + row_chunk)
                # rows r0..r1-1 see keys 0..r1-1 at most (j <= i)
                S = (q[r0:r1] @ k[:r1].T) * scale
                ii = np.arange(r0, r1)[:, None]
                jj = np.arange(r1)[None, :]
                S[jj > ii] = -np.inf
                O[s + r0:s + r1, cols] = softmax_rows(S) @ v[:r1]
    G = sigmoid(Go) if gates else 1.0
    return (O * G) @ _f64(layer["w_o"])


def ffn_sublayer(y: np.ndarray, layer: dict) -> np.ndarray:
    """SwiGLU FFN of the LLaMA-style block (§3.2): (SiLU(y W_1) * y W_3) W_2."""
    W13 = _f64(layer["w_ffn13"])
    dff = W13.shape[1] // 2
    A = y @ W13
    return (silu(A[:, :dff]) * A[:, dff:]) @ _f64(layer["w_ffn2"])


def srn(x: np.ndarray, sub, alpha: float, post: bool, g: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Eq. 6 (Stabilized Residual Normalization) around one sublayer.

    post:  LN(x + alpha * Sub(x));   pre:  x + alpha * Sub(LN(x)).
    """
    if post:
        return layer_norm(x + alpha * sub(x), g, b)
    return x + alpha * sub(layer_norm(x, g, b))


# --------------------------------------------------------------------------
# encoder T, cross decoder C, rank_request
# --------------------------------------------------------------------------

def encoder(inp: dict, gates: bool = True, angle_scale: float = 1.0,
            time_origin=None, pos_offset: int = 0, n_layers: Optional[int] = None,
            kv_out: Optional[list] = None) -> np.ndarray:
    """Encoder T (§3.2, Fig. 1 left): n_layers blocks of [DGA, SwiGLU FFN],
    each sublayer wrapped by eq. 6 with post-LN for l <= l_switch (1-based).

    Readings: one layer = attention sublayer then FFN sublayer (the LLaMA
    block the page starts from); no final norm; separate alpha per sublayer.
    ``kv_out`` (a list) receives each layer's (R k, V') pair, layer by layer.
    """
    x = _f64(inp["x"]).copy()
    taus = np.asarray(inp["taus"], dtype=np.int64)
    H = len(taus)
    d = x.shape[1]
    hd = d // H
    idx = rotation_index(inp["ts"], inp["cu_seqlens"], taus, time_origin, pos_offset)
    phi = rotation_angles(idx, hd, inp["rope_base"], angle_scale)
    layers = inp["layers"] if n_layers is None else inp["layers"][:n_layers]
    for l, lay in enumerate(layers, start=1):
        post = l <= inp["l_switch"]
        x = srn(x, lambda y: dga_sublayer(y, phi, inp["cu_seqlens"], lay, H, gates, kv_out=kv_out),
                lay["alpha_attn"], post, lay["ln_attn_g"], lay["ln_attn_b"])
        if lay.get("w_ffn13") is not None:
            x = srn(x, lambda y: ffn_sublayer(y, lay),
                    lay["alpha_ffn"], post, lay["ln_ffn_g"], lay["ln_ffn_b"])
    return x


# --------------------------------------------------------------------------
# §3.5 ULT: the attention core's forward statistics and its backward
# --------------------------------------------------------------------------

def attention_core(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: np.ndarray, n_heads: int):
    """The causal attention core of a DGA sublayer over packed histories:
    per user and head, O = softmax(q k^T / sqrt(d_h) + M_causal) V, with q, k
    the rotated queries and keys and V the gated values V' (eq. 3), and
    lse[i, h] = log sum_{j <= i} exp(q_i . k_j / sqrt(d_h)), the statistic a
    backward pass reuses. Returns (O [T, d], lse [T, n_heads]).

    ULT (§3.5) encodes the union history of a user's samples once under a
    prefix-valid causal mask; since a sample ending at row c reads rows < c
    and every row i sees rows j <= i only, that mask is this causal mask on
    the union sequence (reading).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    hd = d // n_heads
    scale = 1.0 / math.sqrt(hd)
    O = np.zeros((T, d))
    lse = np.zeros((T, n_heads))
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        if e == s:
            continue
        for h in range(n_heads):
            c = slice(h * hd, (h + 1) * hd)
            S = (q[s:e, c] @ k[s:e, c].T) * scale
            S[np.triu_indices(e - s, 1)] = -np.inf
            m = S.max(axis=1, keepdims=True)
            lse[s:e, h] = (m + np.log(np.exp(S - m).sum(axis=1, keepdims=True)))[:, 0]
            O[s:e, c] = softmax_rows(S) @ v[s:e, c]
    return O, lse


def attention_core_backward(q, k, v, cu_seqlens, n_heads, d_o):
    """Gradients of a scalar loss through attention_core, given dO = dL/dO:
    with S = q k^T / sqrt(d_h) (causal), P = softmax(S) and O = P V,

        dV = P^T dO,   dP = dO V^T,   dS = P * (dP - rowsum(dP * P)),
        dq = dS k / sqrt(d_h),   dk = dS^T q / sqrt(d_h),

    per user and head (the chain rule through the row softmax; rowsum(dP * P)
    equals rowsum(dO * O)). Returns (dq, dk, dv), each [T, d]."""
    q, k, v, d_o = _f64(q), _f64(k), _f64(v), _f64(d_o)
    T, d = q.shape
    hd = d // n_heads
    scale = 1.0 / math.sqrt(hd)
    dq, dk, dv = np.zeros((T, d)), np.zeros((T, d)), np.zeros((T, d))
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        if e == s:
            continue
        for h in range(n_heads):
            c = slice(h * hd, (h + 1) * hd)
            S = (q[s:e, c] @ k[s:e, c].T) * scale
            S[np.triu_indices(e - s, 1)] = -np.inf
            P = softmax_rows(S)
            dv[s:e, c] = P.T @ d_o[s:e, c]
            dP = d_o[s:e, c] @ v[s:e, c].T
            dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
            dq[s:e, c] = dS @ k[s:e, c] * scale
            dk[s:e, c] = dS.T @ q[s:e, c] * scale
    return dq, dk, dv


def attention_core_dq_rows(q, k, v, cu_seqlens, n_heads, d_o, rows: Sequence[int]):
    """Rows of attention_core_backward's dq, each computed on its own: row i
    needs only its own scores against keys j <= i (same definition), so rows
    of a 16k-token history can be checked without the L x L matrices."""
    q, k, v, d_o = _f64(q), _f64(k), _f64(v), _f64(d_o)
    d = q.shape[1]
    hd = d // n_heads
    scale = 1.0 / math.sqrt(hd)
    cu = np.asarray(cu_seqlens)
    out = np.zeros((len(rows), d))
    for n, i in enumerate(rows):
        s = int(cu[np.searchsorted(cu, i, side="right") - 1])
        for h in range(n_heads):
            c = slice(h * hd, (h + 1) * hd)
            sc = (k[s:i + 1, c] @ q[i, c]) * scale
            p = np.exp(sc - sc.max())
            p /= p.sum()
            dp = v[s:i + 1, c] @ d_o[i, c]
            ds = p * (dp - (p * dp).sum())
            out[n, c] = (ds @ k[s:i + 1, c]) * scale
    return out


def encoder_append(hist: dict, cached: Sequence[int]):
    """Append-only encoding of the tokens that follow a cached prefix.

    Why a prefix can be cached: the encoder's attention is causal (eqs. 3-5:
    row i reads rows j <= i only), every other step acts on one row at a time,
    and RoTE counts time from the history's first timestamp t_1 (§3.2.2),
    which appending does not move. So H and every layer's rotated keys R k and
    gated values V' on a history's first c rows stay the same when tokens are
    appended after them (the same argument §3.5 makes for the prefix a request
    reads). An append therefore computes only the new rows, attending to the
    cached keys and values of the old ones.

    Definition: ``hist`` is each user's whole history (the cached tokens, then
    the new ones) in the encoder's input form; user u has cached[u] tokens in
    the cache. The result holds rows cached[u] .. L_u - 1 of every user, packed
    in user order:
        H_new  [T_new, d]      those rows of encoder(hist)
        kv     [(K_l, V_l)]    those rows of layer l's R k and V'
        cu_new [n_users + 1]   prefix sums of L_u - cached[u]
    """
    cu = np.asarray(hist["cu_seqlens"], dtype=np.int64)
    n_users = len(cu) - 1
    if len(cached) != n_users:
        raise ValueError("one cached length per user")
    for u in range(n_users):
        if not 0 <= int(cached[u]) <= cu[u + 1] - cu[u]:
            raise ValueError(f"user {u}: cached length outside 0..L_u")
    kv = []
    H = encoder(hist, kv_out=kv)
    rows = [np.arange(cu[u] + int(cached[u]), cu[u + 1], dtype=np.int64) for u in range(n_users)]
    rows = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    cu_new = np.zeros(n_users + 1, dtype=np.int64)
    cu_new[1:] = np.cumsum([cu[u + 1] - cu[u] - int(cached[u]) for u in range(n_users)])
    return H[rows], [(k[rows], v[rows]) for k, v in kv], cu_new


def encoder_rows(inp: dict, rows: Sequence[int]) -> np.ndarray:
    """Selected rows of H for a one-layer encoder, each computed on its own.

    Same definition as ``encoder`` (§3.2, eqs. 3-6); a query row of a single
    layer only needs its own row and the keys/values of the rows before it,
    so a handful of rows of a 16k-token history can be checked without the
    full L x L computation.
    """
    assert len(inp["layers"]) == 1, "row sampling is exact only for one layer"
    lay = inp["layers"][0]
    post = 1 <= inp["l_switch"]
    x = _f64(inp["x"])
    taus = np.asarray(inp["taus"], dtype=np.int64)
    H = len(taus)
    d = x.shape[1]
    hd = d // H
    cu = np.asarray(inp["cu_seqlens"])
    idx = rotation_index(inp["ts"], cu, taus)
    phi = rotation_angles(idx, hd, inp["rope_base"])
    W = _f64(lay["w_qkvgg"])
    scale = 1.0 / math.sqrt(hd)
    out = np.zeros((len(rows), d))
    cache = {}
    for n, i in enumerate(rows):
        u = int(np.searchsorted(cu, i, side="right") - 1)
        s = int(cu[u])
        if u not in cache:   # projections of the user's rows 0..L-1
            e = int(cu[u + 1])
            y = x[s:e] if post else layer_norm(x[s:e], lay["ln_attn_g"], lay["ln_attn_b"])
            P5 = y @ W
            Q, Kx, V, Gv, Go = (P5[:, j * d:(j + 1) * d] for j in range(5))
            cache = {u: (rotate(Q, phi[s:e]), rotate(Kx, phi[s:e]), V * sigmoid(Gv), sigmoid(Go))}
        Qr, Kr, Vg, G = cache[u]
        p = i - s
        o = np.zeros(d)
        for h in range(H):
            c = slice(h * hd, (h + 1) * hd)
            sc = (Kr[:p + 1, c] @ Qr[p, c]) * scale
            w = np.exp(sc - sc.max())
            o[c] = (w / w.sum()) @ Vg[:p + 1, c]
        a = (o * G[p]) @ _f64(lay["w_o"])
        xi = x[i]
        x1 = layer_norm(xi + lay["alpha_attn"] * a, lay["ln_attn_g"], lay["ln_attn_b"]) if post \
            else xi + lay["alpha_attn"] * a
        if lay.get("w_ffn13") is not None:
            y2 = x1 if post else layer_norm(x1, lay["ln_ffn_g"], lay["ln_ffn_b"])
            f = ffn_sublayer(y2[None, :], lay)[0]
            x1 = layer_norm(x1 + lay["alpha_ffn"] * f, lay["ln_ffn_g"], lay["ln_ffn_b"]) if post \
                else x1 + lay["alpha_ffn"] * f
        out[n] = x1
    return out


def cross_decode(Hmem: np.ndarray, cu_seqlens: np.ndarray, req_user, req_cutoff, cu_cands,
                 z: np.ndarray, dec: dict, n_heads: int, gates: bool = True,
                 row_chunk: int = 1024) -> np.ndarray:
    """Cross decoder C (§3.3, eqs. 7-8) -> y [N_total, K, d].

    Projection-free keys and values: the first c_r rows of the user's H are
    used directly as K and V. Token-specific W_Q^(k), W_go^(k) (eq. 8); a
    shared W_o. Readings: one decoder layer exactly as eq. 7 (no residual,
    no rotation); scale 1/sqrt(d_h).
    """
    Hm = _f64(Hmem)
    z = _f64(z)
    N, K, d = z.shape
    hd = d // n_heads
    Wq, Wg, Wo = _f64(dec["w_q"]), _f64(dec["w_go"]), _f64(dec["w_o"])
    q = np.einsum("nkd,kde->nke", z, Wq)
    g = sigmoid(np.einsum("nkd,kde->nke", z, Wg)) if gates else np.ones_like(q)
    o = np.zeros_like(q)
    scale = 1.0 / math.sqrt(hd)
    for r in range(len(req_user)):
        u, c = int(req_user[r]), int(req_cutoff[r])
        n0, n1 = int(cu_cands[r]), int(cu_cands[r + 1])
        if n1 <= n0:
            continue
        s = int(cu_seqlens[u])
        mem = Hm[s:s + c]
        qr = q[n0:n1].reshape(-1, d)
        orows = np.zeros_like(qr)
        for h in range(n_heads):
            cols = slice(h * hd, (h + 1) * hd)
            for r0 in range(0, qr.shape[0], row_chunk):
                r1 = min(qr.shape[0], r0 + row_chunk)
                S = (qr[r0:r1, cols] @ mem[:, cols].T) * scale
                orows[r0:r1, cols] = softmax_rows(S) @ mem[:, cols]
        o[n0:n1] = orows.reshape(n1 - n0, K, d)
    return (o * g) @ Wo


def score_head(z: np.ndarray, y: np.ndarray, sp: dict):
    """Decoder block and candidate score (§3.3.2 eq. 8, Fig. 1 right) -> (f, score).

    Readings: the query token plus eq. 7's output, a = z + y; then a pre-LN
    FFN sublayer whose LN and SwiGLU weights are specific to the token type
    (eq. 8), f = a + SwiGLU_k(LN_k(a)); the score is a linear logit on token 0
    ([CLS]): f[:, 0] . w_s + b_s.
    """
    z = _f64(z)
    a = z + _f64(y)
    N, K, d = a.shape
    f = np.empty_like(a)
    for k in range(K):
        layer = {"w_ffn13": sp["w_ffn13"][k], "w_ffn2": sp["w_ffn2"][k]}
        u = layer_norm(a[:, k], _f64(sp["ln_g"][k]), _f64(sp["ln_b"][k]))
        f[:, k] = a[:, k] + ffn_sublayer(u, layer)
    score = f[:, 0] @ _f64(sp["w_s"]) + float(sp["b_s"])
    return f, score


def rank_request(inp: dict, **kw):
    """Shared-prefix serving (§3.5): H = T(S_u) once, then C for every
    candidate of every request against it. Returns (H, y)."""
    Hm = encoder(inp, **kw)
    y = cross_decode(Hm, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"],
                     inp["z"], inp["dec"], len(inp["taus"]))
    return Hm, y

"""Literal, loop-by-loop restatement of the ReST forward for tiny inputs.

TEST INFRASTRUCTURE ONLY (used to pin oracle/rest_oracle.py; never used by
the library). It follows the equations of the page "From Language to
Behavior" (ReST reading) term by term, with Python integers for the buckets,
an explicit d_h x d_h block-diagonal matrix R_Theta for every rotation
(eq. 5, eq. 14), an explicit masked score matrix per head (eq. 3), and
scalar loops for softmax, LayerNorm (eq. 6) and the gates. It is written
independently of the vectorized oracle so that a dropped term, a wrong sign
or a transposed operand in either shows up as a disagreement.
"""
from __future__ import annotations

import math

import numpy as np


def bucket(t: int, t_first: int, tau: int) -> int:
    """b = floor((t - t_1) / tau) with Python's exact integer floor division."""
    return (int(t) - int(t_first)) // int(tau)


def index_table(ts, cu_seqlens, taus):
    out = []
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        for i in range(s, e):
            row = []
            for tau in taus:
                row.append(i - s if int(tau) == 0 else bucket(ts[i], ts[s], tau))
            out.append(row)
    return out


def R_matrix(idx: int, hd: int, base: float) -> np.ndarray:
    """Explicit block-diagonal rotation R_Theta(idx) (eq. 5)."""
    R = np.zeros((hd, hd))
    for j in range(hd // 2):
        a = idx * base ** (-2.0 * j / hd)
        c, s = math.cos(a), math.sin(a)
        R[2 * j, 2 * j], R[2 * j, 2 * j + 1] = c, -s
        R[2 * j + 1, 2 * j], R[2 * j + 1, 2 * j + 1] = s, c
    return R


def sig(z: float) -> float:
    return 1.0 / (1.0 + math.exp(-z))


def ln_row(v, g, b, eps=1e-5):
    n = len(v)
    mu = sum(v) / n
    var = sum((a - mu) * (a - mu) for a in v) / n
    inv = 1.0 / math.sqrt(var + eps)
    return [(v[i] - mu) * inv * float(g[i]) + float(b[i]) for i in range(n)]


def matvec(row, W):
    """row (length n) times W (n x m) with an explicit loop over n."""
    W = np.asarray(W, dtype=np.float64)
    acc = np.zeros(W.shape[1])
    for i, a in enumerate(row):
        acc += a * W[i]
    return acc


def softmax_list(scores):
    m = max(scores)
    e = [math.exp(s - m) for s in scores]
    tot = sum(e)
    return [v / tot for v in e]


def weight_blocks(lay, d):
    """The attention projection's d-wide column blocks by name: W_Q, W_K, W_V,
    then the gates the layer has (value + output by default; output only;
    or value, output, Q and K), in that order."""
    order = {"vo": "q k v gv go", "o": "q k v go", "qkvo": "q k v gv go gq gk"}[lay.get("gates", "vo")].split()
    W = np.asarray(lay["w_qkvgg"], dtype=np.float64)
    return {name: W[:, i * d:(i + 1) * d] for i, name in enumerate(order)}


def gate_mul(vec, gate_pre):
    """vec * sigmoid(gate_pre), element by element."""
    return np.array([vec[c] * sig(gate_pre[c]) for c in range(len(vec))])


def dga(yrows, idx, cu_seqlens, lay, H, base):
    d = len(yrows[0])
    hd = d // H
    Wb = weight_blocks(lay, d)
    out = []
    for u in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[u]), int(cu_seqlens[u + 1])
        q = [matvec(yrows[i], Wb["q"]) for i in range(s, e)]
        k = [matvec(yrows[i], Wb["k"]) for i in range(s, e)]
        v = [matvec(yrows[i], Wb["v"]) for i in range(s, e)]
        go = [matvec(yrows[i], Wb["go"]) for i in range(s, e)]
        if "gq" in Wb:  # Q and K gated before they are rotated
            q = [gate_mul(q[i], matvec(yrows[s + i], Wb["gq"])) for i in range(e - s)]
            k = [gate_mul(k[i], matvec(yrows[s + i], Wb["gk"])) for i in range(e - s)]
        if "gv" in Wb:
            vg = [gate_mul(v[i], matvec(yrows[s + i], Wb["gv"])) for i in range(e - s)]
        else:
            vg = [np.array(v[i]) for i in range(e - s)]
        for n in range(e - s):
            o = np.zeros(d)
            for h in range(H):
                sl = slice(h * hd, (h + 1) * hd)
                qn = R_matrix(idx[s + n][h], hd, base) @ q[n][sl]
                sc = []
                for m in range(n + 1):                      # causal: m <= n
                    km = R_matrix(idx[s + m][h], hd, base) @ k[m][sl]
                    sc.append(float(qn @ km) / math.sqrt(hd))
                p = softmax_list(sc)
                for m in range(n + 1):
                    o[sl] += p[m] * vg[m][sl]
            gated = [o[c] * sig(go[n][c]) for c in range(d)]
            out.append(matvec(gated, lay["w_o"]))
    return out


def ffn(yrows, lay):
    W13 = np.asarray(lay["w_ffn13"], dtype=np.float64)
    dff = W13.shape[1] // 2
    out = []
    for y in yrows:
        a = matvec(y, W13)
        hmid = [a[j] * sig(a[j]) * a[dff + j] for j in range(dff)]
        out.append(matvec(hmid, lay["w_ffn2"]))
    return out


def encoder(inp, gates_on: bool = True):
    assert gates_on
    x = [list(map(float, r)) for r in np.asarray(inp["x"], dtype=np.float64)]
    taus = [int(t) for t in inp["taus"]]
    H = len(taus)
    idx = index_table(inp["ts"], inp["cu_seqlens"], taus)
    base = float(inp["rope_base"])
    for l, lay in enumerate(inp["layers"], start=1):
        post = l <= inp["l_switch"]
        subs = [("attn", lambda ys: dga(ys, idx, inp["cu_seqlens"], lay, H, base))]
        if lay.get("w_ffn13") is not None:
            subs.append(("ffn", lambda ys: ffn(ys, lay)))
        for name, fn in subs:
            g, b, a = lay[f"ln_{name}_g"], lay[f"ln_{name}_b"], float(lay[f"alpha_{name}"])
            if post:
                upd = fn(x)
                x = [ln_row([x[i][c] + a * upd[i][c] for c in range(len(x[i]))], g, b) for i in range(len(x))]
            else:
                ys = [ln_row(r, g, b) for r in x]
                upd = fn(ys)
                x = [[x[i][c] + a * upd[i][c] for c in range(len(x[i]))] for i in range(len(x))]
    return np.array(x)


def encoder_stream(inp, cached):
    """The encoder as a server with a per-layer cache runs it: each user's
    tokens arrive one at a time, in order, and pass through all layers; at
    every layer the token appends its rotated key (explicit R_Theta per head)
    and gated value to that layer's cache and attends to the cache as it then
    stands (every earlier token and itself). No full-sequence score matrix is
    ever formed. Returns the H rows and each layer's cache rows of the tokens
    at positions >= cached[u], packed in user order."""
    X = np.asarray(inp["x"], dtype=np.float64)
    ts = [int(t) for t in inp["ts"]]
    taus = [int(t) for t in inp["taus"]]
    H = len(taus)
    d = X.shape[1]
    hd = d // H
    base = float(inp["rope_base"])
    layers = inp["layers"]
    cu = [int(c) for c in inp["cu_seqlens"]]
    h_rows, k_rows, v_rows = [], [[] for _ in layers], [[] for _ in layers]
    for u in range(len(cu) - 1):
        s, e = cu[u], cu[u + 1]
        kc = [[] for _ in layers]  # per layer: rotated keys of the tokens seen so far
        vc = [[] for _ in layers]  # per layer: gated values
        for i in range(s, e):
            pos = i - s
            idx = [pos if tau == 0 else bucket(ts[i], ts[s], tau) for tau in taus]
            x = [float(c) for c in X[i]]
            for l, lay in enumerate(layers, start=1):
                post = l <= inp["l_switch"]
                g, b, a = lay["ln_attn_g"], lay["ln_attn_b"], float(lay["alpha_attn"])
                y = x if post else ln_row(x, g, b)
                Wb = weight_blocks(lay, d)
                q, k, v, go = (matvec(y, Wb[n]) for n in ("q", "k", "v", "go"))
                if "gq" in Wb:
                    q, k = gate_mul(q, matvec(y, Wb["gq"])), gate_mul(k, matvec(y, Wb["gk"]))
                vgt = gate_mul(v, matvec(y, Wb["gv"])) if "gv" in Wb else np.array(v)
                qr, kr = np.zeros(d), np.zeros(d)
                for h in range(H):
                    sl = slice(h * hd, (h + 1) * hd)
                    R = R_matrix(idx[h], hd, base)
                    qr[sl] = R @ q[sl]
                    kr[sl] = R @ k[sl]
                kc[l - 1].append(kr)
                vc[l - 1].append(vgt)
                o = np.zeros(d)
                for h in range(H):
                    sl = slice(h * hd, (h + 1) * hd)
                    p = softmax_list([float(qr[sl] @ km[sl]) / math.sqrt(hd) for km in kc[l - 1]])
                    for m, pm in enumerate(p):
                        o[sl] += pm * vc[l - 1][m][sl]
                upd = matvec([o[c] * sig(go[c]) for c in range(d)], lay["w_o"])
                x = [x[c] + a * upd[c] for c in range(d)]
                if post:
                    x = ln_row(x, g, b)
                if lay.get("w_ffn13") is not None:
                    g, b, a = lay["ln_ffn_g"], lay["ln_ffn_b"], float(lay["alpha_ffn"])
                    y = x if post else ln_row(x, g, b)
                    upd = ffn([y], lay)[0]
                    x = [x[c] + a * upd[c] for c in range(d)]
                    if post:
                        x = ln_row(x, g, b)
            if pos >= int(cached[u]):
                h_rows.append(x)
                for l in range(len(layers)):
                    k_rows[l].append(kc[l][-1])
                    v_rows[l].append(vc[l][-1])
    shape = (-1, d)
    return (np.array(h_rows, dtype=np.float64).reshape(shape),
            [(np.array(k_rows[l]).reshape(shape), np.array(v_rows[l]).reshape(shape)) for l in range(len(layers))])


def cross_decode(Hmem, cu_seqlens, req_user, req_cutoff, cu_cands, z, dec, n_heads):
    Hm = np.asarray(Hmem, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    N, K, d = z.shape
    hd = d // n_heads
    y = np.zeros((N, K, d))
    for r in range(len(req_user)):
        s = int(cu_seqlens[int(req_user[r])])
        c = int(req_cutoff[r])
        for n in range(int(cu_cands[r]), int(cu_cands[r + 1])):
            for k in range(K):
                q = matvec(z[n, k], dec["w_q"][k])
                g = [sig(a) for a in matvec(z[n, k], dec["w_go"][k])]
                o = np.zeros(d)
                for h in range(n_heads):
                    sl = slice(h * hd, (h + 1) * hd)
                    sc = [float(q[sl] @ Hm[s + j, sl]) / math.sqrt(hd) for j in range(c)]
                    p = softmax_list(sc)
                    for j in range(c):
                        o[sl] += p[j] * Hm[s + j, sl]
                y[n, k] = matvec([o[i] * g[i] for i in range(d)], dec["w_o"])
    return y


def score_head(z, y, sp):
    """Decoder block and score, candidate by candidate and token by token:
    a = z + y; u = LN_k(a); f = a + SwiGLU_k(u); score = f[token 0] . w_s + b_s."""
    z = np.asarray(z, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    N, K, d = z.shape
    f = np.zeros((N, K, d))
    score = np.zeros(N)
    for n in range(N):
        for k in range(K):
            a = [z[n, k, i] + y[n, k, i] for i in range(d)]
            u = ln_row(a, sp["ln_g"][k], sp["ln_b"][k])
            hid = ffn([u], {"w_ffn13": sp["w_ffn13"][k], "w_ffn2": sp["w_ffn2"][k]})[0]
            for i in range(d):
                f[n, k, i] = a[i] + hid[i]
        score[n] = sum(f[n, 0, i] * float(sp["w_s"][i]) for i in range(d)) + float(sp["b_s"])
    return f, score

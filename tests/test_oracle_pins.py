"""Pins of the fp64 oracle to things other than itself (no GPU needed).

Each check ties the oracle to the ReST page ("From Language to Behavior",
ReST reading) through an identity the page states, a closed form, a library
routine (torch fp64 attention / layer norm), or a literal loop
implementation with explicit rotation matrices (oracle/brute.py).
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import brute
from oracle import rest_oracle as O


def tiny_inputs(seed=3, lengths=(7, 5), d=16, n_heads=4, n_layers=2, l_switch=1, alpha=0.5,
                levels=(7, 600, 86400), requests=None, ln_affine=True, ffn=True, n_rope=None):
    w = W.small_workload("f32", lengths=lengths, d=d, n_heads=n_heads, n_layers=n_layers, n_rope=n_rope,
                         l_switch=l_switch, alpha=alpha, levels=list(levels), ffn=ffn,
                         requests=requests, ncand=3, duplicate_frac=0.2)
    return w, W.make_inputs(w, seed, ln_affine=ln_affine)


def rel_err(a, b):
    return np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(1e-300, np.max(np.abs(b)))


# ----------------------------------------------------------------- buckets

def test_buckets_match_integer_brute_force():
    w = W.small_workload("f32", lengths=(300, 129, 64, 1), d=32, n_heads=8, n_rope=2,
                         levels=[1, 7, 60, 600, 3600, 86400], duplicate_frac=0.1)
    inp = W.make_inputs(w, 11)
    got = O.rotation_index(inp["ts"], inp["cu_seqlens"], inp["taus"])
    want = np.array(brute.index_table(inp["ts"], inp["cu_seqlens"], inp["taus"]), dtype=np.int64)
    assert got.dtype == np.int64
    assert np.array_equal(got, want)


def test_bucket_unit_granularity_is_time_offset_and_shift_free():
    w = W.small_workload("f32", lengths=(50, 20), d=8, n_heads=2, n_rope=0, levels=[1])
    inp = W.make_inputs(w, 5)
    idx = O.rotation_index(inp["ts"], inp["cu_seqlens"], inp["taus"])
    for u in range(2):
        s, e = inp["cu_seqlens"][u], inp["cu_seqlens"][u + 1]
        assert np.array_equal(idx[s:e, 0], inp["ts"][s:e] - inp["ts"][s])
    shifted = O.rotation_index(inp["ts"] + 987_654_321, inp["cu_seqlens"], inp["taus"])
    assert np.array_equal(idx, shifted)


def test_rope_heads_use_zero_based_position():
    w = W.small_workload("f32", lengths=(9, 4), d=8, n_heads=2, n_rope=2)
    inp = W.make_inputs(w, 5)
    idx = O.rotation_index(inp["ts"], inp["cu_seqlens"], inp["taus"])
    assert list(idx[:9, 0]) == list(range(9)) and list(idx[9:, 1]) == list(range(4))


def test_unsorted_timestamps_rejected():
    ts = np.array([5, 6, 4], dtype=np.int64)
    with pytest.raises(O.UnsortedTimestamps):
        O.rotation_index(ts, np.array([0, 3]), np.array([1]))


def test_equal_timestamps_are_legal():
    ts = np.array([100, 100, 100, 250], dtype=np.int64)
    idx = O.rotation_index(ts, np.array([0, 4]), np.array([0, 100]))
    assert list(idx[:, 1]) == [0, 0, 0, 1]


# ---------------------------------------------------------------- rotation

def test_rotation_matches_explicit_block_diagonal_matrix():
    rng = np.random.default_rng(0)
    hd, H = 8, 3
    idx = rng.integers(-50_000, 40_000_000, size=(5, H))
    v = rng.standard_normal((5, H * hd))
    phi = O.rotation_angles(idx, hd, 10000.0)
    got = O.rotate(v, phi)
    for i in range(5):
        for h in range(H):
            R = brute.R_matrix(int(idx[i, h]), hd, 10000.0)
            want = R @ v[i, h * hd:(h + 1) * hd]
            assert np.allclose(got[i, h * hd:(h + 1) * hd], want, rtol=0, atol=1e-9)


def test_rotation_scores_depend_only_on_index_difference():
    """Eq. 14: (R(n) q)^T (R(m) k) = q^T R(m - n) k."""
    rng = np.random.default_rng(1)
    hd = 16
    q, k = rng.standard_normal((1, hd)), rng.standard_normal((1, hd))
    for n, m in [(0, 0), (3, 17), (1000, -5), (123456, 123400)]:
        lhs = O.rotate(q, O.rotation_angles(np.array([[n]]), hd, 1e4)) @ \
            O.rotate(k, O.rotation_angles(np.array([[m]]), hd, 1e4)).T
        rhs = q @ O.rotate(k, O.rotation_angles(np.array([[m - n]]), hd, 1e4)).T
        assert abs(lhs - rhs).item() < 1e-10
        R = brute.R_matrix(m - n, hd, 1e4)
        assert abs((q @ R @ k.T) - rhs).item() < 1e-10


def test_frequencies_follow_rope_schedule():
    th = O.frequencies(8, 10000.0)
    assert th[0] == 1.0 and np.isclose(th[1], 10000.0 ** -0.25) and np.isclose(th[3], 10000.0 ** -0.75)


# ------------------------------------------------------------ elementwise

def test_layer_norm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 24)) * 3 + 1
    g, b = rng.standard_normal(24), rng.standard_normal(24)
    want = torch.nn.functional.layer_norm(torch.from_numpy(x), (24,), torch.from_numpy(g),
                                          torch.from_numpy(b), eps=1e-5).numpy()
    assert rel_err(O.layer_norm(x, g, b), want) < 1e-13


def test_gates_and_silu_closed_forms():
    assert O.sigmoid(np.array(0.0)) == 0.5
    assert O.silu(np.array(0.0)) == 0.0
    z = np.array([-3.0, 0.7, 20.0])
    assert np.allclose(O.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(), rtol=1e-15)
    assert np.allclose(O.sigmoid(z), torch.sigmoid(torch.from_numpy(z)).numpy(), rtol=1e-15)


def test_softmax_rows_sum_to_one_and_are_causal():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal((40, 8)), rng.standard_normal((40, 8))
    P = O.causal_attention_probs(q, k, 1 / math.sqrt(8))
    assert np.max(np.abs(P.sum(axis=1) - 1.0)) < 1e-12
    assert np.all(P[np.triu_indices(40, 1)] == 0.0)
    assert P[0, 0] == 1.0


# ------------------------------------------------------ whole-model pins

def test_oracle_matches_literal_brute_force():
    req = [(0, 7, 3), (0, 4, 2), (1, 5, 2), (1, 1, 1)]
    w, inp = tiny_inputs(requests=req)
    Hm = O.encoder(inp)
    Hb = brute.encoder(inp)
    assert rel_err(Hm, Hb) < 1e-12
    args = (inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"], inp["z"], inp["dec"], 4)
    assert rel_err(O.cross_decode(Hm, *args), brute.cross_decode(Hm, *args)) < 1e-12


def test_oracle_matches_brute_force_attention_only_prelayers():
    w, inp = tiny_inputs(seed=9, lengths=(6, 3, 1), n_layers=3, l_switch=0, ffn=False)
    assert rel_err(O.encoder(inp), brute.encoder(inp)) < 1e-12


def _sdpa(q, k, v, causal):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal)[0, 0].numpy()


def test_reduces_to_textbook_causal_attention_without_gates_and_angles():
    """Eq. 3 with both gates at 1 and zero angles is softmax(QK^T/sqrt(d_h)+M)V."""
    w, inp = tiny_inputs(seed=6, lengths=(33, 17), d=32, n_heads=4, n_layers=1, l_switch=0,
                         alpha=1.0, ffn=False)
    lay = inp["layers"][0]
    got = O.encoder(inp, gates=False, angle_scale=0.0)
    x = inp["x"].astype(np.float64)
    y = torch.nn.functional.layer_norm(torch.from_numpy(x), (32,), torch.from_numpy(lay["ln_attn_g"].astype(np.float64)),
                                       torch.from_numpy(lay["ln_attn_b"].astype(np.float64)), eps=1e-5).numpy()
    Wm = lay["w_qkvgg"].astype(np.float64)
    Q, K, V = y @ Wm[:, :32], y @ Wm[:, 32:64], y @ Wm[:, 64:96]
    Oa = np.zeros_like(Q)
    for u in range(2):
        s, e = inp["cu_seqlens"][u], inp["cu_seqlens"][u + 1]
        for h in range(4):
            c = slice(8 * h, 8 * h + 8)
            Oa[s:e, c] = _sdpa(Q[s:e, c], K[s:e, c], V[s:e, c], True)
    want = x + Oa @ lay["w_o"].astype(np.float64)
    assert rel_err(got, want) < 1e-12


def test_decoder_matches_library_attention_with_gates():
    w = W.small_workload("f32", lengths=(50, 20), d=32, n_heads=4,
                         requests=[(0, 50, 5), (0, 13, 4), (1, 20, 3)])
    inp = W.make_inputs(w, 8)
    Hm = W.make_memory(w, 8).astype(np.float64)
    got = O.cross_decode(Hm, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"],
                         inp["z"], inp["dec"], 4)
    z = inp["z"].astype(np.float64)
    dec = {k: v.astype(np.float64) for k, v in inp["dec"].items()}
    for r in range(3):
        s = inp["cu_seqlens"][inp["req_user"][r]]
        c = inp["req_cutoff"][r]
        for n in range(inp["cu_cands"][r], inp["cu_cands"][r + 1]):
            for k in range(3):
                q = z[n, k] @ dec["w_q"][k]
                g = torch.sigmoid(torch.from_numpy(z[n, k] @ dec["w_go"][k])).numpy()
                o = np.zeros(32)
                for h in range(4):
                    cs = slice(8 * h, 8 * h + 8)
                    o[cs] = _sdpa(q[None, cs], Hm[s:s + c, cs], Hm[s:s + c, cs], False)[0]
                assert rel_err(got[n, k], (o * g) @ dec["w_o"]) < 1e-12


def test_first_causal_row_closed_form():
    """Row 0 attends only to itself: its output is (V'_0 * sigma(Go_0)) W_o."""
    w, inp = tiny_inputs(seed=12, lengths=(9, 4), d=16, n_layers=1)
    lay = inp["layers"][0]
    y = O.layer_norm(inp["x"].astype(np.float64), lay["ln_attn_g"], lay["ln_attn_b"])
    idx = O.rotation_index(inp["ts"], inp["cu_seqlens"], inp["taus"])
    phi = O.rotation_angles(idx, 4, 1e4)
    sub = O.dga_sublayer(y, phi, inp["cu_seqlens"], lay, 4)
    Wm = lay["w_qkvgg"].astype(np.float64)
    for s in inp["cu_seqlens"][:-1]:
        v = y[s] @ Wm[:, 32:48] * O.sigmoid(y[s] @ Wm[:, 48:64])
        want = (v * O.sigmoid(y[s] @ Wm[:, 64:80])) @ lay["w_o"]
        assert rel_err(sub[s], want) < 1e-13


def test_decoder_cutoff_one_closed_form():
    w = W.small_workload("f32", lengths=(10,), d=16, n_heads=2, requests=[(0, 1, 4)])
    inp = W.make_inputs(w, 2)
    Hm = W.make_memory(w, 2).astype(np.float64)
    y = O.cross_decode(Hm, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"],
                       inp["z"], inp["dec"], 2)
    for n in range(4):
        for k in range(3):
            g = O.sigmoid(inp["z"][n, k] @ inp["dec"]["w_go"][k].astype(np.float64))
            assert rel_err(y[n, k], (Hm[0] * g) @ inp["dec"]["w_o"]) < 1e-13


def test_srn_alpha_zero_is_identity_or_pure_norm():
    w, inp = tiny_inputs(seed=13, n_layers=1, l_switch=0, alpha=0.0)
    assert np.array_equal(O.encoder(inp), inp["x"].astype(np.float64))
    w, inp = tiny_inputs(seed=13, n_layers=1, l_switch=1, alpha=0.0)
    lay = inp["layers"][0]
    x = inp["x"].astype(np.float64)
    want = O.layer_norm(O.layer_norm(x, lay["ln_attn_g"], lay["ln_attn_b"]), lay["ln_ffn_g"], lay["ln_ffn_b"])
    assert rel_err(O.encoder(inp), want) < 1e-14
    t = torch.nn.functional.layer_norm(torch.from_numpy(x), (16,), torch.from_numpy(lay["ln_attn_g"].astype(np.float64)),
                                       torch.from_numpy(lay["ln_attn_b"].astype(np.float64)), eps=1e-5)
    t = torch.nn.functional.layer_norm(t, (16,), torch.from_numpy(lay["ln_ffn_g"].astype(np.float64)),
                                       torch.from_numpy(lay["ln_ffn_b"].astype(np.float64)), eps=1e-5)
    assert rel_err(O.encoder(inp), t.numpy()) < 1e-13


# ------------------------------------------------------------ invariances

def test_rope_scores_invariant_under_global_position_shift():
    w, inp = tiny_inputs(seed=14, lengths=(40, 23), d=32, n_heads=4, n_layers=2)
    a = O.encoder(inp)
    b = O.encoder(inp, pos_offset=100_003)
    assert rel_err(b, a) < 1e-9


def test_rote_invariant_under_whole_coarsest_bucket_shift():
    """With a fixed time origin, shifting every timestamp by k * tau_max moves
    every bucket by a whole number (each tau divides tau_max), so the
    pairwise differences (eq. 14) and the output do not change."""
    levels = (1, 600, 86400 * 4)
    w, inp = tiny_inputs(seed=15, lengths=(40, 23), d=32, n_heads=4, n_rope=1, levels=levels)
    origin = [int(inp["ts"][s]) - 12_345 for s in inp["cu_seqlens"][:-1]]
    a = O.encoder(inp, time_origin=origin)
    shifted = dict(inp, ts=inp["ts"] + 3 * 86400 * 4)
    b = O.encoder(shifted, time_origin=origin)
    assert rel_err(b, a) < 1e-9
    # negative control: half a 600 s bucket moves some bucket boundaries
    c = O.encoder(dict(inp, ts=inp["ts"] + 300), time_origin=origin)
    assert rel_err(c, a) > 1e-6


def test_causality_rows_unchanged_when_later_tokens_change():
    w, inp = tiny_inputs(seed=16, lengths=(40, 23), d=32, n_heads=4, n_layers=2)
    a = O.encoder(inp)
    i = 17
    x2, ts2 = inp["x"].copy(), inp["ts"].copy()
    rng = np.random.default_rng(0)
    x2[i + 1:40] = rng.standard_normal((40 - i - 1, 32)).astype(np.float32)
    ts2[i + 1:40] = ts2[i + 1:40] + rng.integers(0, 5000)
    b = O.encoder(dict(inp, x=x2, ts=ts2))
    assert np.array_equal(a[:i + 1], b[:i + 1])
    assert np.array_equal(a[40:], b[40:])
    assert not np.allclose(a[i + 1:40], b[i + 1:40])


def test_candidate_permutation_equivariance():
    w = W.small_workload("f32", lengths=(60,), d=32, n_heads=4, requests=[(0, 60, 9)])
    inp = W.make_inputs(w, 17)
    Hm = W.make_memory(w, 17)
    args = lambda z: (Hm, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"], z, inp["dec"], 4)
    perm = np.random.default_rng(1).permutation(9)
    a = O.cross_decode(*args(inp["z"]))
    b = O.cross_decode(*args(inp["z"][perm]))
    assert rel_err(b, a[perm]) < 1e-14


def test_shared_prefix_equals_scoring_each_candidate_alone():
    w = W.small_workload("f32", lengths=(60, 30), d=32, n_heads=4, requests=[(0, 60, 6), (1, 11, 4)])
    inp = W.make_inputs(w, 18)
    Hm = W.make_memory(w, 18)
    together = O.cross_decode(Hm, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"],
                              inp["z"], inp["dec"], 4)
    for r in range(2):
        for n in range(inp["cu_cands"][r], inp["cu_cands"][r + 1]):
            alone = O.cross_decode(Hm, inp["cu_seqlens"], [inp["req_user"][r]], [inp["req_cutoff"][r]],
                                   [0, 1], inp["z"][n:n + 1], inp["dec"], 4)
            assert rel_err(alone[0], together[n]) < 1e-13


def test_union_encoding_equals_encoding_each_prefix_alone():
    """§3.5: encode the union history once; a request at cutoff c reads
    H[0:c], which equals encoding the first c tokens alone."""
    w, inp = tiny_inputs(seed=19, lengths=(40,), d=32, n_heads=4, n_layers=2,
                         requests=[(0, 40, 3), (0, 21, 3)])
    Hm, y = O.rank_request(inp)
    c = 21
    sub = dict(inp, x=inp["x"][:c], ts=inp["ts"][:c], cu_seqlens=np.array([0, c], dtype=np.int32))
    Hc = O.encoder(sub)
    assert rel_err(Hc, Hm[:c]) < 1e-13
    yc = O.cross_decode(Hc, sub["cu_seqlens"], [0], [c], [0, 3], inp["z"][3:6], inp["dec"], 4)
    assert rel_err(yc, y[3:6]) < 1e-12


# ---------------------------------------------- gate variants (ablation flags)

def gate_inputs(gates, seed, n_rope=2, lengths=(7, 5), n_layers=2):
    w = W.small_workload("f32", lengths=lengths, d=16, n_heads=4, n_rope=n_rope, n_layers=n_layers, l_switch=1,
                         alpha=0.5, levels=[7, 600, 86400], ncand=3, duplicate_frac=0.2, gates=gates)
    return W.make_inputs(w, seed, ln_affine=True)


def with_blocks(inp, gates, build):
    """inp with every layer's projection weight replaced by build(blocks of d columns)."""
    d = inp["x"].shape[1]
    layers = []
    for lay in inp["layers"]:
        W_ = np.asarray(lay["w_qkvgg"], dtype=np.float64)
        blocks = [W_[:, i * d:(i + 1) * d] for i in range(W_.shape[1] // d)]
        layers.append(dict(lay, w_qkvgg=np.concatenate(build(blocks), axis=1), gates=gates))
    return dict(inp, layers=layers)


@pytest.mark.parametrize("gates", ["o", "qkvo"])
def test_gate_variants_match_literal_brute_force(gates):
    inp = gate_inputs(gates, 24)
    assert rel_err(O.encoder(inp), brute.encoder(inp)) < 1e-12
    Hn, kv, _ = O.encoder_append(inp, [3, 2])
    Hb, kvb = brute.encoder_stream(inp, [3, 2])
    assert rel_err(Hn, Hb) < 1e-12
    for (k, v), (kb, vb) in zip(kv, kvb):
        assert rel_err(k, kb) < 1e-12 and rel_err(v, vb) < 1e-12


def test_output_gate_only_is_dga_with_a_constant_half_value_gate():
    """sigmoid(0) = 1/2 exactly: the DGA layer with W_gv = 0 and W_V doubled has
    V' = V, which is the layer with the output gate alone."""
    inp = gate_inputs("o", 25)
    same = with_blocks(inp, "vo", lambda b: [b[0], b[1], 2.0 * b[2], 0.0 * b[2], b[3]])
    assert rel_err(O.encoder(inp), O.encoder(same)) < 1e-14


def test_qkv_gates_with_zero_gate_weights_halve_q_and_k():
    """With W_gq = W_gk = 0 the Q and K gates are the constant 1/2: the DGA
    layer with W_Q and W_K halved."""
    inp = with_blocks(gate_inputs("qkvo", 26), "qkvo", lambda b: b[:5] + [0.0 * b[5], 0.0 * b[6]])
    same = with_blocks(inp, "vo", lambda b: [0.5 * b[0], 0.5 * b[1]] + b[2:5])
    assert rel_err(O.encoder(inp), O.encoder(same)) < 1e-14


def test_qkv_gates_keep_scores_relative_in_position():
    """Q and K are gated before the rotation, so a global shift of every
    RoPE position leaves the layer's output unchanged (eq. 14); gating after
    the rotation would not."""
    inp = gate_inputs("qkvo", 27, n_rope=4, lengths=(30,), n_layers=1)
    assert rel_err(O.encoder(inp, pos_offset=12345), O.encoder(inp)) < 1e-10


# ------------------------------------------------ attention core and its backward (ULT)

def core_inputs(seed, lengths=(5, 3, 1), n_heads=2, hd=4):
    rng = np.random.default_rng(seed)
    T, d = sum(lengths), n_heads * hd
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    q, k, v, d_o = (rng.standard_normal((T, d)) for _ in range(4))
    return q, k, v, d_o, cu, n_heads


def test_attention_core_matches_torch_sdpa_forward_and_autograd():
    q, k, v, d_o, cu, H = core_inputs(30, lengths=(7, 4))
    O_, lse = O.attention_core(q, k, v, cu, H)
    dq, dk, dv = O.attention_core_backward(q, k, v, cu, H, d_o)
    hd = q.shape[1] // H
    for u in range(len(cu) - 1):
        s, e = cu[u], cu[u + 1]
        for h in range(H):
            c = slice(h * hd, (h + 1) * hd)
            tq, tk, tv = (torch.tensor(a[s:e, c], dtype=torch.float64, requires_grad=True) for a in (q, k, v))
            out = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None], is_causal=True)[0]
            (out * torch.tensor(d_o[s:e, c])).sum().backward()
            assert rel_err(O_[s:e, c], out.detach().numpy()) < 1e-13
            for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
                assert rel_err(mine[s:e, c], ref.grad.numpy()) < 1e-12
            S = (q[s:e, c] @ k[s:e, c].T) / math.sqrt(hd)
            want = [math.log(sum(math.exp(S[i, j]) for j in range(i + 1))) for i in range(e - s)]
            assert np.max(np.abs(lse[s:e, h] - np.array(want))) < 1e-12


def test_attention_core_backward_matches_finite_differences():
    q, k, v, d_o, cu, H = core_inputs(31)
    loss = lambda q_, k_, v_: float((O.attention_core(q_, k_, v_, cu, H)[0] * d_o).sum())
    grads = O.attention_core_backward(q, k, v, cu, H, d_o)
    eps = 1e-5
    for which, g in enumerate(grads):
        fd = np.zeros_like(q)
        for i in range(q.shape[0]):
            for c in range(q.shape[1]):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][i, c] += eps
                args_m[which][i, c] -= eps
                fd[i, c] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert np.max(np.abs(fd - g)) < 1e-8 * max(1.0, np.max(np.abs(g)))


def test_attention_core_backward_closed_forms():
    """Per user and head: the values' gradients sum to the sum of dO (each
    softmax row sums to 1); the keys' gradients sum to zero (each row of dS
    sums to zero); a first row sees one key, so its query gets no gradient."""
    q, k, v, d_o, cu, H = core_inputs(32, lengths=(9, 6, 1), n_heads=3, hd=4)
    dq, dk, dv = O.attention_core_backward(q, k, v, cu, H, d_o)
    for u in range(len(cu) - 1):
        s, e = cu[u], cu[u + 1]
        assert np.allclose(dv[s:e].sum(axis=0), d_o[s:e].sum(axis=0), atol=1e-12)
        assert np.allclose(dk[s:e].sum(axis=0), 0.0, atol=1e-12)
        assert np.all(dq[s] == 0.0)


def test_row_sampled_dq_equals_full_backward():
    q, k, v, d_o, cu, H = core_inputs(35, lengths=(13, 6, 1), n_heads=2, hd=8)
    dq, _, _ = O.attention_core_backward(q, k, v, cu, H, d_o)
    rows = [0, 1, 12, 13, 18, 19]
    assert rel_err(O.attention_core_dq_rows(q, k, v, cu, H, d_o, rows), dq[rows]) < 1e-12


def test_ult_union_gradient_is_the_sum_of_per_sample_gradients():
    """ULT (§3.5): a user's samples ending at rows c_1 < c_2 < ... are encoded
    once as their union history; with the causal mask, a loss that reads each
    sample's own rows gives, on the union, the sum of the gradients each
    sample would give encoded alone on its prefix."""
    q, k, v, _, _, H = core_inputs(33, lengths=(11,), n_heads=2, hd=4)
    rng = np.random.default_rng(34)
    cuts = [4, 8, 11]
    d_os = []
    for c in cuts:  # sample m's loss reads rows < c_m of the history
        g = np.zeros_like(q)
        g[:c] = rng.standard_normal((c, q.shape[1]))
        d_os.append(g)
    union = O.attention_core_backward(q, k, v, np.array([0, 11]), H, sum(d_os))
    alone = [np.zeros_like(q) for _ in range(3)]
    for c, g in zip(cuts, d_os):
        parts = O.attention_core_backward(q[:c], k[:c], v[:c], np.array([0, c]), H, g[:c])
        for acc, p_ in zip(alone, parts):
            acc[:c] += p_
    for a, b in zip(union, alone):
        assert rel_err(a, b) < 1e-12


# ------------------------------------------------- append-only encoder cache

def truncate(inp, lengths):
    """Each user's first lengths[u] tokens, in the encoder's input form."""
    cu = inp["cu_seqlens"]
    rows = np.concatenate([np.arange(cu[u], cu[u] + lengths[u]) for u in range(len(lengths))])
    cu2 = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu2[1:] = np.cumsum(lengths)
    return dict(inp, x=inp["x"][rows], ts=inp["ts"][rows], cu_seqlens=cu2)


@pytest.mark.parametrize("l_switch,ffn", [(1, True), (0, False), (2, True)])
def test_encoder_append_matches_token_by_token_stream(l_switch, ffn):
    """The append's definition (rows of the full-history encoder) against a
    server loop that sees one token at a time and only a per-layer cache of
    rotated keys and gated values."""
    w, inp = tiny_inputs(seed=21, lengths=(7, 5, 3), n_layers=2, l_switch=l_switch, ffn=ffn, n_rope=1)
    cached = [3, 0, 3]
    Hn, kv, cu_new = O.encoder_append(inp, cached)
    Hb, kvb = brute.encoder_stream(inp, cached)
    assert list(cu_new) == [0, 4, 9, 9]
    assert Hn.shape == (9, 16) and len(kv) == 2
    assert rel_err(Hn, Hb) < 1e-12
    for (k, v), (kb, vb) in zip(kv, kvb):
        assert rel_err(k, kb) < 1e-12 and rel_err(v, vb) < 1e-12


def test_cache_of_a_prefix_is_unchanged_by_later_tokens():
    """Keys, values and H cached while the history was shorter stay valid:
    the prefix alone gives the prefix rows of the longer history (causality,
    and RoTE's origin is the first timestamp, which appending keeps)."""
    w, inp = tiny_inputs(seed=22, lengths=(9, 6), n_layers=2, l_switch=1, n_rope=1)
    cut = [4, 2]
    H_pre, kv_pre, _ = O.encoder_append(truncate(inp, cut), [0, 0])
    H_all, kv_all, _ = O.encoder_append(inp, [0, 0])
    rows = np.r_[0:4, 9:11]
    assert rel_err(H_pre, H_all[rows]) < 1e-13
    for (kp, vp), (ka, va) in zip(kv_pre, kv_all):
        assert rel_err(kp, ka[rows]) < 1e-13 and rel_err(vp, va[rows]) < 1e-13
    # the rest of the history, appended to that cache, gives the remaining rows
    H_new, kv_new, cu_new = O.encoder_append(inp, cut)
    rest = np.r_[4:9, 11:15]
    assert list(cu_new) == [0, 5, 9]
    assert rel_err(H_new, H_all[rest]) < 1e-13


def test_encoder_append_of_nothing_and_of_everything():
    w, inp = tiny_inputs(seed=23, lengths=(5, 4), n_layers=1, l_switch=0)
    H_new, kv, cu_new = O.encoder_append(inp, [5, 4])
    assert H_new.shape == (0, 16) and list(cu_new) == [0, 0, 0] and kv[0][0].shape == (0, 16)
    H_all, _, _ = O.encoder_append(inp, [0, 0])
    assert np.array_equal(H_all, O.encoder(inp))
    with pytest.raises(ValueError):
        O.encoder_append(inp, [6, 0])


# ------------------------------------------------------------ input module

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(20)
    x = (rng.standard_normal(100_000) * 10.0 ** rng.integers(-6, 6, 100_000)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(W.round_bf16(x), want)


def test_named_workloads_are_well_formed():
    for i in range(5):
        w = W.workload(i)
        assert w.d == w.n_heads * w.head_dim and w.head_dim % 2 == 0
        assert all(1 <= c <= w.lengths[u] for u, c in zip(w.req_user, w.req_cutoff))
    w = W.workload(4)
    assert 128 <= min(w.lengths) and max(w.lengths) <= 16384 and w.n_users == 64
    assert 64 <= min(w.req_ncand) and max(w.req_ncand) <= 1024
    assert list(W.workload(1).taus) == [0, 0, 0, 0, 1, 4096, 524288, 33554432]
    assert list(W.workload(0).taus) == [0, 0, 64, 65536]
    assert [W.ffn_width(d) for d in (64, 256, 512)] == [192, 704, 1408]


@pytest.mark.parametrize("l_switch,ffn", [(0, True), (1, True), (0, False)])
def test_row_sampled_encoder_equals_full_encoder(l_switch, ffn):
    w, inp = tiny_inputs(seed=21, lengths=(40, 23), d=32, n_heads=4, n_layers=1, l_switch=l_switch, ffn=ffn)
    full = O.encoder(inp)
    rows = [0, 5, 39, 40, 41, 62]
    assert rel_err(O.encoder_rows(inp, rows), full[rows]) < 1e-13


# ------------------------------------------------------------ decoder block and score (eq. 8, R23-R25)

def _score_case(seed=31, n=4, K=3, d=16, ln_affine=True):
    w, inp = tiny_inputs(seed=seed, lengths=(9,), d=d, n_heads=4, n_layers=1, requests=[(0, 9, n)],
                         ln_affine=ln_affine)
    rng = np.random.default_rng(seed + 1)
    y = rng.standard_normal(inp["z"].shape)
    return inp["z"], y, inp["score"]


def test_score_head_matches_brute_force():
    z, y, sp = _score_case()
    f, s = O.score_head(z, y, sp)
    fb, sb = brute.score_head(z, y, sp)
    assert rel_err(f, fb) < 1e-13 and rel_err(s, sb) < 1e-13


def test_score_head_without_ffn_is_the_residual_sum():
    """W_2 = 0 removes the FFN: f = z + y exactly and the score is its [CLS] logit."""
    z, y, sp = _score_case(seed=32)
    sp0 = dict(sp, w_ffn2=np.zeros_like(sp["w_ffn2"]))
    f, s = O.score_head(z, y, sp0)
    a = z.astype(np.float64) + y
    assert np.array_equal(f, a)
    assert rel_err(s, a[:, 0] @ sp["w_s"].astype(np.float64) + sp["b_s"]) < 1e-14


def test_score_head_single_token_type_is_the_encoder_pre_ln_ffn_sublayer():
    """With one token type the block's FFN is eq. 6's pre-LN sublayer with alpha = 1."""
    z, y, sp = _score_case(seed=33)
    sp1 = {k: (v[:1] if isinstance(v, np.ndarray) and v.ndim >= 2 else v) for k, v in sp.items()}
    f, _ = O.score_head(z[:, :1], y[:, :1], sp1)
    a = z[:, 0].astype(np.float64) + y[:, 0]
    layer = {"w_ffn13": sp["w_ffn13"][0], "w_ffn2": sp["w_ffn2"][0]}
    want = O.srn(a, lambda u: O.ffn_sublayer(u, layer), 1.0, False, sp["ln_g"][0], sp["ln_b"][0])
    assert rel_err(f[:, 0], want) < 1e-14


def test_score_head_token_types_use_only_their_own_parameters():
    """Eq. 8: swapping the parameters of token types 1 and 2 together with their
    input rows swaps their outputs; changing type 2's weights leaves types 0 and 1."""
    z, y, sp = _score_case(seed=34)
    f, s = O.score_head(z, y, sp)
    perm = [0, 2, 1]
    spp = {k: (v[perm] if isinstance(v, np.ndarray) and v.ndim >= 2 else v) for k, v in sp.items()}
    fp, sp_score = O.score_head(z[:, perm], y[:, perm], spp)
    assert rel_err(fp, f[:, perm]) < 1e-14 and rel_err(sp_score, s) < 1e-14
    sp2 = dict(sp, w_ffn2=sp["w_ffn2"].copy())
    sp2["w_ffn2"][2] *= -3.0
    f2, s2 = O.score_head(z, y, sp2)
    assert np.array_equal(f2[:, :2], f[:, :2]) and np.array_equal(s2, s)
    assert not np.allclose(f2[:, 2], f[:, 2])

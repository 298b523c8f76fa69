"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small ragged cases (several 128-row tiles and a ragged tail) are compared
element by element on every output; the five named workloads run at full
size in the launch configuration the benchmark times and are compared on
sampled users, rows and requests that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import shared_prefix_behavior_b200 as R
import workloads as W
from oracle import rest_oracle as O
from tests.parity import assert_parity, subset_users

pytestmark = pytest.mark.gpu


def run_rank(inp, dev):
    t = R.to_device(inp, dev)
    H, y = R.rank_request(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"], t["reqs"],
                          t["z"], t["dec"], t["rope_base"])
    torch.cuda.synchronize()
    return H.float().cpu().numpy(), y.cpu().numpy()


def run_encoder(inp, dev):
    t = R.to_device(inp, dev)
    H = R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                       rope_base=t["rope_base"])
    return H.float().cpu().numpy()


def run_decoder(inp, Hmem, dev):
    t = R.to_device(inp, dev)
    wdt = torch.bfloat16 if inp["dtype"] == "bf16" else torch.float32
    Hd = torch.from_numpy(np.ascontiguousarray(Hmem)).to(dev, wdt)
    y = R.cross_decode(Hd, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    return y.cpu().numpy()


def oracle_decode(inp, Hmem):
    return O.cross_decode(Hmem, inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"], inp["z"],
                          inp["dec"], len(inp["taus"]))


# ------------------------------------------------------------- rotation index

@pytest.mark.parametrize("wl", ["small", "year"])
def test_rotation_table_is_exact(cuda, wl):
    if wl == "small":
        w = W.small_workload("bf16", lengths=(300, 129, 64, 1, 0, 7), d=128, n_heads=8, n_rope=2,
                             levels=[1, 7, 60, 600, 3600, 86400], duplicate_frac=0.1)
    else:
        w = W.workload(3)
    inp = W.make_inputs(w, 31)
    ts = torch.from_numpy(inp["ts"]).to(cuda)
    idx, cos, sin = R.rotation_table(ts, inp["cu_seqlens"], inp["taus"], w.head_dim, w.rope_base)
    ref = O.rotation_index(inp["ts"], inp["cu_seqlens"], inp["taus"])
    assert np.array_equal(idx.cpu().numpy(), ref)
    phi = O.rotation_angles(ref, w.head_dim, w.rope_base)
    assert np.max(np.abs(cos.cpu().numpy() - np.cos(phi))) < 2e-7
    assert np.max(np.abs(sin.cpu().numpy() - np.sin(phi))) < 2e-7


def test_unsorted_timestamps_set_the_device_status(cuda):
    w = W.small_workload("bf16", lengths=(50, 20), d=64, n_heads=2)
    inp = W.make_inputs(w, 1)
    inp["ts"][55] = inp["ts"][54] - 5
    ts = torch.from_numpy(inp["ts"]).to(cuda)
    with pytest.raises(R.RestError) as e:
        R.rotation_table(ts, inp["cu_seqlens"], inp["taus"], 32)
    assert e.value.status == 2


# ------------------------------------------------------------- fp32 workload

def test_tiny_fp32_workload_full(cuda):
    w = W.workload(0)
    inp = W.make_inputs(w, 1000)
    H, y = run_rank(inp, cuda)
    Hr, yr = O.rank_request(inp)
    assert_parity(H, Hr, "f32", "H")
    assert_parity(y, yr, "f32", "y")


@pytest.mark.parametrize("hd", [16, 32, 64])
def test_fp32_small_ragged(cuda, hd):
    w = W.small_workload("f32", lengths=(300, 129, 1, 64), d=4 * hd, n_heads=4, n_layers=2, l_switch=1,
                         requests=[(0, 300, 50), (0, 77, 3), (1, 129, 0), (2, 1, 5), (3, 64, 44)])
    inp = W.make_inputs(w, 41, ln_affine=True)
    H, y = run_rank(inp, cuda)
    Hr, yr = O.rank_request(inp)
    assert_parity(H, Hr, "f32", "H")
    assert_parity(y, yr, "f32", "y")


# ------------------------------------------------------------- bf16 small cases

@pytest.mark.parametrize("hd,n_layers,l_switch,ffn", [(32, 2, 1, True), (64, 2, 0, True), (16, 1, 0, False),
                                                       (64, 3, 3, False)])
def test_bf16_small_ragged_rank_request(cuda, hd, n_layers, l_switch, ffn):
    w = W.small_workload("bf16", lengths=(300, 129, 1, 64, 255), d=4 * hd, n_heads=4, n_layers=n_layers,
                         l_switch=l_switch, ffn=ffn,
                         requests=[(0, 300, 50), (0, 77, 3), (1, 129, 0), (2, 1, 5), (3, 64, 44), (4, 200, 43)])
    inp = W.make_inputs(w, 42, ln_affine=True)
    H, y = run_rank(inp, cuda)
    Hr, yr = O.rank_request(inp)
    assert_parity(H, Hr, "bf16", "H")
    assert_parity(y, yr, "bf16", "y")


@pytest.mark.parametrize("dtype,hd,d,gates", [("f32", 16, 64, "o"), ("f32", 32, 128, "qkvo"), ("bf16", 32, 128, "o"),
                                               ("bf16", 32, 256, "o"), ("bf16", 32, 128, "qkvo"),
                                               ("bf16", 64, 256, "qkvo")])
def test_gate_variants_small_ragged(cuda, dtype, hd, d, gates):
    """The gated-attention ablation's variants (output gate only; Q, K, V and
    output gates) through the whole forward."""
    w = W.small_workload(dtype, lengths=(300, 129, 1, 64, 255), d=d, n_heads=d // hd, n_layers=2, l_switch=1,
                         gates=gates, requests=[(0, 300, 20), (1, 129, 7), (2, 1, 3), (4, 200, 11)])
    inp = W.make_inputs(w, 61, ln_affine=True)
    H, y = run_rank(inp, cuda)
    Hr, yr = O.rank_request(inp)
    assert_parity(H, Hr, dtype, "H")
    assert_parity(y, yr, dtype, "y")


def test_bf16_decoder_with_synthetic_memory(cuda):
    w = W.small_workload("bf16", lengths=(700, 129, 3), d=256, n_heads=8,
                         requests=[(0, 700, 60), (0, 1, 2), (0, 333, 0), (1, 129, 45), (2, 2, 7), (0, 129, 1)])
    inp = W.make_inputs(w, 43)
    Hm = W.make_memory(w, 43)
    y = run_decoder(inp, Hm, cuda)
    assert_parity(y, oracle_decode(inp, Hm), "bf16", "y")


@pytest.mark.parametrize("hd", [32, 64])
def test_bf16_decoder_split_keys(cuda, hd):
    """Few query rows against long prefixes: the tensor-core decoder splits the
    keys across CTAs (the 1-key request's first split is empty) and combines
    the partial results."""
    w = W.small_workload("bf16", lengths=(2000, 300), d=4 * hd, n_heads=4,
                         requests=[(0, 2000, 20), (1, 300, 7), (0, 1, 3), (0, 1500, 2)])
    inp = W.make_inputs(w, 47)
    Hm = W.make_memory(w, 47)
    y = run_decoder(inp, Hm, cuda)
    assert_parity(y, oracle_decode(inp, Hm), "bf16", "y")


def _growing_memory(w, inp, seed):
    """A synthetic memory whose rows grow with their position in the user's
    history (x (1 + position // 128)): each 128-key block scores well above the
    ones before it."""
    Hm = W.make_memory(w, seed).astype(np.float64)
    cu = inp["cu_seqlens"]
    for u in range(len(cu) - 1):
        pos = np.arange(cu[u + 1] - cu[u])
        Hm[cu[u]:cu[u + 1]] *= (1 + pos // 128)[:, None]
    return W.round_bf16(Hm)


@pytest.mark.parametrize("hd", [32, 64])
def test_bf16_decoder_row_max_growth(cuda, hd):
    """Keys whose scores grow block by block: a row's running max rises by more
    than the kernel's 2^8 threshold several times, so it rescales the row's
    accumulated output in TMEM (the online softmax's correction)."""
    w = W.small_workload("bf16", lengths=(1000, 300), d=4 * hd, n_heads=4,
                         requests=[(0, 1000, 40), (1, 300, 9), (0, 600, 3)])
    inp = W.make_inputs(w, 49)
    Hm = _growing_memory(w, inp, 49)
    y = run_decoder(inp, Hm, cuda)
    assert_parity(y, oracle_decode(inp, Hm), "bf16", "y")


def test_decoder_reports_values_beyond_fp16(cuda):
    """The tensor-core decoder multiplies in fp16: a memory value that bf16
    holds but fp16 does not (1e5 > 65504) is reported on the device status
    word as REST_ERR_RANGE instead of turning the scores into infinities."""
    w = W.small_workload("bf16", lengths=(300,), d=128, n_heads=4, requests=[(0, 300, 5)])
    inp = W.make_inputs(w, 50)
    Hm = W.make_memory(w, 50)
    Hm[17, 5] = 1.0e5
    with pytest.raises(R.RestError) as e:
        run_decoder(inp, Hm, cuda)
    assert e.value.status == 8


@pytest.mark.parametrize("hd", [32, 64])
def test_bf16_rank_request_split_keys(cuda, hd):
    """The split decoder after an encoder in the same call, reading the fp16
    copy of H that the encoder's last launch writes beside H."""
    w = W.small_workload("bf16", lengths=(1800, 300), d=4 * hd, n_heads=4, n_layers=1, l_switch=0,
                         requests=[(0, 1800, 12), (1, 300, 5), (0, 400, 3)])
    inp = W.make_inputs(w, 48)
    H, y = run_rank(inp, cuda)
    Hr, yr = O.rank_request(inp)
    assert_parity(H, Hr, "bf16", "H")
    assert_parity(y, yr, "bf16", "y")


# ------------------------------------------------------------- properties on the GPU

def test_causality_on_gpu(cuda):
    w = W.small_workload("bf16", lengths=(400,), d=128, n_heads=4, n_layers=2, l_switch=1)
    inp = W.make_inputs(w, 44)
    a = run_encoder(inp, cuda)
    i = 200
    inp2 = dict(inp, x=inp["x"].copy(), ts=inp["ts"].copy())
    rng = np.random.default_rng(0)
    inp2["x"][i + 1:] = W.round_bf16(rng.standard_normal((400 - i - 1, 128)))
    inp2["ts"][i + 1:] += 12345
    b = run_encoder(inp2, cuda)
    assert np.array_equal(a[:i + 1], b[:i + 1])
    assert not np.array_equal(a[i + 1:], b[i + 1:])


def test_shared_prefix_equals_each_candidate_alone_on_gpu(cuda):
    w = W.small_workload("bf16", lengths=(300,), d=128, n_heads=4, requests=[(0, 300, 9)])
    inp = W.make_inputs(w, 45)
    Hm = W.make_memory(w, 45)
    together = run_decoder(inp, Hm, cuda)
    for n in range(9):
        one = dict(inp, z=inp["z"][n:n + 1], cu_cands=np.array([0, 1], dtype=np.int32))
        alone = run_decoder(one, Hm, cuda)
        assert np.max(np.abs(alone[0] - together[n])) <= 1e-5 * np.max(np.abs(together))


def test_candidate_permutation_on_gpu(cuda):
    w = W.small_workload("bf16", lengths=(200,), d=128, n_heads=4, requests=[(0, 200, 50)])
    inp = W.make_inputs(w, 46)
    Hm = W.make_memory(w, 46)
    a = run_decoder(inp, Hm, cuda)
    perm = np.random.default_rng(2).permutation(50)
    b = run_decoder(dict(inp, z=inp["z"][perm]), Hm, cuda)
    assert np.max(np.abs(b - a[perm])) <= 1e-5 * np.max(np.abs(a))


# ------------------------------------------------------------- full-size workloads

def _sampled_users(w, k, seed):
    rng = np.random.default_rng(seed)
    order = np.argsort(w.lengths)
    pick = {int(order[-1]), int(order[0])}
    while len(pick) < min(k, w.n_users):
        pick.add(int(rng.integers(0, w.n_users)))
    return sorted(pick)


@pytest.mark.parametrize("cfg,users", [(1, 3), (2, 1)])
def test_full_workload_multilayer_sampled_users(cuda, cfg, users):
    """Workloads with several layers: the whole batch on the GPU, a few users
    end to end (H and every candidate score) in the oracle."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    H, y = run_rank(inp, cuda)
    sub = subset_users(inp, _sampled_users(w, users, cfg))
    Hr, yr = O.rank_request(sub)
    assert_parity(H[sub["_rows"]], Hr, "bf16", "H")
    assert_parity(y[sub["_cand_rows"]], yr, "bf16", "y")


@pytest.mark.parametrize("cfg", [3, 4])
def test_full_workload_single_layer_sampled_rows(cuda, cfg):
    """One-layer workloads at full length: the whole batch on the GPU, sampled
    rows of H (first, last, tile edges, random) in the oracle row by row."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    H, _ = run_rank(inp, cuda)
    cu = inp["cu_seqlens"]
    rng = np.random.default_rng(cfg)
    rows = []
    for u in _sampled_users(w, 4, cfg):
        s, L = int(cu[u]), int(cu[u + 1] - cu[u])
        rows += [s, s + min(127, L - 1), s + min(128, L - 1), s + L - 1] + list(s + rng.integers(0, L, 4))
    rows = sorted(set(rows))
    assert_parity(H[rows], O.encoder_rows(inp, rows), "bf16", "H rows")


def _end_to_end_users(w, cfg):
    """Users whose whole forward the oracle runs: on the 16k workload one of
    its two users; on the ragged one the shortest user, the first user whose
    every request is under 1024 keys (short prefixes average H's fp16
    rounding least), the first user with requests on both sides of 1024
    keys, and the first user of 4096-6144 tokens."""
    if cfg == 3:
        return [0]
    L = np.asarray(w.lengths)
    ru, rc = np.asarray(w.req_user), np.asarray(w.req_cutoff)
    short = [u for u in range(w.n_users) if (rc[ru == u] < 1024).all()]
    mixed = [u for u in range(w.n_users) if (rc[ru == u] < 1024).any() and (rc[ru == u] >= 1024).any()]
    long_ = [u for u in range(w.n_users) if 4096 <= L[u] <= 6144]
    return sorted({int(np.argmin(L)), short[0], mixed[0], long_[0]})


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [3, 4])
def test_full_workload_single_layer_end_to_end(cuda, cfg):
    """The one-layer workloads at full size through rank_request, y included:
    the GPU runs the whole batch; the oracle encodes the sampled users in full
    and scores every candidate of their requests. This checks the product's
    decoder on real encoder output: the fp16 copy of H that the encoder
    writes from its fp32 residual stream, at every cutoff length (each
    request is also held to the bar on its own). The passage: scoring with a
    request's prefix of the union history equals scoring that prefix alone
    (§3.5)."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    H, y = run_rank(inp, cuda)
    users = _end_to_end_users(w, cfg)
    sub = subset_users(inp, users)
    Hr, yr = O.rank_request(sub)
    assert_parity(H[sub["_rows"]], Hr, "bf16", "H")
    yg = y[sub["_cand_rows"]]
    assert_parity(yg, yr, "bf16", "y")
    cc = sub["cu_cands"]
    for r in range(len(sub["req_user"])):
        if cc[r + 1] > cc[r]:
            assert_parity(yg[cc[r]:cc[r + 1]], yr[cc[r]:cc[r + 1]], "bf16",
                          f"request {r} (cutoff {int(sub['req_cutoff'][r])})")


@pytest.mark.parametrize("cfg,n_req", [(3, 2), (4, 6)])
def test_full_workload_decoder_sampled_requests(cuda, cfg, n_req):
    """The decoder over the full workload's requests with a synthetic memory;
    a sample of requests (all their candidates) in the oracle."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    Hm = W.make_memory(w, cfg)
    y = run_decoder(inp, Hm, cuda)
    rng = np.random.default_rng(cfg)
    reqs = sorted(set([0, w.n_req - 1] + list(rng.integers(0, w.n_req, n_req))))[:max(n_req, 2)]
    cc = inp["cu_cands"]
    for r in reqs:
        one = dict(inp, req_user=inp["req_user"][r:r + 1], req_cutoff=inp["req_cutoff"][r:r + 1],
                   cu_cands=np.array([0, cc[r + 1] - cc[r]], dtype=np.int32), z=inp["z"][cc[r]:cc[r + 1]])
        assert_parity(y[cc[r]:cc[r + 1]], oracle_decode(one, Hm), "bf16", f"request {r}")


# ------------------------------------------------------------- decoder block and candidate score

@pytest.mark.parametrize("dtype,hd", [("f32", 16), ("bf16", 32), ("bf16", 64)])
def test_score_head_small_ragged(cuda, dtype, hd):
    """Encoder, decoder and the score head end to end (eq. 8 FFN sublayer, [CLS] logit)."""
    w = W.small_workload(dtype, lengths=(300, 129, 1, 64), d=4 * hd, n_heads=4, n_layers=1, l_switch=0,
                         requests=[(0, 300, 50), (0, 77, 3), (1, 129, 1), (2, 1, 5), (3, 64, 44)])
    inp = W.make_inputs(w, 51, ln_affine=True)
    t = R.to_device(inp, cuda)
    _, y = R.rank_request(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"], t["reqs"],
                          t["z"], t["dec"], t["rope_base"])
    f, s = R.score_head(t["z"], y, t["score"])
    torch.cuda.synchronize()
    _, yr = O.rank_request(inp)
    fr, sr = O.score_head(inp["z"], yr, inp["score"])
    assert_parity(f.cpu().numpy(), fr, dtype, "f")
    assert_parity(s.cpu().numpy(), sr, dtype, "score")


@pytest.mark.parametrize("cfg", [1, 4])
def test_score_head_full_size_sampled_candidates(cuda, cfg):
    """The score head over every candidate of a full workload with a synthetic
    decoder output; a sample of candidates (first, last, random) in the oracle."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    t = R.to_device(inp, cuda)
    rng = np.random.default_rng(cfg)
    y_h = (0.5 * rng.standard_normal(inp["z"].shape)).astype(np.float32)
    f, s = R.score_head(t["z"], torch.from_numpy(y_h).to(cuda), t["score"])
    torch.cuda.synchronize()
    n = w.total_cands
    pick = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 62)]))
    fr, sr = O.score_head(inp["z"][pick], y_h[pick], inp["score"])
    assert_parity(f.cpu().numpy()[pick], fr, "bf16", "f")
    assert_parity(s.cpu().numpy()[pick], sr, "bf16", "score")

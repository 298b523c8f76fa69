"""The causal attention core for training (ULT) on the GPU, through the C
ABI: forward with its log-sum-exp statistics, and the backward, against the
fp64 oracle element by element on ragged histories, and at 16k tokens on
sampled rows and closed-form sums."""
import numpy as np
import pytest
import torch

import shared_prefix_behavior_b200 as R
import workloads as W
from oracle import rest_oracle as O
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def core_case(dtype, hd, lengths, seed, n_heads=4):
    rng = np.random.default_rng(seed)
    T, d = sum(lengths), n_heads * hd
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    arrs = [rng.standard_normal((T, d)).astype(np.float32) for _ in range(4)]
    if dtype == "bf16":
        arrs = [W.round_bf16(a) for a in arrs]
    return arrs, cu, n_heads


def to_dev(arrs, dtype, dev):
    wdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return [torch.from_numpy(np.ascontiguousarray(a)).to(dev, wdt) for a in arrs]


def run_core(arrs, cu, H, dtype, dev):
    """(O, lse, dq, dk, dv) from the GPU; in bf16, O is the pair o + o_lo the
    forward returns (o alone carries bf16's rounding, 1.4e-3 on average)."""
    tq, tk, tv, tg = to_dev(arrs, dtype, dev)
    o, o_lo, lse = R.attn_forward(tq, tk, tv, cu, H)
    dq, dk, dv = R.attn_backward(tq, tk, tv, o, o_lo, lse, tg, cu, H)
    torch.cuda.synchronize()
    full_o = o.float() + (o_lo.float() if o_lo is not None else 0.0)
    return [x.float().cpu().numpy() for x in (full_o, lse, dq, dk, dv)]


@pytest.mark.parametrize("dtype,hd", [("f32", 16), ("f32", 32), ("f32", 64), ("bf16", 16), ("bf16", 32),
                                      ("bf16", 64)])
def test_attention_core_small_ragged(cuda, dtype, hd):
    (q, k, v, d_o), cu, H = core_case(dtype, hd, (300, 129, 1, 64, 255), 71)
    o, lse, dq, dk, dv = run_core([q, k, v, d_o], cu, H, dtype, cuda)
    O_ref, lse_ref = O.attention_core(q, k, v, cu, H)
    assert_parity(o, O_ref, dtype, "O")
    assert np.max(np.abs(lse - lse_ref)) <= 1e-4
    for got, ref, name in zip((dq, dk, dv), O.attention_core_backward(q, k, v, cu, H, d_o), ("dq", "dk", "dv")):
        assert_parity(got, ref, dtype, name)


@pytest.mark.parametrize("hd", [32, 64])
def test_attention_core_row_max_growth(cuda, hd):
    """Keys that grow with their position (x (1 + position // 128)): every
    causal row's running max rises block by block past the kernel's 2^8
    threshold, so the forward rescales the accumulated output in TMEM."""
    (q, k, v, _), cu, H = core_case("bf16", hd, (700, 300), 74)
    for u in range(len(cu) - 1):
        pos = np.arange(cu[u + 1] - cu[u])
        k[cu[u]:cu[u + 1]] = W.round_bf16(k[cu[u]:cu[u + 1]] * (1 + pos // 128)[:, None])
    tq, tk, tv = to_dev([q, k, v], "bf16", cuda)
    o, o_lo, lse = R.attn_forward(tq, tk, tv, cu, H)
    torch.cuda.synchronize()
    O_ref, lse_ref = O.attention_core(q, k, v, cu, H)
    assert_parity((o.float() + o_lo.float()).cpu().numpy(), O_ref, "bf16", "O")
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= 1e-3 * np.max(np.abs(lse_ref))


def test_ult_union_gradients_equal_per_sample_sums_on_gpu(cuda):
    """Samples of one user ending at rows 100, 257 and 400, encoded once as
    their union (one call) and each alone on its prefix (three calls)."""
    (q, k, v, _), cu, H = core_case("bf16", 32, (400,), 72)
    rng = np.random.default_rng(73)
    cuts = [100, 257, 400]
    d_os = []
    for c in cuts:
        g = np.zeros_like(q)
        g[:c] = W.round_bf16(rng.standard_normal((c, q.shape[1])))
        d_os.append(g)
    d_o = W.round_bf16(sum(d_os))      # the union's dO, as the GPU receives it
    union = run_core([q, k, v, d_o], cu, H, "bf16", cuda)[2:]
    alone = [np.zeros_like(q) for _ in range(3)]
    for c, g in zip(cuts, d_os):
        parts = run_core([q[:c], k[:c], v[:c], g[:c]], np.array([0, c], dtype=np.int32), H, "bf16", cuda)[2:]
        for acc, p_ in zip(alone, parts):
            acc[:c] += p_
    ref = O.attention_core_backward(q, k, v, cu, H, d_o)
    for u, a, r, name in zip(union, alone, ref, ("dq", "dk", "dv")):
        assert_parity(u, r, "bf16", name + " (union)")
        # the per-sample sums see each sample's dO rounded on its own
        assert np.abs(u - a).max() <= 1e-2 * np.abs(r).max(), name


def test_attention_core_16k_sampled_rows_and_column_sums(cuda):
    """Two 16384-token histories, d 512, 8 heads of 64 (the long-history
    workload's shape): dq on sampled rows in the oracle row by row; per user
    and head the values' gradients sum to the sum of dO and the keys'
    gradients to zero."""
    (q, k, v, d_o), cu, H = core_case("bf16", 64, (16384, 16384), 74, n_heads=8)
    o, lse, dq, dk, dv = run_core([q, k, v, d_o], cu, H, "bf16", cuda)
    rng = np.random.default_rng(75)
    rows = sorted(set([0, 1, 127, 128, 16383, 16384, 32767] + list(rng.integers(0, 32768, 6))))
    assert_parity(dq[rows], O.attention_core_dq_rows(q, k, v, cu, H, d_o, rows), "bf16", "dq rows")
    for u in range(2):
        s, e = cu[u], cu[u + 1]
        want = d_o[s:e].astype(np.float64).sum(axis=0)
        assert np.abs(dv[s:e].astype(np.float64).sum(axis=0) - want).max() <= 1e-3 * np.abs(d_o[s:e]).sum(axis=0).max()
        assert np.abs(dk[s:e].astype(np.float64).sum(axis=0)).max() <= 1e-3 * np.abs(dk[s:e]).sum(axis=0).max()

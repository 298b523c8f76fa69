"""Append-only encoder cache on the GPU (through the C ABI).

A history is encoded in two appends (its first tokens into an empty cache,
then the rest against the cached keys and values) and compared with the fp64
oracle's append (rows of the full-history encoder), and, at full size, bit
for bit with the GPU's own encoder run over the whole history: every step
acts per row or per key block in the same order either way.
"""
import numpy as np
import pytest
import torch

import shared_prefix_behavior_b200 as R
import workloads as W
from oracle import rest_oracle as O
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def split_rows(inp, lo, hi):
    """Tokens lo[u] .. hi[u]-1 of every user, packed, in the encoder's input form."""
    cu = inp["cu_seqlens"]
    n = len(cu) - 1
    rows = [np.arange(cu[u] + lo[u], cu[u] + hi[u]) for u in range(n)]
    rows = np.concatenate(rows).astype(np.int64) if n else np.zeros(0, np.int64)
    cu2 = np.zeros(n + 1, dtype=np.int32)
    cu2[1:] = np.cumsum([hi[u] - lo[u] for u in range(n)])
    return rows, cu2


def append_in_two(inp, cut, dev, slack=37):
    """Encode each user's first cut[u] tokens into an empty cache, then the
    rest. Returns (H of the first part, H of the rest, the cache)."""
    t = R.to_device(inp, dev)
    cu = inp["cu_seqlens"]
    L = np.diff(cu)
    wdt = t["x"].dtype
    cache = R.KVCache(L + slack, len(t["layers"]), t["x"].shape[1], wdt, dev)
    out = []
    for lo, hi in ((np.zeros_like(L), np.asarray(cut)), (np.asarray(cut), L)):
        rows, cu2 = split_rows(inp, lo, hi)
        ri = torch.from_numpy(rows).to(dev)
        H = R.encoder_append(t["x"][ri].contiguous(), t["ts"][ri].contiguous(), cu2, t["taus"], t["layers"],
                             t["l_switch"], cache, rope_base=t["rope_base"], ts_host=inp["ts"][rows])
        out.append(H)
    torch.cuda.synchronize()
    return out[0], out[1], cache


# The cache arrays are intermediate activations stored in the call's dtype: in
# bf16 a cached key is bf16(fp32 product of a bf16-rounded input row). Each of
# the two roundings has a mean relative error of about 2^-9 / ln 2 / 2 ~ 1.4e-3
# (measured alone: 1.41e-3 where the input row is exact), so the bar for these
# arrays is twice one rounding's bound, 2 * 2^-9 ~ 3.9e-3, on the mean relative
# error, with the output bar on the largest error. The outputs (H) keep the
# output bar.
CACHE_BF16_MEAN_REL = 2.0 * 2.0 ** -9


def assert_cache_parity(got, ref, dtype, what):
    if dtype == "f32":
        return assert_parity(got, ref, dtype, what)
    diff = np.abs(np.asarray(got, dtype=np.float64) - ref)
    assert np.all(np.isfinite(got)), what
    assert diff.max() <= 1e-2 * np.abs(ref).max(), f"{what}: {diff.max()}"
    mean_rel = diff.sum() / np.abs(ref).sum()
    assert mean_rel <= CACHE_BF16_MEAN_REL, f"{what}: mean_rel {mean_rel}"


def cache_rows(cache, cut, hi):
    """Cache rows of positions cut[u] .. hi[u]-1 of every user, packed."""
    return np.concatenate([np.arange(cache.cu_cap[u] + cut[u], cache.cu_cap[u] + hi[u])
                           for u in range(cache.n_users)]).astype(np.int64)


@pytest.mark.parametrize("dtype,hd,n_layers,l_switch", [("f32", 16, 2, 1), ("f32", 32, 1, 0),
                                                         ("bf16", 32, 2, 1), ("bf16", 64, 2, 0)])
def test_append_matches_oracle_small_ragged(cuda, dtype, hd, n_layers, l_switch):
    lengths = (300, 129, 1, 64, 255)
    cut = [200, 0, 1, 63, 130]       # cached before the append: mid-tile, empty, whole user, ...
    w = W.small_workload(dtype, lengths=lengths, d=4 * hd, n_heads=4, n_layers=n_layers, l_switch=l_switch)
    inp = W.make_inputs(w, 51, ln_affine=True)
    H_pre, H_new, cache = append_in_two(inp, cut, cuda)
    Hr, kvr, cu_new = O.encoder_append(inp, cut)
    assert_parity(H_new.float().cpu().numpy(), Hr, dtype, "H of the appended rows")
    pre_rows, _ = split_rows(inp, [0] * 5, cut)
    assert_parity(H_pre.float().cpu().numpy(), O.encoder(inp)[pre_rows], dtype, "H of the first append")
    # the cache holds every layer's R k and V' of the appended tokens (and their H)
    rows = torch.from_numpy(cache_rows(cache, cut, np.diff(inp["cu_seqlens"]))).to(cuda)
    assert np.array_equal(cache.h[rows].float().cpu().numpy(), H_new.float().cpu().numpy())
    for l, (kr, vr) in enumerate(kvr):
        assert_cache_parity(cache.k[l][rows].float().cpu().numpy(), kr, dtype, f"cached keys, layer {l}")
        assert_cache_parity(cache.v[l][rows].float().cpu().numpy(), vr, dtype, f"cached values, layer {l}")
    assert list(cache.len) == list(lengths)


@pytest.mark.parametrize("cfg,n_new,exact", [(1, 64, True), (3, 256, False), (4, 100, True)])
def test_append_equals_full_encoder_bitwise(cuda, cfg, n_new, exact):
    """Full-size workloads: the history minus its last n_new tokens (all of a
    shorter one) into the cache, then those tokens. The first append (an empty
    cache) equals the encoder over the whole history bit for bit; so do the new
    rows where every (user, head) item runs on one CTA. On the 2 x 16384
    workload the second append has 2 users x 8 heads of items, so each item's
    cached keys are split over several CTAs and the partial results merged,
    which reorders the attention's sums: there the new rows match the full
    encoder within the bf16 output bar."""
    w = W.workload(cfg)
    inp = W.make_inputs(w, 1000 + cfg)
    t = R.to_device(inp, cuda)
    H_full = R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                            rope_base=t["rope_base"])
    L = np.diff(inp["cu_seqlens"])
    cut = np.maximum(L - n_new, 0)
    H_pre, H_new, cache = append_in_two(inp, cut, cuda)
    pre_rows, _ = split_rows(inp, np.zeros_like(L), cut)
    new_rows, _ = split_rows(inp, cut, L)
    assert torch.equal(H_pre, H_full[torch.from_numpy(pre_rows).to(cuda)])
    H_new_full = H_full[torch.from_numpy(new_rows).to(cuda)]
    if exact:
        assert torch.equal(H_new, H_new_full)
        all_rows = torch.from_numpy(cache_rows(cache, np.zeros_like(L), L)).to(cuda)
        assert torch.equal(cache.h[all_rows], H_full)
    else:
        assert_parity(H_new.float().cpu().numpy(), H_new_full.double().cpu().numpy(), "bf16", "H of the appended rows")
        pre_cache = torch.from_numpy(cache_rows(cache, np.zeros_like(L), cut)).to(cuda)
        assert torch.equal(cache.h[pre_cache], H_full[torch.from_numpy(pre_rows).to(cuda)])


@pytest.mark.parametrize("hd", [32, 64])
def test_append_split_keys_matches_oracle(cuda, hd):
    """Few users with long cached prefixes: the tensor-core attention splits
    every item's cached keys over several CTAs and merges the partial results.
    The appended rows and their cached keys and values match the oracle."""
    lengths, cut = (2064, 1500), [2000, 1450]
    w = W.small_workload("bf16", lengths=lengths, d=4 * hd, n_heads=4, n_layers=2, l_switch=1)
    inp = W.make_inputs(w, 54, ln_affine=True)
    H_pre, H_new, cache = append_in_two(inp, cut, cuda)
    Hr, kvr, _ = O.encoder_append(inp, cut)
    assert_parity(H_new.float().cpu().numpy(), Hr, "bf16", "H of the appended rows")
    rows = torch.from_numpy(cache_rows(cache, cut, np.diff(inp["cu_seqlens"]))).to(cuda)
    for l, (kr, vr) in enumerate(kvr):
        assert_cache_parity(cache.k[l][rows].float().cpu().numpy(), kr, "bf16", f"cached keys, layer {l}")
        assert_cache_parity(cache.v[l][rows].float().cpu().numpy(), vr, "bf16", f"cached values, layer {l}")


def test_decoder_reads_the_cached_memory(cuda):
    """rest_cross_decode on the cache's H regions (cu_cap as the batch) gives
    what it gives on the packed H of a full encode."""
    w = W.small_workload("bf16", lengths=(300, 129), d=128, n_heads=4, n_layers=2, l_switch=1,
                         requests=[(0, 300, 20), (0, 57, 4), (1, 129, 9)])
    inp = W.make_inputs(w, 52)
    t = R.to_device(inp, cuda)
    H_full = R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                            rope_base=t["rope_base"])
    _, _, cache = append_in_two(inp, [250, 100], cuda)
    y_full = R.cross_decode(H_full, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    cu_cap, lens = cache.batch()
    assert all(int(c) <= int(lens[int(u)]) for u, c in zip(t["reqs"][0], t["reqs"][1]))
    y_cache = R.cross_decode(cache.h, cu_cap, t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    assert torch.equal(y_full, y_cache)


def test_append_before_the_last_cached_time_sets_the_device_status(cuda):
    w = W.small_workload("bf16", lengths=(40, 20), d=64, n_heads=2, n_layers=1, l_switch=0)
    inp = W.make_inputs(w, 53)
    t = R.to_device(inp, cuda)
    cache = R.KVCache([64, 64], 1, 64, torch.bfloat16, cuda)
    R.encoder_append(t["x"], t["ts"], inp["cu_seqlens"], t["taus"], t["layers"], 0, cache, ts_host=inp["ts"])
    late = t["ts"][:2].clone() - 10**6    # earlier than user 0's cached tokens
    with pytest.raises(R.RestError) as e:
        R.encoder_append(t["x"][:2].contiguous(), late, [0, 2, 2], t["taus"], t["layers"], 0, cache, advance=False)
    assert e.value.status == 2

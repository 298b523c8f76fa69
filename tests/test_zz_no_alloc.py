"""rest_cross_decode_static_ws: the decoder for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plain-C host program with no device
allocator of its own, or a serving process that handed all device memory to
a fixed arena at start-up). For them the library keeps the decoder's scratch
in a fixed array of its own device image. These tests call that entry point
through the C ABI and check that it gives the same scores as rest_cross_decode
with a caller workspace, on two calls in a row (the second on a different
batch, so stale contents of the shared array would show), and that a batch
too large for the array is refused. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import shared_prefix_behavior_b200 as R
import workloads as W
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def _case(lengths, d, n_heads, requests, seed, dev):
    w = W.small_workload("bf16", lengths=lengths, d=d, n_heads=n_heads, requests=requests)
    inp = W.make_inputs(w, seed)
    t = R.to_device(inp, dev)
    Hd = torch.from_numpy(W.make_memory(w, seed)).to(dev, torch.bfloat16)
    return t, Hd


def _both(t, Hd):
    args = (Hd, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    with_ws = R.cross_decode(*args)
    static = R.cross_decode_static_ws(*args)
    torch.cuda.synchronize()
    return static.cpu().numpy(), with_ws.cpu().numpy()


def test_static_ws_decoder_matches_workspace_decoder_twice(cuda):
    t1, H1 = _case((700, 129, 3), 256, 8, [(0, 700, 60), (0, 1, 2), (1, 129, 45), (2, 2, 7)], 51, cuda)
    t2, H2 = _case((300, 40), 128, 4, [(1, 40, 9), (0, 300, 31), (0, 17, 5)], 52, cuda)
    for t, Hd in ((t1, H1), (t2, H2)):
        got, ref = _both(t, Hd)
        assert got.shape == ref.shape
        assert_parity(got, ref, "bf16", "static scratch vs workspace")


def test_static_ws_decoder_refuses_a_batch_beyond_its_array(cuda):
    d, K = 512, 3
    n = R.STATIC_WS_BYTES // (12 * d * K) + 8  # q, g, o rows beyond the array
    w = W.small_workload("bf16", lengths=(64,), d=d, n_heads=8, requests=[(0, 64, n)])
    inp = W.make_inputs(w, 53)
    t = R.to_device(inp, cuda)
    Hd = torch.from_numpy(W.make_memory(w, 53)).to(cuda, torch.bfloat16)
    with pytest.raises(R.RestError) as e:
        R.cross_decode_static_ws(Hd, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    assert e.value.status == 6  # REST_ERR_WORKSPACE

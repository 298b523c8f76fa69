"""rest_cross_decode_static_ws: the decoder for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plain-C host program with no device
allocator of its own, or a serving process that handed all device memory to
a fixed arena at start-up). For them the library keeps the decoder's scratch
in a fixed array of its own device image. These tests call that entry point
through the C ABI and check that it gives the same scores as rest_cross_decode
with a caller workspace, on two calls in a row (the second on a different
batch, so stale contents of the shared array would show), that a batch too
large for the array is refused, that a call leaves torch's allocations and
the device's free memory as they were, and that a call with no candidates
loads the array in a fresh process (the warm-up a caller makes before handing
its device memory to an arena). This file is collected last on purpose.
"""
import os
import subprocess
import sys

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


def test_static_ws_decoder_allocates_nothing(cuda):
    """Given its output and status word, a call changes neither torch's
    allocations nor the device's free memory (after a first call, which
    loads the library's kernels and the array)."""
    t, Hd = _case((700, 129, 3), 256, 8, [(0, 700, 60), (1, 129, 45), (2, 2, 7)], 55, cuda)
    y = torch.empty(t["z"].shape, dtype=torch.float32, device=cuda)
    err = torch.zeros(1, dtype=torch.int32, device=cuda)
    args = (Hd, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"])
    R.cross_decode_static_ws(*args, y_out=y, err=err)
    torch.cuda.synchronize()
    first = y.clone()
    allocated, free = torch.cuda.memory_allocated(cuda), torch.cuda.mem_get_info(cuda)[0]
    for _ in range(2):
        R.cross_decode_static_ws(*args, y_out=y, err=err)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(cuda) == allocated
        assert torch.cuda.mem_get_info(cuda)[0] == free
    assert torch.equal(y, first)


# A fresh interpreter: the decoder with no candidates, then the device's free
# memory before and after it.
_EMPTY_CALL = r"""
import sys
import torch
sys.path.insert(0, sys.argv[1])
import shared_prefix_behavior_b200 as R
import workloads as W
dev = torch.device("cuda:0")
w = W.small_workload("bf16", lengths=(64,), d=128, n_heads=4, requests=[(0, 64, 0)])
t = R.to_device(W.make_inputs(w, 54), dev)
Hd = torch.zeros((64, 128), dtype=torch.bfloat16, device=dev)
y = torch.empty((0, 3, 128), dtype=torch.float32, device=dev)
err = torch.zeros(1, dtype=torch.int32, device=dev)
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info(dev)[0]
R.cross_decode_static_ws(Hd, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"], y_out=y,
                         err=err)
torch.cuda.synchronize()
print("DROP", free0 - torch.cuda.mem_get_info(dev)[0])
"""


def test_static_ws_empty_call_loads_the_array(cuda):
    """In a fresh process, a call with no candidates loads the scratch array
    on the device (its free memory drops by at least the array's size), so a
    caller can reserve it before giving the rest of the memory to an arena."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _EMPTY_CALL, root], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    drop = int(r.stdout.split("DROP")[-1].split()[0])
    assert drop >= R.STATIC_WS_BYTES, (drop, R.STATIC_WS_BYTES)

"""Failure detection on the GPU without a fault: the library's bounded wait
runs out on a barrier nothing completes, the device reports
REST_ERR_TIMEOUT, every CTA stops, and the context keeps working."""
import time

import numpy as np
import pytest
import torch

import shared_prefix_behavior_b200 as R
import workloads as W
from oracle import rest_oracle as O
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_recovers(cuda):
    t0 = time.perf_counter()
    # CTA 0 gives up after 2e7 cycles (about 10 ms); the 147 others wait with the
    # library's one-second bound and must stop on seeing CTA 0's error word
    status = R.selftest_wait_timeout(cuda, n_ctas=148, limit_cycles=20_000_000)
    elapsed = time.perf_counter() - t0
    assert status == 5  # REST_ERR_TIMEOUT
    assert elapsed < 0.9, f"the other CTAs did not stop on the error word ({elapsed:.2f} s)"
    # the context is usable: a normal call afterwards succeeds and is correct
    w = W.small_workload("bf16", lengths=(200, 37), d=128, n_heads=4, n_layers=1, l_switch=0,
                         requests=[(0, 200, 5), (1, 37, 3)])
    inp = W.make_inputs(w, 81)
    t = R.to_device(inp, cuda)
    H = R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                       rope_base=t["rope_base"])
    assert_parity(H.float().cpu().numpy(), O.encoder(inp), "bf16", "H after a timeout")

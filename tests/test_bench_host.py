"""Host-side pieces of bench.py that need no GPU: the digest that ties a
recorded ncu traffic figure to the kernel code it was taken on, and the
no-sharing inputs (every candidate its own user with its request's prefix)
used by the sharing comparison and the oracle's no-sharing timing."""
import os
import shutil

import numpy as np

import bench
import workloads as W


def _copy_sources(tmp_path):
    d = tmp_path / "csrc"
    d.mkdir()
    for f in bench.KERNEL_SOURCES["attn"]:
        shutil.copy(os.path.join(bench.CSRC, f), d / f)
    return d


def test_digest_ignores_comments_and_blank_space_but_not_code(tmp_path, monkeypatch):
    d = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "CSRC", str(d))
    base = bench.source_digest("attn")
    f = d / bench.KERNEL_SOURCES["attn"][0]
    text = f.read_text()
    f.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.source_digest("attn") == base
    f.write_text(text + "\nconstexpr int an_extra_constant = 64;\n")
    assert bench.source_digest("attn") != base


def test_traffic_is_reported_only_for_the_code_it_was_taken_on(tmp_path, monkeypatch):
    key = next(iter(bench.TRAFFIC))
    nbytes, kind, digest, _ = bench.TRAFFIC[key]
    d = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "CSRC", str(d))
    if bench.source_digest(kind) == digest:
        assert bench.traffic_for(*key)[0] == nbytes
    f = d / bench.KERNEL_SOURCES[kind][0]
    f.write_text(f.read_text() + "\nint an_extra_symbol;\n")
    value, note = bench.traffic_for(*key)
    assert value is None and "changed" in note
    assert bench.traffic_for("enc_attn", "no such workload")[0] is None


def test_no_sharing_inputs_give_each_candidate_its_request_prefix():
    w = W.small_workload("bf16", lengths=(40, 25), d=32, n_heads=2, n_layers=1, l_switch=0,
                         requests=[(0, 40, 3), (0, 11, 2), (1, 25, 4)])
    inp = W.make_inputs(w, 7)
    ns, rows = bench.no_sharing_inputs(inp, [0, 1])
    cuts = [40] * 3 + [11] * 2 + [25] * 4
    assert list(np.diff(ns["cu_seqlens"])) == cuts
    assert list(ns["req_cutoff"]) == cuts and list(ns["req_user"]) == list(range(9))
    assert list(ns["cu_cands"]) == list(range(10))
    # each candidate's history is its user's first `cutoff` rows, and its z row its own
    starts = [0, 0, 0, 0, 0, 40, 40, 40, 40]
    expect = np.concatenate([np.arange(s, s + c) for s, c in zip(starts, cuts)])
    assert np.array_equal(rows, expect)
    assert np.array_equal(ns["x"], inp["x"][expect]) and np.array_equal(ns["ts"], inp["ts"][expect])
    assert np.array_equal(ns["z"], inp["z"])
    # a cap keeps the first candidates of the listed users only
    ns2, _ = bench.no_sharing_inputs(inp, [1], max_cands=2)
    assert list(np.diff(ns2["cu_seqlens"])) == [25, 25]
    assert np.array_equal(ns2["z"], inp["z"][5:7])

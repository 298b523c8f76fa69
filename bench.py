"""Benchmark of the ReST encode-once / decode-many ranking forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl reference]

One step = one ``rank_request`` plus ``score_head`` over a batch of the
named workload (default: the ragged shared-prefix batch, 64 users with
log-normal history lengths in [128, 16384] (173,846 tokens), d=256, 8 heads
of 32 (4 RoPE + 4 RoTE), 1 encoder layer, 1-4 request cutoffs per user with
64-1024 candidates x 3 query tokens each, bf16): the encoder over every
history, then every candidate of every request against its user's encoder
output truncated at the request's cutoff, then the candidate scores. Multi-GPU runs shard users across ranks (weak scaling: every
rank runs its own batch), with no collective on the data path.

Rank 0 prints one JSON line. ``value`` is candidate scores/s over all ranks
with inputs resident in HBM, timed with CUDA events (max over ranks);
``e2e`` is the same metric with the step's inputs copied from pinned host
memory and the scores copied back inside the timed region. ``roofline`` is
for the kernel with the largest share of device time, from a second pass of
the same steps with per-kernel CUDA events. ``cpu_baseline`` times the fp64
oracle on the host cores on a bounded sample. ``--impl reference`` times that
oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import dataclasses
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "candidate scores/s & encoder tokens/s on 1 B200; % bf16 tensor peak / HBM roofline"
UNIT = "candidate scores/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TENSOR_KERNELS = ("gemm", "enc_attn", "dec_attn")
# A GPU-side pause before each separately timed call (after its L2 flush): the
# host enqueues the call's launches meanwhile, so the call's events measure its
# kernels, not the host's planning and launch latency (reported separately).
PAD_CYCLES = 2_000_000  # about 1 ms of SM clock

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# workload's dominant kernel from one ncu capture, with a digest of the kernel
# sources it was taken on: reported only while those sources are unchanged.
CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "shared_prefix_behavior_b200", "csrc")
KERNEL_SOURCES = {
    "attn": ("sm100_attn.cu", "sm100_common.cuh", "common.cuh", "kernels.h"),
    "gemm": ("sm100_gemm.cu", "sm100_common.cuh", "common.cuh", "kernels.h"),
}
TRAFFIC = {  # (kernel, workload): (bytes per launch, sources, digest, summary)
    ("dec_attn", "bf16-ragged64-d256"): (522458880, "attn", "6fdb154546b94f5a",
                                         "profiles/attn_tc_kernel_bf16-ragged64-d256.md"),
    ("enc_attn", "bf16-ragged64-d256"): (905321472, "attn", "6fdb154546b94f5a",
                                         "profiles/attn_tc_kernel_bf16-ragged64-d256.md"),
}


def source_digest(kind: str) -> str:
    """Digest of the kernel's code: its sources with comments and blank space
    removed, so that a comment edit keeps a capture's figures."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """(bytes per launch or None, note)."""
    t = TRAFFIC.get((kernel, workload))
    if t is None:
        return None, "no ncu capture of this kernel on this workload"
    nbytes, kind, digest, src = t
    try:
        if source_digest(kind) != digest:
            return None, "kernel sources changed since the capture in " + src
    except OSError:
        return None, "kernel sources not found"
    return nbytes, "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch (" + src + ")"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ablation", action="store_true",
                    help="also time the encoder under the gated-attention and RoTE ablation variants")
    ap.add_argument("--sharing", action="store_true",
                    help="also run the no-sharing variant (every candidate re-encodes its own history)")
    ap.add_argument("--core-only", action="store_true",
                    help="the step, its per-kernel pass, e2e and the two halves alone; no append, training or "
                         "CPU baseline (for profiler runs)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w: W.Workload, n: int, ws_bytes: int | None = None) -> dict:
    n_rope = int(np.sum(w.taus == 0))
    return {
        "workload": w.name,
        "users_per_gpu": w.n_users,
        "history_len": w.lengths[0] if len(set(w.lengths)) == 1 else "ragged",
        "tokens_per_gpu": w.total_tokens,
        "d": w.d,
        "heads": f"{w.n_heads}x{w.head_dim} ({n_rope} RoPE + {w.n_heads - n_rope} RoTE)",
        "encoder_layers": w.n_layers,
        "candidates_per_gpu": w.total_cands,
        "query_tokens": w.K,
        "parallelism": f"dp{n}: users LPT-sharded across ranks, no collective",
        "l2": ("not flushed: one step writes and reads its workspace of activations "
               + (f"({ws_bytes / 2**30:.2f} GiB) " if ws_bytes else "")
               + "plus the inputs and H, well above the 126 MB L2"),
    }


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons during the timed region: NVML read every
    10 ms from a host thread (read-only queries), or nvidia-smi every 200 ms when
    NVML is not available. Only samples taken after mark() count."""

    REASONS = ((0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"))

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.t_mark = 0.0
        self.source = None

    def mark(self):
        """Call when the timed region starts: earlier samples are not counted."""
        self.t_mark = time.time()

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, h):
        import pynvml
        while not self.stop.is_set():
            try:
                clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), float(clk), float(mx), int(rs)))
            except Exception:
                pass
            self.stop.wait(0.01)

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        try:
            h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll, args=(h,), daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
        except Exception:
            self.thread = None
            self._smi_start()
        return self

    def _smi_start(self):
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=timestamp,clocks.sm,"
                                          "clocks.max.sm,clocks_event_reasons.active", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 200 ms"
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def __exit__(self, *a):
        self.t_end = time.time()
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)
        elif getattr(self, "proc", None) is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    try:
                        whole, _, frac = parts[0].partition(".")
                        ts = time.mktime(time.strptime(whole, "%Y/%m/%d %H:%M:%S")) + float("0." + (frac or "0"))
                        self.samples.append((ts, float(parts[1]), float(parts[2]), int(parts[3], 16)))
                    except (ValueError, IndexError):
                        continue
            os.unlink(self.path)

    def summary(self):
        inside = [s for s in self.samples if self.t_mark <= s[0] <= getattr(self, "t_end", float("inf"))]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = sorted({nm for s in inside for bit, nm in self.REASONS if s[3] & bit})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "sm_mhz_min": min(s[1] for s in inside), "reasons": reasons, "samples": len(inside),
                "source": self.source}


# --------------------------------------------------------------------- the two halves on their own

def tensor_peak(peaks) -> float:
    """The bf16 dense peak for kernels timed here: the burst figure. Every timed
    region of this benchmark lasts milliseconds to tens of milliseconds at the
    full SM clock, not the seconds-long power-capped loop of the sustained one."""
    return float(peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained")))


# Exponentials per SM per clock of the special-function unit (16 per SM, four
# per sub-partition): the floor of a softmax whose every score needs one.
EXP_PER_CLK_SM = 16
N_SMS = 148


def exp_floor_s(n_exp: float, sm_mhz: float) -> float:
    """Seconds the exponentials alone take on the special-function units."""
    return n_exp / (EXP_PER_CLK_SM * N_SMS * sm_mhz * 1e6)


def peaks_for_parts():
    peaks, src = load_peaks()
    return tensor_peak(peaks), float(peaks["hbm_gbs"]), src


def component_timings(args, w, t, H, Y, ws, dev, peaks):
    """Encoder alone (rest_encoder_attn) and the decoder alone (rest_cross_decode),
    the latter with L2 flushed before every call (a 256 MB write), so that the
    shared prefix H is read from HBM as it would be when it is not resident."""
    import torch
    import shared_prefix_behavior_b200 as R
    t_peak, hbm_peak, src = peaks
    n = max(3, min(args.steps, 50))

    def enc():
        R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                       rope_base=t["rope_base"], h_out=H, ws=ws, check=False)

    def dec():
        R.cross_decode(H, t["cu_seqlens"], t["taus"], t["reqs"], t["z"], t["dec"], t["rope_base"], y_out=Y, ws=ws,
                       check=False)

    for _ in range(3):
        enc()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        enc()
    b.record()
    torch.cuda.synchronize()
    enc_ms = a.elapsed_time(b) / n
    enc_part = {"tokens_per_s": w.total_tokens / (enc_ms * 1e-3), "ms": enc_ms, "calls": n, "l2": "not flushed"}

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for _ in range(3):
        dec()
    R.profile_begin()
    for i in range(n):
        flush.fill_(i & 0xff)
        torch.cuda._sleep(PAD_CYCLES)
        evs[i][0].record()
        dec()
        evs[i][1].record()
    stats = R.profile_end()
    torch.cuda.synchronize()
    dec_ms = sum(x.elapsed_time(y) for x, y in evs) / n
    attn = [s_ for s_ in stats if s_["name"] == "dec_attn"]
    d, K = w.d, w.K
    flops = sum(4.0 * d * K * nr * c for nr, c in zip(w.req_ncand, w.req_cutoff))
    # algorithmic bytes of the attention: every H prefix once per request, q and g in (fp32), o * g out (4 B)
    nk = K * w.total_cands
    h_bytes = sum(2.0 * c * d for c in w.req_cutoff)
    abytes = h_bytes + 12.0 * nk * d
    dec_part = {"candidate_scores_per_s": w.total_cands / (dec_ms * 1e-3), "ms": dec_ms, "calls": n,
                "l2": "flushed before every call (256 MB write)", "pad": "1 ms GPU pause before each timed call"}
    if attn:
        t_attn = attn[0]["ms"] / n * 1e-3  # seconds of decoder attention per call (all its launches)
        t_roof = max(flops / (t_peak * 1e12), abytes / (hbm_peak * 1e9))
        dec_part["attention"] = {
            "ms": t_attn * 1e3, "tflops": flops / t_attn / 1e12, "algorithmic_flops": flops,
            "algorithmic_bytes": abytes, "roofline_ms": t_roof * 1e3, "roofline_frac": t_roof / t_attn,
            "roofline": f"max(FLOPs / burst bf16 peak, bytes / HBM copy bandwidth), measured peaks ({src})",
            "exponentials": flops / (4.0 * w.head_dim)}
    return {"encoder_only": enc_part, "decoder_only": dec_part}


def no_sharing_inputs(inp: dict, users, max_cands=None):
    """The candidates of the given users without the shared prefix: each one a
    user of its own whose history is its request's prefix (at most max_cands
    of them). Returns (inputs, the source rows of the re-encoded tokens)."""
    cu = np.asarray(inp["cu_seqlens"])
    ru, rc, cc = (np.asarray(inp[k]) for k in ("req_user", "req_cutoff", "cu_cands"))
    rows, z_rows, lens = [], [], []
    for r in range(len(ru)):
        if ru[r] not in users:
            continue
        s0 = int(cu[ru[r]])
        for c in range(int(cc[r]), int(cc[r + 1])):
            if max_cands is not None and len(lens) >= max_cands:
                break
            rows.append(np.arange(s0, s0 + int(rc[r])))
            z_rows.append(c)
            lens.append(int(rc[r]))
    rows = np.concatenate(rows)
    n = len(lens)
    ns = dict(inp, x=inp["x"][rows], ts=inp["ts"][rows],
              cu_seqlens=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32),
              req_user=np.arange(n, dtype=np.int32), req_cutoff=np.asarray(lens, dtype=np.int32),
              cu_cands=np.arange(n + 1, dtype=np.int32), z=inp["z"][np.asarray(z_rows)])
    return ns, rows


def sharing_comparison(w, inp, dev, ms_shared):
    """The same candidates without the shared prefix: every candidate becomes a
    user of its own whose history is its request's prefix, encoded and decoded
    alone (what the decoder's sharing avoids). Run on whole users of the batch,
    as many as keep the re-encoded tokens near 1M, and compared per candidate."""
    import torch
    import shared_prefix_behavior_b200 as R
    cu = np.asarray(inp["cu_seqlens"])
    ru, rc, cc = (np.asarray(inp[k]) for k in ("req_user", "req_cutoff", "cu_cands"))
    users, tok = [], 0
    for u in range(len(cu) - 1):
        need = sum(int(rc[r]) * int(cc[r + 1] - cc[r]) for r in range(len(ru)) if ru[r] == u)
        if users and tok + need > (1 << 20):
            break
        users.append(u)
        tok += need
    ns, rows = no_sharing_inputs(inp, users)
    n = len(ns["req_user"])
    t = R.to_device(ns, dev)
    args_rank = (t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"], t["reqs"], t["z"],
                 t["dec"], t["rope_base"])
    R.rank_request(*args_rank, check=True)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(3):
        R.rank_request(*args_rank, check=False)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / 3
    shared_per_cand = ms_shared / w.total_cands
    alone_per_cand = ms / n
    return {"users": len(users), "candidates": n, "reencoded_tokens": int(len(rows)), "ms": ms,
            "ms_per_candidate_alone": alone_per_cand, "ms_per_candidate_shared": shared_per_cand,
            "speedup_of_sharing": alone_per_cand / shared_per_cand}


def append_comparison(w, inp, dev, full_ms, n_new=64):
    """Append-only encoding: every user's history minus its last n_new tokens
    sits in the key/value cache, and the call encodes those n_new tokens
    against it; compared with re-encoding the whole history (the encoder-only
    time above). L2 is flushed (a 256 MB write) before every timed call, so
    the cached keys and values come from HBM."""
    import torch
    import shared_prefix_behavior_b200 as R
    t = R.to_device(inp, dev)
    cu = np.asarray(inp["cu_seqlens"])
    L = np.diff(cu)
    cut = np.maximum(L - n_new, 0)
    cache = R.KVCache(L, len(t["layers"]), w.d, t["x"].dtype, dev, keep_h=True)

    def part(lo, hi):
        rows = np.concatenate([np.arange(cu[u] + lo[u], cu[u] + hi[u]) for u in range(len(L))]).astype(np.int64)
        cu2 = np.zeros(len(L) + 1, dtype=np.int32)
        cu2[1:] = np.cumsum(hi - lo)
        ri = torch.from_numpy(rows).to(dev)
        return t["x"][ri].contiguous(), t["ts"][ri].contiguous(), cu2, inp["ts"][rows]

    xp, tp, cup, tsp = part(np.zeros_like(L), cut)
    R.encoder_append(xp, tp, cup, t["taus"], t["layers"], t["l_switch"], cache, rope_base=t["rope_base"],
                     ts_host=tsp)
    xn, tn, cun, _ = part(cut, L)
    ws = torch.empty(max(256, R.append_workspace_size(R.REST_BF16 if w.dtype == "bf16" else R.REST_F32, t["taus"],
                                                      w.d, cun, t["layers"], t["rope_base"])),
                     dtype=torch.uint8, device=dev)
    h_out = torch.empty_like(xn)

    def app(check=False):
        R.encoder_append(xn, tn, cun, t["taus"], t["layers"], t["l_switch"], cache, rope_base=t["rope_base"],
                         advance=False, h_out=h_out, ws=ws, check=check)

    app(check=True)
    for _ in range(3):
        app()
    torch.cuda.synchronize()
    n = 20
    # host time to enqueue one call (the GPU is kept busy by flushes meanwhile)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for i in range(8):
        flush.fill_(i & 0xff)
    t_host = time.perf_counter()
    for _ in range(n):
        app()
    host_ms = (time.perf_counter() - t_host) * 1e3 / n
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush.fill_(i & 0xff)
        torch.cuda._sleep(PAD_CYCLES)
        evs[i][0].record()
        app()
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = sum(x.elapsed_time(y) for x, y in evs) / n
    # per-kernel split (a separate pass: every launch bracketed by its own events)
    R.profile_begin()
    for i in range(n):
        flush.fill_(i & 0xff)
        app()
    stats = R.profile_end()
    torch.cuda.synchronize()
    new = int((L - cut).sum())
    out = {"cached_tokens": int(cut.sum()), "new_tokens": new, "new_per_user": n_new, "ms": ms,
           "new_tokens_per_s": new / (ms * 1e-3), "full_reencode_ms": full_ms,
           "speedup_vs_reencode": full_ms / ms, "l2": "flushed before every call (256 MB write)", "pad": "1 ms GPU pause before each timed call",
           "launches_per_call": sum(s_["launches"] for s_ in stats) / n, "host_enqueue_ms": host_ms,
           "kernels_ms_per_call": {s_["name"]: s_["ms"] / n for s_ in sorted(stats, key=lambda x: -x["ms"])}}
    attn = [s_ for s_ in stats if s_["name"] == "enc_attn"]
    if attn:
        # a few new query rows against every cached key: the cached K and V' must cross
        # HBM once per layer, which bounds the kernel (far below the ridge point)
        sec = attn[0]["ms"] * 1e-3
        peaks, src = load_peaks()
        t_roof = max(attn[0]["flops"] / (tensor_peak(peaks) * 1e12),
                     attn[0]["bytes"] / (float(peaks["hbm_gbs"]) * 1e9))
        out["attention"] = {"ms": attn[0]["ms"] / n, "tflops": attn[0]["flops"] / sec / 1e12,
                            "gbs": attn[0]["bytes"] / sec / 1e9, "roofline_frac": t_roof / sec,
                            "roofline": f"max(FLOPs / burst bf16 peak, bytes / HBM copy bandwidth) ({src})"}
    return out


def ablation_comparison(w, dev, n=20):
    """The encoder (rest_encoder_attn) of the same workload under the page's
    ablation variants: the gates of the attention sublayer (value + output,
    the DGA layer; output only; Q, K, V and output) and RoTE with a single
    1-second granularity on every time head. Each variant has its own seeded
    weights; only its cost is compared here (parity is in the tests). FLOPs
    are the encoder's algorithmic FLOPs, projections included."""
    import torch
    import shared_prefix_behavior_b200 as R
    out = {}
    base_ms = None
    for name, wv in (("dga_value_output", w), ("output_gate_only", dataclasses.replace(w, gates="o")),
                     ("qkv_output_gates", dataclasses.replace(w, gates="qkvo")),
                     ("rote_single_1s", dataclasses.replace(w, taus=np.where(w.taus > 0, 1, 0).astype(np.int64)))):
        inp = W.make_inputs(wv, 1000 + 17)
        t = R.to_device(inp, dev)
        H = torch.empty_like(t["x"])
        ws = torch.empty(R.workspace_size(R.REST_BF16 if wv.dtype == "bf16" else R.REST_F32, t["taus"], wv.d,
                                          t["cu_seqlens"], t["layers"], rope_base=t["rope_base"]),
                         dtype=torch.uint8, device=dev)

        def enc(check=False):
            R.encoder_attn(t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"],
                           rope_base=t["rope_base"], h_out=H, ws=ws, check=check)

        enc(check=True)
        for _ in range(3):
            enc()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            enc()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / n
        nb = {"vo": 5, "o": 4, "qkvo": 7}[wv.gates]
        T, d = wv.total_tokens, wv.d
        pairs = sum(L * (L + 1) / 2 for L in wv.lengths)
        flops = wv.n_layers * (2.0 * T * d * nb * d + 2.0 * T * d * d + 6.0 * T * d * wv.d_ff + 4.0 * d * pairs)
        if base_ms is None:
            base_ms, base_flops = ms, flops
        out[name] = {"gates": wv.gates, "taus": [int(x) for x in wv.taus], "ms": ms,
                     "tokens_per_s": T / (ms * 1e-3), "time_vs_dga": ms / base_ms, "flops": flops,
                     "flops_vs_dga": flops / base_flops}
    return out


def training_comparison(w, inp, dev, n=10):
    """The attention core a training step runs (ULT, §3.5): rest_attn_forward
    and rest_attn_backward on the workload's histories (seeded bf16 q, k, V'
    and dO stand in for a layer's activations), with L2 flushed before every
    call (a 256 MB write). ULT's comparison: the same core run once per
    request instead, each request a training sample of its own whose history
    is its prefix (what encoding the union history once saves)."""
    import torch
    import shared_prefix_behavior_b200 as R
    H, d = w.n_heads, w.d
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    peaks, src = load_peaks()
    t_peak = tensor_peak(peaks)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + 29)

    def run(cu):
        T = int(cu[-1])
        q, k, v, d_o = (torch.randn((T, d), generator=g, device=dev).to(dt) for _ in range(4))
        ws = torch.empty(R.attn_workspace_size(R.REST_BF16 if dt == torch.bfloat16 else R.REST_F32, H, d // H, cu),
                         dtype=torch.uint8, device=dev)
        o, o_lo, lse = R.attn_forward(q, k, v, cu, H, ws=ws)
        dq, dk, dv = R.attn_backward(q, k, v, o, o_lo, lse, d_o, cu, H, ws=ws)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for i in range(n):
            flush.fill_(i & 0xff)
            torch.cuda._sleep(PAD_CYCLES)
            ev[i][0].record()
            R.attn_forward(q, k, v, cu, H, o=o, o_lo=o_lo, lse=lse, ws=ws, check=False)
            ev[i][1].record()
            torch.cuda._sleep(PAD_CYCLES)  # the backward's inputs stay in L2 from the forward
            ev[i][2].record()
            R.attn_backward(q, k, v, o, o_lo, lse, d_o, cu, H, dq=dq, dk=dk, dv=dv, ws=ws, check=False)
            ev[i][3].record()
        torch.cuda.synchronize()
        fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / n
        bwd = sum(e[2].elapsed_time(e[3]) for e in ev) / n
        pairs = sum(L * (L + 1) / 2 for L in np.diff(cu))
        return fwd, bwd, pairs, T

    cu = np.asarray(inp["cu_seqlens"], dtype=np.int32)
    fwd, bwd, pairs, T = run(cu)
    f_fwd, f_bwd = 4.0 * d * pairs, 10.0 * d * pairs
    out = {"tokens": T, "fwd_ms": fwd, "bwd_ms": bwd,
           "fwd_tflops": f_fwd / fwd / 1e9, "bwd_tflops": f_bwd / bwd / 1e9,
           "fwd_roofline_frac": f_fwd / fwd / 1e9 / t_peak, "bwd_roofline_frac": f_bwd / bwd / 1e9 / t_peak,
           "roofline": f"algorithmic FLOPs (fwd 4 d, bwd 10 d per visible pair) / burst bf16 peak ({src})",
           "l2": "flushed before every call (256 MB write)", "pad": "1 ms GPU pause before each timed call"}
    # ULT: every request's prefix as a sample of its own, packed into one batch
    lens = [int(c) for c in inp["req_cutoff"]]
    cu_s = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s_fwd, s_bwd, s_pairs, s_T = run(cu_s)
    out["ult"] = {"samples": len(lens), "union_tokens": T, "per_sample_tokens": s_T,
                  "per_sample_ms": s_fwd + s_bwd, "union_ms": fwd + bwd,
                  "speedup_of_union": (s_fwd + s_bwd) / (fwd + bwd), "flop_ratio": s_pairs / pairs}
    return out


# --------------------------------------------------------------------- oracle (CPU baseline / reference arm)

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_sample(w: W.Workload, inp: dict, users):
    """Time the fp64 oracle on a subset of users: returns (seconds, candidates, tokens)."""
    from oracle import rest_oracle as O
    sub = W.subset_users(inp, users)
    t0 = time.perf_counter()
    O.rank_request(sub)
    dt = time.perf_counter() - t0
    return dt, int(sub["cu_cands"][-1]), int(sub["cu_seqlens"][-1])


# Users whose fp64 oracle run stays within a few seconds: the CPU samples take
# users of at most this many tokens (a 13k-token user alone takes minutes).
ORACLE_MAX_LEN = 4096


def oracle_users(w: W.Workload):
    """The workload's users in order, without those longer than ORACLE_MAX_LEN
    (all of them when none is short enough)."""
    users = [u for u in range(w.n_users) if w.lengths[u] <= ORACLE_MAX_LEN]
    return users or list(range(w.n_users))


def cpu_baseline(w: W.Workload, inp: dict, budget_s: float) -> dict:
    t_tot, c_tot, tok_tot, users = 0.0, 0, 0, []
    for u in oracle_users(w):
        dt, c, tok = oracle_sample(w, inp, [u])
        t_tot += dt
        c_tot += c
        tok_tot += tok
        users.append(u)
        if t_tot >= budget_s:
            break
    short = all(w.lengths[u] <= ORACLE_MAX_LEN for u in users)
    rule = (f"skipping users of more than {ORACLE_MAX_LEN} tokens" if short
            else f"no user has {ORACLE_MAX_LEN} tokens or fewer")
    out = {"value": c_tot / t_tot, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": f"{len(users)} of {w.n_users} users of {w.name} in order, {rule} "
                     f"(encoder + all their candidates), fp64 numpy, {t_tot:.1f} s",
           "encoder_tokens_per_s": tok_tot / t_tot}
    # the oracle without the shared prefix: candidates of user 0, each re-encoding
    # its request's prefix, one at a time until a quarter of the budget is spent
    # (prefixes of at most 2048 tokens: longer ones take one candidate past it)
    from oracle import rest_oracle as O
    own = [r for r in range(len(inp["req_user"])) if int(inp["req_user"][r]) == 0]
    if max(int(inp["req_cutoff"][r]) for r in own) > 2048:
        out["no_sharing"] = {"skipped": "user 0 has a prefix longer than 2048 tokens"}
        return out
    ns, _ = no_sharing_inputs(inp, [0], max_cands=16)
    t_alone, n_alone = 0.0, 0
    while t_alone < budget_s / 4 and n_alone < len(ns["req_user"]):
        one = W.subset_users(ns, [n_alone])
        t0 = time.perf_counter()
        O.rank_request(one)
        t_alone += time.perf_counter() - t0
        n_alone += 1
    shared = t_tot / c_tot
    out["no_sharing"] = {"candidates": n_alone, "s_per_candidate_alone": t_alone / n_alone,
                         "s_per_candidate_shared": shared, "speedup_of_sharing": t_alone / n_alone / shared,
                         "sample": f"the first {n_alone} candidates of user 0, each encoding its request's "
                                   f"prefix alone, fp64 numpy, {t_alone:.1f} s"}
    return out


def run_reference(args, rank: int):
    if rank != 0:
        return
    w = W.workload(args.workload)
    inp = W.make_inputs(w, 1000 + args.workload)
    pool = oracle_users(w)
    for i in range(args.warmup):
        oracle_sample(w, inp, [pool[i % len(pool)]])
    t_tot, c_tot, tok_tot = 0.0, 0, 0
    for i in range(args.steps):
        dt, c, tok = oracle_sample(w, inp, [pool[(args.warmup + i) % len(pool)]])
        t_tot += dt
        c_tot += c
        tok_tot += tok
    value = c_tot / t_tot
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: 1 of the {len(pool)} users of {w.name} with at most "
                                   f"{ORACLE_MAX_LEN} tokens, in turn (encoder + its candidates)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "encoder_tokens_per_s": tok_tot / t_tot,
    }
    print(json.dumps(out), flush=True)


# --------------------------------------------------------------------- GPU arm

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    import shared_prefix_behavior_b200 as R

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = W.workload(args.workload)
    if world == 1:
        inp = W.make_inputs(w, 1000 + args.workload)
    else:
        # one global batch of world x the workload's users (one model); this
        # rank runs its LPT shard of the users (weak scaling, no collective)
        from shared_prefix_behavior_b200 import shard as S
        gw = W.tile_workload(w, world)
        g = W.make_inputs(gw, 1000 + args.workload)
        plan = S.partition_users(S.user_costs(g["cu_seqlens"], g["req_user"], g["req_cutoff"], g["cu_cands"],
                                              gw.d, gw.n_layers, gw.d_ff, gw.K), world)
        rows, cu, ru, rc, cc, cand_rows, _ = S.shard_arrays(g["cu_seqlens"], g["req_user"], g["req_cutoff"],
                                                            g["cu_cands"], plan[rank])
        inp = dict(g, x=g["x"][rows], ts=g["ts"][rows], cu_seqlens=cu, req_user=ru, req_cutoff=rc, cu_cands=cc,
                   z=g["z"][cand_rows])
        w = dataclasses.replace(w, lengths=[int(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)],
                                req_user=list(ru), req_cutoff=list(rc), req_ncand=list(np.diff(cc)))
    t = R.to_device(inp, dev)
    dt_name = "bf16" if w.dtype == "bf16" else "f32"
    args_rank = (t["x"], t["ts"], t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"], t["reqs"], t["z"],
                 t["dec"], t["rope_base"])
    nbytes = R.workspace_size(R.REST_BF16 if w.dtype == "bf16" else R.REST_F32, t["taus"], w.d, t["cu_seqlens"],
                              t["layers"], t["reqs"], w.K, t["rope_base"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    H = torch.empty_like(t["x"])
    Y = torch.empty(t["z"].shape, dtype=torch.float32, device=dev)
    # the decoder block and [CLS] logit turn y into the candidate scores
    dt_code = R.REST_BF16 if w.dtype == "bf16" else R.REST_F32
    ws_s = torch.empty(R.score_workspace_size(dt_code, w.d, w.K, w.total_cands, int(t["score"]["w_ffn2"].shape[1])),
                       dtype=torch.uint8, device=dev)
    F = torch.empty_like(Y)
    S = torch.empty((w.total_cands,), dtype=torch.float32, device=dev)

    def step():
        R.rank_request(*args_rank, h_out=H, y_out=Y, ws=ws, check=False)
        R.score_head(t["z"], Y, t["score"], f_out=F, score_out=S, ws=ws_s, check=False)

    def barrier():
        if world > 1:
            dist.barrier()

    # correctness guard: the device status word must stay clear
    R.rank_request(*args_rank, h_out=H, y_out=Y, ws=ws, check=True)
    R.score_head(t["z"], Y, t["score"], f_out=F, score_out=S, ws=ws_s, check=True)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    R.launch_count(reset=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.mark()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    launches = R.launch_count(reset=True)
    ms = e0.elapsed_time(e1)
    if world > 1:
        tm = torch.tensor([ms], device=dev)
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        ms = float(tm.item())
    ms_step = ms / args.steps
    cands = w.total_cands
    tokens = w.total_tokens
    if world > 1:  # whole-job totals: every rank's shard
        tot = torch.tensor([float(cands), float(tokens)], device=dev)
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
        cands, tokens = int(tot[0].item()), int(tot[1].item())
    value = cands / (ms_step * 1e-3)

    # per-kernel pass: the same steps with CUDA events around every launch
    R.profile_begin()
    for _ in range(args.steps):
        step()
    stats = R.profile_end()
    torch.cuda.synchronize()

    # end to end through the public API: pinned host inputs in, scores out.
    # Two buffer sets: step i+1's host->device copies (copy stream) overlap
    # step i's compute; every copy of every step is inside the timed region.
    x_h = t["x"].cpu().pin_memory()
    ts_h = t["ts"].cpu().pin_memory()
    z_h = t["z"].cpu().pin_memory()
    s_h = [torch.empty(S.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    bufs = [(torch.empty_like(t["x"]), torch.empty_like(t["ts"]), torch.empty_like(t["z"]),
             torch.empty_like(S)) for _ in range(2)]
    s_copy, s_comp = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]

    # copy stream: H2D(i), D2H(i-1), H2D(i+1), D2H(i), ...; compute stream: step i.
    # D2H(i) waits for step i's compute; H2D(i+2) follows D2H(i) on the copy
    # stream, so buffer set i%2 is free again when it is overwritten.
    def h2d(i):
        x_d, ts_d, z_d, _ = bufs[i % 2]
        with torch.cuda.stream(s_copy):
            x_d.copy_(x_h, non_blocking=True)
            ts_d.copy_(ts_h, non_blocking=True)
            z_d.copy_(z_h, non_blocking=True)
            copied[i % 2].record(s_copy)

    def compute(i):
        x_d, ts_d, z_d, s_d = bufs[i % 2]
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(copied[i % 2])
            R.rank_request(x_d, ts_d, t["cu_seqlens"], t["taus"], t["layers"], t["l_switch"], t["reqs"], z_d,
                           t["dec"], t["rope_base"], h_out=H, y_out=Y, ws=ws, stream=s_comp, check=False)
            R.score_head(z_d, Y, t["score"], f_out=F, score_out=s_d, ws=ws_s, stream=s_comp, check=False)
            computed[i % 2].record(s_comp)

    def d2h(i):
        with torch.cuda.stream(s_copy):
            s_copy.wait_event(computed[i % 2])
            s_h[i % 2].copy_(bufs[i % 2][3], non_blocking=True)

    def e2e_run(n):
        h2d(0)
        for i in range(n):
            compute(i)
            if i + 1 < n:
                h2d(i + 1)
            d2h(i)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_copy)
    s_comp.wait_stream(s_copy)
    e2e_run(args.steps)
    s_comp.wait_stream(s_copy)
    t1.record(s_comp)
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1)
    if world > 1:
        tm = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        e2e_ms = float(tm.item())
    e2e_value = cands / (e2e_ms / args.steps * 1e-3)

    parts = component_timings(args, w, t, H, Y, ws, dev, peaks_for_parts())
    if args.sharing and world == 1:
        parts["sharing"] = sharing_comparison(w, inp, dev, ms_step)
    if world == 1 and not args.core_only:
        parts["append"] = append_comparison(w, inp, dev, parts["encoder_only"]["ms"])
    if args.ablation and world == 1:
        parts["ablation"] = ablation_comparison(w, dev)
    if world == 1 and not args.core_only:
        parts["training"] = training_comparison(w, inp, dev)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    total_ms = sum(s["ms"] for s in stats)
    top = max(stats, key=lambda s: s["ms"])
    per_launch_s = top["ms"] / top["launches"] * 1e-3
    if top["name"].startswith(TENSOR_KERNELS):
        bound, unit = "tensor", "TFLOP/s"
        achieved = top["flops"] / top["launches"] / per_launch_s / 1e12
        peak = tensor_peak(peaks)
        peak_note = f"bf16 dense, burst ({peak_src}): the step runs at the full SM clock"
    else:
        bound, unit = "hbm", "GB/s"
        achieved = top["bytes"] / top["launches"] / per_launch_s / 1e9
        peak = float(peaks["hbm_gbs"])
        peak_note = f"HBM copy ({peak_src})"
    traffic, traffic_note = traffic_for(top["name"], w.name)
    clocks = clk.summary()
    sm_mhz = clocks["sm_mhz"] or float(peaks.get("sm_max_mhz", 1965.0))

    def exp_floor(s_):
        """Attention kernels: one exponential per (query, key, head) score, 4 head_dim FLOPs each."""
        if not s_["name"].endswith("attn") or s_["flops"] <= 0:
            return None
        n_exp = s_["flops"] / (4.0 * w.head_dim)
        floor = exp_floor_s(n_exp, sm_mhz)
        return {"exponentials_per_step": n_exp / args.steps, "floor_ms_per_step": floor * 1e3 / args.steps,
                "frac": floor / (s_["ms"] * 1e-3), "sm_mhz": sm_mhz,
                "rate": f"{EXP_PER_CLK_SM} per SM per clock x {N_SMS} SMs at the median SM clock of the timed region"}

    kernels = []
    for s in sorted(stats, key=lambda s: -s["ms"]):
        sec = s["ms"] * 1e-3
        kernels.append({"name": s["name"], "launches_per_step": s["launches"] / args.steps,
                        "ms_per_step": s["ms"] / args.steps, "share": s["ms"] / total_ms,
                        "tflops": s["flops"] / sec / 1e12 if sec > 0 else None,
                        "gbs": s["bytes"] / sec / 1e9 if sec > 0 else None})
        if exp_floor(s) is not None:
            kernels[-1]["exp_floor"] = exp_floor(s)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dt_name, "data": "synthetic (seeded; shapes of the named workload)",
        "config": workload_config(w, world, nbytes),
        "encoder_tokens_per_s": tokens / (ms_step * 1e-3),
        "roofline": {"kernel": top["name"], "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "peak_source": peak_note, "traffic": traffic,
                     "traffic_note": traffic_note,
                     "algorithmic_bytes_per_launch": top["bytes"] / top["launches"],
                     "algorithmic_flops_per_launch": top["flops"] / top["launches"],
                     "share_of_step": top["ms"] / total_ms},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": int(x_h.numel() * x_h.element_size() + ts_h.numel() * 8 +
                                          z_h.numel() * z_h.element_size()),
                "d2h_bytes_per_step": int(s_h[0].numel() * 4),
                "overlap": "double-buffered: step i+1's input copies and step i-1's score copy-back run on a "
                           "copy stream while step i computes"},
        "gpu_launches": launches,
        "clocks": clocks,
        "encoder_only": parts["encoder_only"],
        "decoder_only": parts["decoder_only"],
    }
    if bound == "tensor":
        out["roofline"]["peak_sustained"] = float(peaks.get("bf16_tflops_sustained", peak))
        out["roofline"]["frac_of_sustained"] = achieved / out["roofline"]["peak_sustained"]
    if exp_floor(top) is not None:
        out["roofline"]["exp_floor"] = exp_floor(top)
    for k in ("sharing", "append", "ablation", "training"):
        if k in parts:
            out[k] = parts[k]
    if world == 1 and not args.no_cpu_baseline and not args.core_only:
        out["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_budget)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()

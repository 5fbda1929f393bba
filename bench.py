#!/usr/bin/env python
"""Benchmark of the YOCO / YOCO++ attention core on B200.

One step is one pass of the whole hot path over one batch of synthetic,
seeded inputs (bf16, ~N(0,1); weights ~N(0,1/d)):

  swa      self-decoder, 16 sliding-window layers over B=4 x T=65536 tokens
           (d=4096, window 1024, 32q/8kv heads, head_dim 128): per layer the
           K/V projection with the YOCO++ blend to the bottom layer's K/V
           (w_l ~ U(0,1)) fused, then the SWA prefill with ring fill; then 256
           decode steps x 16 layers (projection of the 4 new tokens with the
           blend, ring write, window read), replayed from one CUDA graph
  gkv      global KV produced once: LN(x) W_kv^g for T=32768 tokens
  prefill  cross-decoder causal prefill, T=32768, 32q/8kv, head_dim 128,
           14 cross layers (each its own Q) over the one shared K/V   <- value
  decode   one decode step: global-KV append of 16 new tokens, then 16 cross
           layers each read the whole shared cache, batch 16, ragged
           lengths uniform in [65536, 131072]                          <- decode

Beside the step (timed once per run, after it): the 1M-token context (one
sequence, K/V 4 GiB): all 32 chunks of one cross layer's causal prefill, then
64 decode steps x 16 cross layers at full context with one global-KV row
appended per step; plus the early-exit prefill and the extension rows.

`value` is the cross-decoder prefill throughput in TFLOP/s of algorithmic
work (causal pairs only: 4 * Hq * D * sum_i (i + 1) per layer); `decode`
carries tokens/s and HBM GB/s.  Inputs are resident in HBM when the timed
region starts; a 256 MB buffer is rewritten between steps to flush L2 (every
part's inputs are also larger than L2).  Times are CUDA events on the
launching stream; with several GPUs each rank runs an independent replica and
the max over ranks is taken.  The library's device status word is read after
every timed block: a kernel whose bounded wait gave up makes the run fail.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl yoco|reference]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "cross-decoder prefill TFLOP/s + decode tokens/s & HBM GB/s, 1 B200"
WORKLOAD = ("cross-decoder causal prefill B=1 T=32768 32q/8kv D=128 x14 layers over one shared KV "
            "+ decode step B=16 ragged 64K-128K x16 layers + self-decoder SWA prefill B=4 T=65536 W=1024 "
            "x16 layers with YOCO++ blend and 256 decode steps")

P = dict(T=32768, Hq=32, Hkv=8, D=128, layers=14, d=4096)          # cross prefill
DEC = dict(B=16, lo=65536, hi=131072, Hq=32, Hkv=8, D=128, layers=16, d=4096, seed=2000)
SWA = dict(B=4, T=65536, W=1024, Hq=32, Hkv=8, D=128, d=4096, layers=16, steps=256)
# 1M-token context: one cross layer's 32-chunk prefill, 64 decode steps x 16 layers
LONG = dict(T=1 << 20, C=32768, Hq=32, Hkv=8, D=128, d=4096, layers=16, steps=64)
SELF_LAYERS = 14    # self-decoder depth of the early-exit measurement (half of a 28-layer stack)
# gated-retention self-decoder layer (the sliding-window slice's shape with retention heads)
GRET = dict(B=4, T=65536, H=32, D=128, tau=16.0, B_dec=16)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["yoco", "reference"], default="yoco")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-early-exit", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the 1M-token context block")
    ap.add_argument("--chunk-parallel", action="store_true",
                    help="chunk-parallel prefill of one long sequence across the ranks (NCCL)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--case", choices=["prefill", "decode", "swa", "proj", "prefill_layer", "decode_layer",
                                       "gret", "gret_decode", "decode_i8_layer", "gret1", "decode_i8",
                                       "long_prefill", "long_decode", "swa_decode_layer", "swa_step_layer", "proj_small"],
                    default=None,
                    help="time one kernel on a small case larger than L2 (for profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# DRAM bytes (read + write) per launch of the roofline kernels, from one ncu
# capture of the benchmark's own launch shape (--case prefill_layer /
# decode_layer).  Each figure is keyed by the SHA-256 of the kernel's source
# files (the .cu and the headers it includes) as they were when it was
# taken: once any of them changes the figure no longer describes the kernel,
# and the report carries null instead.
_CSRC = "shared_kv_decoder_b200/csrc/"
TRAFFIC = {
    # attn_prefill_pair_kernel<128>, T=32768: 569.859 MB read + 239.108 MB written
    "prefill": {"bytes": 569859328 + 239108096,
                "sources": ["prefill_pair.cu", "schedule.h", "tc.cuh", "common.cuh"],
                "sha256": "836177e0fbe98c89f48dc571b8a23986d590602891340cf2b4ce942e7e583e83"},
    # attn_prefill_pair_kernel<128>, sliding window 1024, B=1 x T=65536 (806.840 MB read +
    # 507.447 MB written), times 4 for the benchmark's B=4 launch: the batches are independent
    # and each reads its own Q, K, V and writes its own O once
    "swa_prefill": {"bytes": 4 * (806840320 + 507446528),
                    "sources": ['prefill_pair.cu', 'schedule.h', 'tc.cuh', 'common.cuh'],
                    "sha256": "836177e0fbe98c89f48dc571b8a23986d590602891340cf2b4ce942e7e583e83"},
    # one decode layer-step at batch 4, window 1024 (yoco_swa_decode_step):
    # linear_few_reg_kernel (the 4-token projection) 16.851 MB read +
    # ring_decode_cluster_kernel<128, 4> (4 CTAs a head) 16.888 MB read
    "swa_decode": {"bytes": 16850944 + 16887552,
                   "sources": ['ring_decode.cu', 'step_proj.cu', 'cluster.cuh', 'tc.cuh', 'common.cuh'],
                   "sha256": "1ba3719db7da2734bf0f878d3b4de9b199d3706259aeb3eea7ef611026e8bfea"},
    # decode_tma_kernel<128, 4>, batch 16 at 64K-128K: 6.416165 GB read + 25.238 MB written
    "decode": {"bytes": 6416165120 + 25238272,
               "sources": ["decode.cu", "schedule.h", "tc.cuh", "common.cuh"],
               "sha256": "e0b8311437112b861d4c0f91d6e071903fe71e380c3dfe04e2c884c4d197bd6f"},
}


def traffic(kind):
    import hashlib
    t = TRAFFIC[kind]
    m = hashlib.sha256()
    try:
        for f in t["sources"]:
            m.update(open(os.path.join(ROOT, _CSRC, f), "rb").read())
    except OSError:
        return None
    return float(t["bytes"]) if m.hexdigest() == t["sha256"] else None


def reduce_max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over every rank of the default
    process group (identity without one): each rank runs an independent
    replica, and the job is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def gret_flops(B, T, H, D, chunk=128):
    """Tensor FLOPs of chunkwise gated retention at the kernel's chunk size: per
    chunk and head, Q K^T and P V over the chunk's causal pairs (counted in
    full, C x C) plus the cross term Q S and the state update K^T V (D x D
    each), 2 FLOP per multiply-add."""
    n_chunks = -(-T // chunk)
    per_chunk = 2 * (2.0 * chunk * chunk * D) + 2 * (2.0 * chunk * D * D)
    return B * H * n_chunks * per_chunk


def prefill_flops_per_layer(T, Hq, D, q_pos0=0, window=0):
    """4 * Hq * D * sum over query rows of the visible key count."""
    import numpy as np
    i = np.arange(T, dtype=np.float64) + q_pos0
    vis = i + 1 if window <= 0 else np.minimum(i + 1, window)
    return 4.0 * Hq * D * float(vis.sum())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        loaded = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- workloads
def make_workload(dev):
    import torch
    import shared_kv_decoder_b200 as yoco
    import workloads as wl
    bf = torch.bfloat16
    W = {}
    # cross prefill: x_mid -> global K/V, then 14 layers each with its own Q
    T, Hq, Hkv, D, d = P["T"], P["Hq"], P["Hkv"], P["D"], P["d"]
    W["x_mid"] = wl.normal((T, d), 1100, bf, dev)
    W["w_g"] = wl.normal((2 * Hkv * D, d), 1101, bf, dev, std=d ** -0.5)
    W["kg"] = torch.empty((1, T, Hkv, D), dtype=bf, device=dev)
    W["vg"] = torch.empty((1, T, Hkv, D), dtype=bf, device=dev)
    W["qs"] = [wl.normal((1, T, Hq, D), 1200 + l, bf, dev) for l in range(P["layers"])]
    W["o"] = torch.empty((1, T, Hq, D), dtype=bf, device=dev)
    # decode: packed shared cache of 16 ragged sequences
    lens = wl.ragged_lengths(DEC["B"], DEC["lo"], DEC["hi"], DEC["seed"])
    starts = torch.cumsum(torch.cat([torch.zeros(1, dtype=torch.int64), lens[:-1]]), 0)
    rows = int(lens.sum())
    W["lens"], W["starts"], W["rows"] = lens, starts, rows
    W["kc"] = wl.normal((rows, Hkv, D), 2001, bf, dev)
    W["vc"] = wl.normal((rows, Hkv, D), 2002, bf, dev)
    W["x_new"] = wl.normal((DEC["B"], d), 2003, bf, dev)
    W["w_gd"] = wl.normal((2 * Hkv * D, d), 2004, bf, dev, std=d ** -0.5)
    W["qd"] = [wl.normal((DEC["B"], Hq, D), 2100 + l, bf, dev) for l in range(DEC["layers"])]
    W["od"] = torch.empty((DEC["B"], Hq, D), dtype=bf, device=dev)
    W["seq_start"] = starts.to(dev)
    W["seq_len"] = lens.to(torch.int32).to(dev)
    W["dst_rows"] = (starts + lens - 1).to(dev)
    W["max_len"] = int(lens.max())
    W["ws"] = torch.empty(yoco.cross_decode_workspace_size(DEC["B"], W["max_len"], Hq, Hkv, D, bf),
                          dtype=torch.uint8, device=dev)
    # self-decoder: 16 sliding-window layers, each with its own x_l, W_kv^l,
    # Q_l and YOCO++ weight w_l (w_1 unused: the bottom layer is not blended)
    B4, T4, W4, L4, S4 = SWA["B"], SWA["T"], SWA["W"], SWA["layers"], SWA["steps"]
    n4 = B4 * T4
    W["x4"] = [wl.normal((n4, d), 3100 + l, bf, dev) for l in range(L4)]
    W["w4"] = [wl.normal((2 * Hkv * D, d), 3200 + l, bf, dev, std=d ** -0.5) for l in range(L4)]
    W["q4"] = [wl.normal((B4, T4, Hq, D), 3300 + l, bf, dev) for l in range(L4)]
    W["w_l"] = [float(v) for v in wl.uniform((L4,), 3005)]
    W["k1"], W["v1"], W["k4"], W["v4"] = (torch.empty((B4, T4, Hkv, D), dtype=bf, device=dev)
                                          for _ in range(4))
    W["o4"] = torch.empty((B4, T4, Hq, D), dtype=bf, device=dev)
    W["rings"] = [(torch.empty((B4, W4, Hkv, D), dtype=bf, device=dev),
                   torch.empty((B4, W4, Hkv, D), dtype=bf, device=dev),
                   torch.empty((B4, W4), dtype=torch.int32, device=dev)) for _ in range(L4)]
    # decode steps past the prompt: per step and layer the 4 new tokens' x and q
    W["x4d"] = wl.normal((S4, L4, B4, d), 3400, bf, dev)
    W["q4d"] = wl.normal((S4, L4, B4, Hq, D), 3401, bf, dev)
    W["pos4"] = (T4 + torch.arange(S4, dtype=torch.int64, device=dev))[:, None].repeat(1, B4).contiguous()
    W["k1t"], W["v1t"] = (torch.empty((B4, Hkv, D), dtype=bf, device=dev) for _ in range(2))
    W["o4t"] = torch.empty((B4, Hq, D), dtype=bf, device=dev)
    W["ws4"] = torch.empty(yoco.swa_decode_step_workspace_size(B4, W4, Hq, Hkv, D, bf),
                           dtype=torch.uint8, device=dev)
    W["flush"] = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    return W


def self_decoder_prefill(W, ev=None):
    """The 16 sliding-window layers over the B=4 x T=65536 prompt: the bottom
    layer's K/V projection, then for every other layer its projection with the
    YOCO++ blend w_l * (K_1, V_1) fused; each followed by the SWA prefill,
    which also fills that layer's ring."""
    import shared_kv_decoder_b200 as yoco
    Hkv, D, Wn = SWA["Hkv"], SWA["D"], SWA["W"]
    flat = lambda t: t.view(-1, Hkv, D)
    for l in range(SWA["layers"]):
        if ev is not None:
            ev["swa_proj"][2 * l].record()
        if l == 0:
            yoco.kv_project_blend(W["x4"][0], W["w4"][0], Hkv, D, k_out=flat(W["k1"]), v_out=flat(W["v1"]))
            k, v = W["k1"], W["v1"]
        else:
            yoco.kv_project_blend(W["x4"][l], W["w4"][l], Hkv, D, flat(W["k1"]), flat(W["v1"]),
                                  W["w_l"][l], W["w_l"][l], k_out=flat(W["k4"]), v_out=flat(W["v4"]))
            k, v = W["k4"], W["v4"]
        if ev is not None:
            ev["swa_proj"][2 * l + 1].record()
            ev["swa_att"][2 * l].record()
        yoco.swa_prefill(W["q4"][l], k, v, Wn, ring=W["rings"][l], o=W["o4"])
        if ev is not None:
            ev["swa_att"][2 * l + 1].record()


def self_decoder_decode(W):
    """256 decode steps of the 16 sliding-window layers: per step and layer
    one yoco_swa_decode_step call -- the 4 new tokens' K/V projection
    (blended with the bottom layer's K/V of the same tokens), the window
    read, the merge with the new token and its ring write.  Position T + s of
    step s overwrites the ring slot of T + s - window, so replaying the steps
    after a prefill is idempotent."""
    import shared_kv_decoder_b200 as yoco
    Wn = SWA["W"]
    for s in range(SWA["steps"]):
        for l in range(SWA["layers"]):
            rk, rv, sp = W["rings"][l]
            if l == 0:   # the bottom layer's new K/V: the base of the layers above
                yoco.swa_decode_step(W["x4d"][s, 0], W["w4"][0], W["q4d"][s, 0], W["pos4"][s], rk, rv, sp, Wn,
                                     k_out=W["k1t"], v_out=W["v1t"], workspace=W["ws4"], o=W["o4t"])
            else:
                yoco.swa_decode_step(W["x4d"][s, l], W["w4"][l], W["q4d"][s, l], W["pos4"][s], rk, rv, sp, Wn,
                                     W["k1t"], W["v1t"], W["w_l"][l], W["w_l"][l], workspace=W["ws4"],
                                     o=W["o4t"])


def capture_self_decoder_decode(W):
    """One CUDA graph of the 256 x 16 decode layer-steps (2 kernels each), so
    the steps run back to back without host launch overhead.  The rings must
    hold a prefill's contents (the graph is recorded after one eager run).
    Returns the number of library kernels one replay launches."""
    import torch
    import shared_kv_decoder_b200 as yoco
    self_decoder_prefill(W)
    self_decoder_decode(W)          # eager once: every kernel's attributes are set
    torch.cuda.synchronize()
    n0 = yoco.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        self_decoder_decode(W)
    torch.cuda.synchronize()
    W["swa_graph"] = g
    W["swa_graph_launches"] = yoco.launch_count() - n0
    return W["swa_graph_launches"]


def run_step(W, ev=None):
    """One pass of the hot path.  ev: dict of per-part event lists to record."""
    import shared_kv_decoder_b200 as yoco
    Hkv, D = P["Hkv"], P["D"]

    def rec(name, i):
        if ev is not None:
            ev[name][i].record()

    # self-decoder: 16-layer prefill (projection + blend, SWA + ring), then
    # 256 decode steps of the 16 layers
    rec("swa", 0)
    self_decoder_prefill(W, ev)
    rec("swa", 1)
    rec("swa_dec", 0)
    W["swa_graph"].replay()
    rec("swa_dec", 1)
    # global KV, produced once
    rec("gkv", 0)
    yoco.kv_project_blend(W["x_mid"], W["w_g"], Hkv, D, k_out=W["kg"].view(-1, Hkv, D),
                          v_out=W["vg"].view(-1, Hkv, D))
    rec("gkv", 1)
    # cross-decoder prefill, 14 layers
    for l in range(P["layers"]):
        if ev is not None:
            ev["prefill_l"][2 * l].record()
        yoco.cross_prefill(W["qs"][l], W["kg"], W["vg"], o=W["o"])
        if ev is not None:
            ev["prefill_l"][2 * l + 1].record()
    # decode step: append 16 new global-KV rows, then 16 cross layers
    rec("decode", 0)
    yoco.kv_project_blend(W["x_new"], W["w_gd"], Hkv, D, dst_rows=W["dst_rows"],
                          k_out=W["kc"], v_out=W["vc"])
    for l in range(DEC["layers"]):
        if ev is not None:
            ev["decode_l"][2 * l].record()
        yoco.cross_decode(W["qd"][l], W["kc"], W["vc"], W["seq_start"], W["seq_len"],
                          W["max_len"], workspace=W["ws"], o=W["od"])
        if ev is not None:
            ev["decode_l"][2 * l + 1].record()
    rec("decode", 1)


def new_events():
    import torch
    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    return {"swa": mk(2), "swa_dec": mk(2), "swa_proj": mk(2 * SWA["layers"]),
            "swa_att": mk(2 * SWA["layers"]), "gkv": mk(2), "decode": mk(2),
            "prefill_l": mk(2 * P["layers"]), "decode_l": mk(2 * DEC["layers"]), "step": mk(2)}


def swa_tile_flops_per_layer(B, T, Hq, D, window):
    """FLOPs the tensor cores execute for a sliding-window prefill layer: every
    visited 128 x 128 (query, key) tile in full, 4 * D FLOP per pair, with the
    visited KV tiles of a query tile being those that hold a visible pair."""
    n = 0
    for qt in range(-(-T // 128)):
        p_first, p_last = qt * 128, min(qt * 128 + 128, T) - 1
        lo = max(0, p_first - window + 1) // 128
        n += p_last // 128 - lo + 1
    return 4.0 * D * 128 * 128 * n * B * Hq


def early_exit(W, reps):
    """Early-exit prefill against the full prefill of one prompt, attention core
    only ("You Only Cache Once", paperlayer summary, section 2: the prompt rows
    skip the cross-decoder, only the last row goes through it).  Both run the
    self-decoder (SELF_LAYERS sliding-window layers: K/V projection with the
    YOCO++ blend, then SWA prefill with the ring fill) and the global K/V
    projection over the T=32768 prompt; then the full prefill runs the 14
    cross layers over every row, the early exit one cross decode of the last
    row per cross layer.  Query / output projections and feed-forward layers
    are not part of the attention core and are left out of both.  Returns
    device milliseconds per prompt (mean over reps after one warm-up)."""
    import torch
    import shared_kv_decoder_b200 as yoco
    import workloads as wl
    bf, dev = torch.bfloat16, W["o"].device
    T, Hq, Hkv, D, d, Wn = P["T"], P["Hq"], P["Hkv"], P["D"], P["d"], SWA["W"]
    x = wl.normal((T, d), 4001, bf, dev)
    ws_ = [wl.normal((2 * Hkv * D, d), 4100 + l, bf, dev, std=d ** -0.5) for l in range(SELF_LAYERS)]
    w_l = [float(v) for v in wl.uniform((SELF_LAYERS,), 4002)]
    k1, v1, kl, vl = (torch.empty((1, T, Hkv, D), dtype=bf, device=dev) for _ in range(4))
    q = wl.normal((1, T, Hq, D), 4003, bf, dev)
    o = torch.empty((1, T, Hq, D), dtype=bf, device=dev)
    ring = (torch.empty((1, Wn, Hkv, D), dtype=bf, device=dev), torch.empty((1, Wn, Hkv, D), dtype=bf, device=dev),
            torch.empty((1, Wn), dtype=torch.int32, device=dev))
    qlast = [q_.view(T, Hq, D)[T - 1:].contiguous() for q_ in W["qs"]]
    od = torch.empty((1, Hq, D), dtype=bf, device=dev)
    ss = torch.zeros(1, dtype=torch.int64, device=dev)
    sl = torch.full((1,), T, dtype=torch.int32, device=dev)
    wsd = torch.empty(yoco.cross_decode_workspace_size(1, T, Hq, Hkv, D, bf), dtype=torch.uint8, device=dev)

    def self_decoder():
        for l in range(SELF_LAYERS):
            if l == 0:
                yoco.kv_project_blend(x, ws_[0], Hkv, D, k_out=k1.view(-1, Hkv, D), v_out=v1.view(-1, Hkv, D))
                k, v = k1, v1
            else:
                yoco.kv_project_blend(x, ws_[l], Hkv, D, k1.view(-1, Hkv, D), v1.view(-1, Hkv, D), w_l[l], w_l[l],
                                      k_out=kl.view(-1, Hkv, D), v_out=vl.view(-1, Hkv, D))
                k, v = kl, vl
            yoco.swa_prefill(q, k, v, Wn, ring=ring, o=o)
        yoco.kv_project_blend(W["x_mid"], W["w_g"], Hkv, D, k_out=W["kg"].view(-1, Hkv, D),
                              v_out=W["vg"].view(-1, Hkv, D))

    def cross_full():
        for l in range(P["layers"]):
            yoco.cross_prefill(W["qs"][l], W["kg"], W["vg"], o=W["o"])

    def cross_last_row():
        for l in range(P["layers"]):
            yoco.cross_decode(qlast[l], W["kg"].view(T, Hkv, D), W["vg"].view(T, Hkv, D), ss, sl, T,
                              workspace=wsd, o=od)

    def timed(fn):
        ts = []
        for i in range(reps + 1):
            W["flush"].zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(); fn(); e1.record()
            torch.cuda.synchronize()
            if i > 0:
                ts.append(e0.elapsed_time(e1))
        return statistics.mean(ts)

    t_self = timed(self_decoder)
    t_full = timed(cross_full)
    t_ee = timed(cross_last_row)
    return {"T": T, "self_layers": SELF_LAYERS, "cross_layers": P["layers"], "window": Wn,
            "self_decoder_ms": t_self, "cross_full_ms": t_full, "cross_last_row_ms": t_ee,
            "prefill_full_ms": t_self + t_full, "prefill_early_exit_ms": t_self + t_ee,
            "speedup": (t_self + t_full) / (t_self + t_ee),
            "note": "attention core only (no Q/O projections, no feed-forward); self_decoder_ms "
                    "includes the global K/V projection"}


def gret_layer(W, reps):
    """The gated-retention self-decoder layer, measured beside the step (it is
    not part of it): the chunkwise prefill over B=4 x T=65536 tokens with 32
    heads (one launch, L2 flushed before it), and the decode step for a batch
    of 16 as a decode loop runs it: 16 layers of their own states (536 MB, far
    beyond L2) back to back in a CUDA graph, the time per layer.  Device ms,
    mean over reps."""
    import torch
    import shared_kv_decoder_b200 as yoco
    import workloads as wl
    bf, dev = torch.bfloat16, W["o"].device
    B, T, H, D, tau, Bd = GRET["B"], GRET["T"], GRET["H"], GRET["D"], GRET["tau"], GRET["B_dec"]
    q, k, v = (wl.normal((B, T, H, D), 5001 + i, bf, dev) for i in range(3))
    g = wl.normal((B, T, H), 5004, torch.float32, dev) + 3.0
    o = torch.empty_like(q)
    st = torch.zeros((B, H, D, D), dtype=torch.float32, device=dev)
    Ld = 16
    qd, kd, vd = ([wl.normal((Bd, H, D), 5011 + 10 * l + i, bf, dev) for l in range(Ld)] for i in range(3))
    gd = [wl.normal((Bd, H), 5014 + l, torch.float32, dev) + 3.0 for l in range(Ld)]
    sd = [torch.zeros((Bd, H, D, D), dtype=torch.float32, device=dev) for _ in range(Ld)]
    od = torch.empty_like(qd[0])

    def timed(fn):
        ts = []
        for i in range(reps + 1):
            W["flush"].zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(); fn(); e1.record()
            torch.cuda.synchronize()
            if i > 0:
                ts.append(e0.elapsed_time(e1))
        return statistics.mean(ts)

    t_pre = timed(lambda: yoco.gret_prefill(q, k, v, g, tau, state=st, o=o))
    dec_layers = lambda: [yoco.gret_decode(qd[l], kd[l], vd[l], gd[l], tau, sd[l], o=od) for l in range(Ld)]
    dec_layers()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dec_layers()
    tl = []
    for i in range(reps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(); graph.replay(); e1.record()
        torch.cuda.synchronize()
        if i > 0:
            tl.append(e0.elapsed_time(e1) / Ld)
    t_dec = statistics.mean(tl)
    del graph
    # batch 1: 32 sequences for 148 SMs, so each runs as superchunks on
    # separate CTAs (the workspace the library asks for)
    q1, k1, v1, g1, o1 = q[:1], k[:1], v[:1], g[:1], o[:1]
    st1 = torch.zeros((1, H, D, D), dtype=torch.float32, device=dev)
    ws1 = torch.empty(max(16, yoco.gret_prefill_workspace_size(1, T, H, D)), dtype=torch.uint8, device=dev)
    t_pre1 = timed(lambda: yoco.gret_prefill(q1, k1, v1, g1, tau, state=st1, o=o1, workspace=ws1))
    pre_bytes = 4.0 * B * T * H * D * 2 + B * T * H * 4.0 + 2.0 * B * H * D * D * 4
    return {"prefill_ms": t_pre, "prefill_tflops": gret_flops(B, T, H, D) / (t_pre * 1e-3) / 1e12,
            "prefill_tokens_per_s": B * T / (t_pre * 1e-3),
            "prefill_hbm_gbs": pre_bytes / (t_pre * 1e-3) / 1e9,
            "prefill_b1_ms": t_pre1, "prefill_b1_tflops": gret_flops(1, T, H, D) / (t_pre1 * 1e-3) / 1e12,
            "decode_ms": t_dec, "decode_gbs": Bd * H * D * D * 8.0 / (t_dec * 1e-3) / 1e9,
            "shape": f"prefill B={B} T={T} H={H} D={D}; decode batch {Bd}",
            "flops": "chunkwise at chunk 128: QK^T and PV over C x C, Q S and K^T V over D x D, per chunk and head",
            "bytes": "q, k, v read and o written once (bf16), gate logits, state in and out (fp32)"}


def decode_i8_step(W, reps):
    """The benchmark's decode step over the 8-bit copy of the same shared cache,
    measured beside the step (it is not part of it): quantise the bf16 cache
    once, then 16 cross layers of yoco_cross_decode_i8 for the 16 sequences.
    Device ms per decode step (mean over reps, L2 rewritten before each)."""
    import torch
    import shared_kv_decoder_b200 as yoco
    Hkv, D = DEC["Hkv"], DEC["D"]
    kq, vq = yoco.kv_quantize_i8(W["kc"], W["vc"])

    def step():
        for l in range(DEC["layers"]):
            yoco.cross_decode_i8(W["qd"][l], kq, vq, Hkv, W["seq_start"], W["seq_len"], W["max_len"],
                                 workspace=W["ws"], o=W["od"])

    ts = []
    for i in range(reps + 1):
        W["flush"].zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(); step(); e1.record()
        torch.cuda.synchronize()
        if i > 0:
            ts.append(e0.elapsed_time(e1))
    ms = statistics.mean(ts)
    layer_bytes = 2.0 * W["rows"] * yoco.kv_i8_row_bytes(Hkv, D)
    del kq, vq
    return {"ms_per_decode_step": ms, "tokens_per_s": DEC["B"] / (ms * 1e-3),
            "hbm_gbs": layer_bytes * DEC["layers"] / (ms * 1e-3) / 1e9, "bytes_per_layer": layer_bytes,
            "note": "same sequences and queries as the decode block; int8 codes with one fp32 scale per "
                    "(token, KV head): half the cache bytes"}


def long_context(W, peaks):
    """The 1M-token context, measured beside the step (once per run): one
    sequence whose shared K/V holds 1,048,576 rows (4 GiB of K and V).

    Prefill: all 32 chunks of 32768 queries of one cross layer, chunk c at
    positions [c C, (c + 1) C) attending causally to keys [0, (c + 1) C) (each
    chunk its own seeded Q; 9.007e15 FLOP of visible pairs).  The other 15
    cross layers repeat the same work on their own Q; one layer is timed in
    full.  Decode: 64 steps, each appending the new token's global-KV row
    (LN(x) W_kv^g written at row T + s) and then 16 cross layers over all
    T + s + 1 rows.  Device ms from CUDA events; the first chunk and two
    decode steps run once untimed first (the decode rows they append are
    appended again, with the same values, by the timed steps)."""
    import torch
    import shared_kv_decoder_b200 as yoco
    import workloads as wl
    bf, dev = torch.bfloat16, W["o"].device
    T, C, Hq, Hkv, D, d, L, S = (LONG[k] for k in ("T", "C", "Hq", "Hkv", "D", "d", "layers", "steps"))
    n_chunks = T // C
    kc = wl.normal((T + S, Hkv, D), 5001, bf, dev)
    vc = wl.normal((T + S, Hkv, D), 5002, bf, dev)
    qs = [wl.normal((1, C, Hq, D), 5100 + c, bf, dev) for c in range(n_chunks)]
    o = torch.empty((1, C, Hq, D), dtype=bf, device=dev)
    xd = wl.normal((S, 1, d), 5003, bf, dev)
    wg = wl.normal((2 * Hkv * D, d), 5004, bf, dev, std=d ** -0.5)
    qd = wl.normal((S, L, 1, Hq, D), 5005, bf, dev)
    od = torch.empty((1, Hq, D), dtype=bf, device=dev)
    rows = [torch.tensor([T + s], dtype=torch.int64, device=dev) for s in range(S)]
    ss = torch.zeros(1, dtype=torch.int64, device=dev)
    sl = [torch.tensor([T + s + 1], dtype=torch.int32, device=dev) for s in range(S)]
    max_len = T + S
    ws = torch.empty(yoco.cross_decode_workspace_size(1, max_len, Hq, Hkv, D, bf), dtype=torch.uint8, device=dev)

    def chunk(c):
        n = (c + 1) * C
        yoco.cross_prefill(qs[c], kc[:n].view(1, n, Hkv, D), vc[:n].view(1, n, Hkv, D), q_pos0=c * C, o=o)

    def step(s):
        yoco.kv_project_blend(xd[s], wg, Hkv, D, dst_rows=rows[s], k_out=kc, v_out=vc)
        for l in range(L):
            yoco.cross_decode(qd[s, l], kc, vc, ss, sl[s], max_len, workspace=ws, o=od)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    chunk(n_chunks - 1)
    step(0); step(1)
    torch.cuda.synchronize()
    W["flush"].zero_()
    ce = [(ev(), ev()) for _ in range(n_chunks)]
    for c in range(n_chunks):
        ce[c][0].record(); chunk(c); ce[c][1].record()
    W["flush"].zero_()
    d0, d1 = ev(), ev()
    d0.record()
    for s in range(S):
        step(s)
    d1.record()
    torch.cuda.synchronize()
    chunk_ms = [a.elapsed_time(b) for a, b in ce]
    pre_ms = sum(chunk_ms)
    pre_fl = sum(prefill_flops_per_layer(C, Hq, D, c * C) for c in range(n_chunks))
    last_fl = prefill_flops_per_layer(C, Hq, D, T - C)
    dec_ms = d0.elapsed_time(d1)
    row_bytes = Hkv * D * 2 * 2
    dec_bytes = L * sum((T + s + 1) * row_bytes for s in range(S))
    pre_tf = pre_fl / (pre_ms * 1e-3) / 1e12
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9
    del kc, vc, qs
    return {"T": T, "chunk": C, "chunks": n_chunks, "prefill_layers_timed": 1,
            "prefill_ms_per_layer": pre_ms, "prefill_flops_per_layer": pre_fl, "prefill_tflops": pre_tf,
            "prefill_frac": pre_tf / peaks["bf16_sus"], "prefill_peak_src": f"{peaks['src']} bf16 sustained",
            "last_chunk_ms": chunk_ms[-1], "last_chunk_tflops": last_fl / (chunk_ms[-1] * 1e-3) / 1e12,
            "decode_steps": S, "decode_layers": L, "decode_ms_per_step": dec_ms / S,
            "decode_tokens_per_s": S / (dec_ms * 1e-3), "decode_hbm_gbs": dec_gbs,
            "decode_frac": dec_gbs / peaks["hbm"], "decode_peak_src": f"{peaks['src']} hbm",
            "note": "one cross layer's 32-chunk prefill timed in full (the other 15 layers repeat it on "
                    "their own Q); decode: per step the appended row's projection + 16 cross layers over "
                    "the whole cache; bytes are the K/V rows each layer reads"}


def e2e_prefill(W, steps, warmup):
    """Prefill through the public API with HOST buffers: every step copies the
    step's Q (14 layers) and the shared K/V from pinned host memory and reads
    every layer's output back into its own pinned host buffer, all inside the
    timed region.  The copies run on their own streams and overlap the
    kernels as a caller serving one prompt after another would arrange them:
    layer l+1's Q goes up while layer l computes, layer l-1's O comes down,
    and the next step's K/V and first Q go up while this step's last layers
    run (two device buffers each, events for the hand-offs).  The steps are
    timed as one region (the same kernels and copies as step by step; L2 is
    flushed between steps on the compute stream).  Returns one time per step
    (the region's time divided evenly) and the bytes each step copies."""
    import torch
    import shared_kv_decoder_b200 as yoco
    L = P["layers"]
    hq = [q.cpu().pin_memory() for q in W["qs"]]
    hk = W["kg"].cpu().pin_memory()
    hv = W["vg"].cpu().pin_memory()
    ho = [torch.empty(W["o"].shape, dtype=W["o"].dtype).pin_memory() for _ in range(L)]
    dq = [torch.empty_like(W["qs"][0]) for _ in range(2)]
    do = [torch.empty_like(W["o"]) for _ in range(2)]
    dk = [torch.empty_like(W["kg"]) for _ in range(2)]
    dv = [torch.empty_like(W["vg"]) for _ in range(2)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()

    def run(n_steps):
        # global layer index g = step * L + l: Q / O buffers alternate by g,
        # K / V buffers by step
        n = n_steps * L
        if n == 0:
            return
        in_ready = [ev() for _ in range(n)]
        comp_done = [ev() for _ in range(n)]
        out_done = [ev() for _ in range(n)]
        kv_ready = [ev() for _ in range(n_steps)]

        def upload(g):
            st, l = divmod(g, L)
            with torch.cuda.stream(s_in):
                if l == 0:
                    if st >= 2:
                        s_in.wait_event(comp_done[(st - 2) * L + L - 1])   # dk/dv[st % 2] free again
                    dk[st % 2].copy_(hk, non_blocking=True)
                    dv[st % 2].copy_(hv, non_blocking=True)
                    kv_ready[st].record(s_in)
                if g >= 2:
                    s_in.wait_event(comp_done[g - 2])                      # dq[g % 2] free again
                dq[g % 2].copy_(hq[l], non_blocking=True)
                in_ready[g].record(s_in)

        upload(0)
        for g in range(n):
            st, l = divmod(g, L)
            if g + 1 < n:
                upload(g + 1)
            if l == 0 and st >= 1:
                W["flush"].zero_()                  # L2 flushed between steps
            comp.wait_event(kv_ready[st])
            comp.wait_event(in_ready[g])
            if g >= 2:
                comp.wait_event(out_done[g - 2])    # do[g % 2] has been read out
            yoco.cross_prefill(dq[g % 2], dk[st % 2], dv[st % 2], o=do[g % 2])
            comp_done[g].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[g])
                ho[l].copy_(do[g % 2], non_blocking=True)
                out_done[g].record(s_out)
        comp.wait_event(out_done[n - 1])
        comp.wait_stream(s_in)

    W["flush"].zero_()
    run(warmup)
    torch.cuda.synchronize()
    W["flush"].zero_()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps)
    e1.record(comp)
    torch.cuda.synchronize()
    total = e0.elapsed_time(e1)
    times = [total / steps] * steps
    h2d = sum(q.numel() * q.element_size() for q in hq) + 2 * hk.numel() * hk.element_size()
    d2h = sum(o.numel() * o.element_size() for o in ho)
    return times, h2d, d2h


# ------------------------------------------------------------ CPU baseline
def cpu_baseline(W, seconds, label="oracle"):
    """The oracle, as it stands, on sampled query rows of the prefill
    workload (layer 0), timed on this host's cores."""
    import numpy as np
    import oracle
    T, Hq, D = P["T"], P["Hq"], P["D"]
    k = W["kg"].double().cpu().numpy() if hasattr(W["kg"], "double") else W["kg"]
    v = W["vg"].double().cpu().numpy() if hasattr(W["vg"], "double") else W["vg"]
    q = W["qs"][0] if not hasattr(W["qs"][0], "double") else W["qs"][0].double().cpu().numpy()
    rng = np.random.default_rng(7)

    def run(n):
        rows = np.sort(rng.integers(0, T, size=n))
        t0 = time.perf_counter()
        oracle.attention(q, k, v, 0, 0, rows=[(0, int(i)) for i in rows])
        dt = time.perf_counter() - t0
        return dt, 4.0 * Hq * D * float((rows + 1).sum()), n

    dt, fl, n = run(4)
    n2 = max(4, int(4 * seconds / max(dt, 1e-3)))
    dt, fl, n = run(n2)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} random query rows (all 32 heads) of cross prefill layer 0, T=32768, "
                      f"fp64, {dt:.1f} s"}


def run_reference(args):
    """The CPU oracle as the reference arm, on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch
    import workloads as wl
    T, Hq, Hkv, D = P["T"], P["Hq"], P["Hkv"], P["D"]
    # the shared K/V and layer-0 Q on the host (bf16-rounded, widened to fp64)
    W = {"kg": wl.normal((1, T, Hkv, D), 1300, torch.bfloat16).double().numpy(),
         "vg": wl.normal((1, T, Hkv, D), 1301, torch.bfloat16).double().numpy(),
         "qs": [wl.normal((1, T, Hq, D), 1200, torch.bfloat16).double().numpy()]}
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals = []
    for it in range(args.warmup + args.steps):
        cb = cpu_baseline(W, per_step)
        if it >= args.warmup:
            vals.append(cb)
    value = statistics.median(c["value"] for c in vals)
    flops_per_step = prefill_flops_per_layer(T, Hq, D) * P["layers"]
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": flops_per_step / (value * 1e12) * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": {"workload": WORKLOAD, "model": "YOCO attention core (synthetic)",
                      "global_batch": 1, "seq_len": T, "parallelism": "replicas",
                      "note": "each step times the oracle on a bounded sample of query rows; "
                              "ms_per_step is extrapolated to the 14-layer prefill"},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": vals[0]["cores"],
                            "kind": "oracle", "sample": vals[0]["sample"]},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_case(args):
    """One kernel on a small case whose inputs still exceed L2 (126 MB):
      prefill  cross prefill T=16384, 32q/8kv, D=128 (Q 128 MB, K+V 64 MB)
      decode   cross decode, batch 16, lengths in [16384, 32768] (cache ~1.6 GB)
      swa      sliding-window prefill B=1, T=65536, window 1024 (Q 512 MB)
      proj     K/V projection + blend, 32768 tokens, d=4096 (x 256 MB)
      prefill_layer / decode_layer  one launch of the full benchmark's own
               prefill layer (T=32768) / decode layer (batch 16, 64K-128K)
      gret     gated-retention chunkwise prefill B=4, T=65536, 32 heads, D=128
      gret_decode  one gated-retention decode step, batch 16, 32 heads (state 34 MB, L2 flushed)
      decode_i8_layer  one decode layer over the 8-bit cache of the benchmark's decode shape
      gret1 / decode_i8  the same at batch 1 / at the decode case's shape (for profiling)
      long_prefill / long_decode  the 1M-token context (K/V 4 GiB): the last 32K-query
               chunk of the causal prefill over the whole prefix / one decode step of one
               sequence over all 1,048,576 rows
      swa_decode_layer  one sliding-window decode call at the self-decoder's shape (batch 4,
               window 1024: window attention + merge with the new token's ring write, 16.8 MB of ring)
      swa_step_layer  one self-decoder decode step call at that shape (the 4 tokens' projection, d=4096,
               then the window decode): 16.8 MB of weights + 16.8 MB of ring
      proj_small  the decode step's K/V projection of 4 tokens, d=4096 -> 2048, with the blend (16.8 MB
               of weights)
    Prints one JSON line with the mean launch time and the work rate."""
    import torch
    import shared_kv_decoder_b200 as yoco
    import workloads as wl
    bf, dev = torch.bfloat16, "cuda"
    yoco.load()
    Hq, Hkv, D = 32, 8, 128
    if args.case in ("prefill", "prefill_layer"):
        T = 16384 if args.case == "prefill" else P["T"]
        q = wl.normal((1, T, Hq, D), 1, bf, dev); k = wl.normal((1, T, Hkv, D), 2, bf, dev)
        v = wl.normal((1, T, Hkv, D), 3, bf, dev); o = torch.empty_like(q)
        fn = lambda: yoco.cross_prefill(q, k, v, o=o)
        work, unit = prefill_flops_per_layer(T, Hq, D), "TFLOP/s"
    elif args.case in ("decode", "decode_layer"):
        lens = (wl.ragged_lengths(16, 16384, 32768, 9) if args.case == "decode" else
                wl.ragged_lengths(DEC["B"], DEC["lo"], DEC["hi"], DEC["seed"]))
        starts = torch.cumsum(torch.cat([torch.zeros(1, dtype=torch.int64), lens[:-1]]), 0)
        rows = int(lens.sum())
        kc = wl.normal((rows, Hkv, D), 4, bf, dev); vc = wl.normal((rows, Hkv, D), 5, bf, dev)
        q = wl.normal((16, Hq, D), 6, bf, dev); o = torch.empty_like(q)
        ss, sl = starts.to(dev), lens.to(torch.int32).to(dev)
        ws = torch.empty(yoco.cross_decode_workspace_size(16, int(lens.max()), Hq, Hkv, D, bf),
                         dtype=torch.uint8, device=dev)
        fn = lambda: yoco.cross_decode(q, kc, vc, ss, sl, int(lens.max()), workspace=ws, o=o)
        work, unit = rows * Hkv * D * 4.0, "GB/s"
    elif args.case == "swa":
        T, Wn = 65536, 1024
        q = wl.normal((1, T, Hq, D), 7, bf, dev); k = wl.normal((1, T, Hkv, D), 8, bf, dev)
        v = wl.normal((1, T, Hkv, D), 9, bf, dev); o = torch.empty_like(q)
        fn = lambda: yoco.swa_prefill(q, k, v, Wn, o=o)
        work, unit = prefill_flops_per_layer(T, Hq, D, 0, Wn), "TFLOP/s"
    elif args.case == "proj_small":
        # the self-decoder decode step's projection: 4 new tokens, d=4096 -> [K | V] 2048, with the blend;
        # 16 weights (one per layer) used in turn, so each launch reads its weight from HBM
        n, d = SWA["B"], SWA["d"]
        ws_ = [wl.normal((2 * Hkv * D, d), 30 + l, bf, dev, std=d ** -0.5) for l in range(16)]
        x = wl.normal((n, d), 10, bf, dev)
        kb = wl.normal((n, Hkv, D), 12, bf, dev); vb = wl.normal((n, Hkv, D), 13, bf, dev)
        ko = torch.empty_like(kb); vo = torch.empty_like(vb)
        turn = [0]

        def fn():
            turn[0] += 1
            yoco.kv_project_blend(x, ws_[turn[0] % 16], Hkv, D, kb, vb, 0.5, 0.5, k_out=ko, v_out=vo)
        work, unit = 2.0 * Hkv * D * d * 2, "GB/s"
    elif args.case == "swa_decode_layer":
        B, T, Wn = SWA["B"], 4096, SWA["W"]
        k = wl.normal((B, T, Hkv, D), 8, bf, dev); v = wl.normal((B, T, Hkv, D), 9, bf, dev)
        ring = (torch.empty((B, Wn, Hkv, D), dtype=bf, device=dev), torch.empty((B, Wn, Hkv, D), dtype=bf, device=dev),
                torch.empty((B, Wn), dtype=torch.int32, device=dev))
        yoco.swa_prefill(wl.normal((B, T, Hq, D), 7, bf, dev), k, v, Wn, ring=ring)
        q = wl.normal((B, Hq, D), 10, bf, dev); o = torch.empty_like(q)
        kn = wl.normal((B, Hkv, D), 11, bf, dev); vn = wl.normal((B, Hkv, D), 12, bf, dev)
        pos = torch.full((B,), T, dtype=torch.int64, device=dev)
        ws = torch.empty(yoco.swa_decode_workspace_size(B, Wn, Hq, Hkv, D, bf), dtype=torch.uint8, device=dev)
        fn = lambda: yoco.swa_decode(q, kn, vn, pos, ring[0], ring[1], ring[2], Wn, workspace=ws, o=o)
        work, unit = 2.0 * B * Wn * Hkv * D * 2, "GB/s"
    elif args.case == "swa_step_layer":
        B, T, Wn, d = SWA["B"], 4096, SWA["W"], SWA["d"]
        k = wl.normal((B, T, Hkv, D), 8, bf, dev); v = wl.normal((B, T, Hkv, D), 9, bf, dev)
        ring = (torch.empty((B, Wn, Hkv, D), dtype=bf, device=dev), torch.empty((B, Wn, Hkv, D), dtype=bf, device=dev),
                torch.empty((B, Wn), dtype=torch.int32, device=dev))
        yoco.swa_prefill(wl.normal((B, T, Hq, D), 7, bf, dev), k, v, Wn, ring=ring)
        q = wl.normal((B, Hq, D), 10, bf, dev); o = torch.empty_like(q)
        x = wl.normal((B, d), 11, bf, dev)
        w = wl.normal((2 * Hkv * D, d), 12, bf, dev, std=d ** -0.5)
        kb = wl.normal((B, Hkv, D), 13, bf, dev); vb = wl.normal((B, Hkv, D), 14, bf, dev)
        pos = torch.full((B,), T, dtype=torch.int64, device=dev)
        ws = torch.empty(yoco.swa_decode_step_workspace_size(B, Wn, Hq, Hkv, D, bf), dtype=torch.uint8, device=dev)
        fn = lambda: yoco.swa_decode_step(x, w, q, pos, ring[0], ring[1], ring[2], Wn, kb, vb, 0.5, 0.5,
                                          workspace=ws, o=o)
        work, unit = 2.0 * B * Wn * Hkv * D * 2 + 2.0 * Hkv * D * d * 2, "GB/s"
    elif args.case in ("decode_i8_layer", "decode_i8"):
        lens = (wl.ragged_lengths(DEC["B"], DEC["lo"], DEC["hi"], DEC["seed"]) if args.case == "decode_i8_layer"
                else wl.ragged_lengths(16, 16384, 32768, 9))
        starts = torch.cumsum(torch.cat([torch.zeros(1, dtype=torch.int64), lens[:-1]]), 0)
        rows = int(lens.sum())
        kc = wl.normal((rows, Hkv, D), 4, bf, dev); vc = wl.normal((rows, Hkv, D), 5, bf, dev)
        kq, vq = yoco.kv_quantize_i8(kc, vc)
        del kc, vc
        q = wl.normal((DEC["B"], Hq, D), 6, bf, dev); o = torch.empty_like(q)
        ss, sl = starts.to(dev), lens.to(torch.int32).to(dev)
        ws = torch.empty(yoco.cross_decode_workspace_size(DEC["B"], int(lens.max()), Hq, Hkv, D, bf),
                         dtype=torch.uint8, device=dev)
        fn = lambda: yoco.cross_decode_i8(q, kq, vq, Hkv, ss, sl, int(lens.max()), workspace=ws, o=o)
        work, unit = rows * 2.0 * yoco.kv_i8_row_bytes(Hkv, D), "GB/s"
    elif args.case in ("long_prefill", "long_decode"):
        T, C = 1 << 20, 32768
        k = wl.normal((1, T, Hkv, D), 5001, bf, dev); v = wl.normal((1, T, Hkv, D), 5002, bf, dev)
        if args.case == "long_prefill":
            q = wl.normal((1, C, Hq, D), 5003, bf, dev); o = torch.empty_like(q)
            fn = lambda: yoco.cross_prefill(q, k, v, q_pos0=T - C, o=o)
            work, unit = prefill_flops_per_layer(C, Hq, D, T - C), "TFLOP/s"
        else:
            q = wl.normal((1, Hq, D), 5004, bf, dev); o = torch.empty_like(q)
            ss = torch.zeros(1, dtype=torch.int64, device=dev)
            sl = torch.tensor([T], dtype=torch.int32, device=dev)
            ws = torch.empty(yoco.cross_decode_workspace_size(1, T, Hq, Hkv, D, bf), dtype=torch.uint8, device=dev)
            fn = lambda: yoco.cross_decode(q, k[0], v[0], ss, sl, T, workspace=ws, o=o)
            work, unit = T * Hkv * D * 4.0, "GB/s"
    elif args.case in ("gret", "gret1"):
        B, T, H = (GRET["B"] if args.case == "gret" else 1), GRET["T"], GRET["H"]
        q = wl.normal((B, T, H, D), 14, bf, dev); k = wl.normal((B, T, H, D), 15, bf, dev)
        v = wl.normal((B, T, H, D), 16, bf, dev); g = wl.normal((B, T, H), 17, torch.float32, dev) + 3.0
        o = torch.empty_like(q)
        fn = lambda: yoco.gret_prefill(q, k, v, g, GRET["tau"], o=o)
        work, unit = gret_flops(B, T, H, D), "TFLOP/s"
    elif args.case == "gret_decode":
        B, H = GRET["B_dec"], GRET["H"]
        q = wl.normal((B, H, D), 18, bf, dev); k = wl.normal((B, H, D), 19, bf, dev)
        v = wl.normal((B, H, D), 20, bf, dev); g = wl.normal((B, H), 21, torch.float32, dev) + 3.0
        st = torch.zeros((B, H, D, D), dtype=torch.float32, device=dev)
        o = torch.empty_like(q)
        fn = lambda: yoco.gret_decode(q, k, v, g, GRET["tau"], st, o=o)
        work, unit = B * H * D * D * 4.0 * 2, "GB/s"
    else:
        n, d = 32768, 4096
        x = wl.normal((n, d), 10, bf, dev); w = wl.normal((2 * Hkv * D, d), 11, bf, dev, std=d ** -0.5)
        kb = wl.normal((n, Hkv, D), 12, bf, dev); vb = wl.normal((n, Hkv, D), 13, bf, dev)
        ko = torch.empty_like(kb); vo = torch.empty_like(vb)
        fn = lambda: yoco.kv_project_blend(x, w, Hkv, D, kb, vb, 0.5, 0.5, k_out=ko, v_out=vo)
        work, unit = 2.0 * n * d * 2 * Hkv * D, "TFLOP/s"
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    times = []
    for it in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(); fn(); e1.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            times.append(e0.elapsed_time(e1))
    ms = statistics.mean(times)
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"case": args.case, "ms": ms, "rate": rate, "unit": unit,
                      "status": yoco.device_status()}), flush=True)


# chunk-parallel prefill across ranks: per rank one chunk of one long sequence
CP = dict(Tc=16384, Hq=32, Hkv=8, D=128, W=1024, self_layers=4, cross_layers=4)


class _Clock:
    """Device time on CUDA (events on the current stream), host time on CPU."""

    def __init__(self, device):
        self.cuda = device.type == "cuda"

    def mark(self):
        import torch
        if self.cuda:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            return e
        return time.perf_counter()

    def ms(self, a, b):
        return a.elapsed_time(b) if self.cuda else (b - a) * 1e3


def chunk_parallel_measure(comm, ops, device, dtype, steps, warmup, Tc, Hq, Hkv, D, W, self_layers,
                           cross_layers):
    """Chunk-parallel prefill of one sequence of world * Tc tokens ("You Only
    Cache Once", paperlayer summary, Appendix A): rank r holds positions
    [r Tc, (r + 1) Tc).  A step runs, on every rank, `self_layers` sliding-
    window layers (each exchanging a window - 1 row halo with the neighbour
    rank), ONE all-gather of the global K/V, then `cross_layers` causal cross
    layers of the rank's rows over the gathered prefix.  Inputs are seeded per
    rank and layer and resident before timing.  Returns this rank's report
    (times, FLOPs) and the last step's outputs (last self layer, last cross
    layer)."""
    import torch
    import workloads as wl
    from shared_kv_decoder_b200 import chunk_parallel as cp
    r, world = comm.rank, comm.world
    s0 = r * Tc
    gen = lambda shape, seed: wl.normal(shape, seed, dtype, device)
    qs = [gen((1, Tc, Hq, D), 6000 + 100 * l + r) for l in range(self_layers)]
    ks = [gen((1, Tc, Hkv, D), 6010 + 100 * l + r) for l in range(self_layers)]
    vs = [gen((1, Tc, Hkv, D), 6020 + 100 * l + r) for l in range(self_layers)]
    kg = gen((1, Tc, Hkv, D), 6030 + r)
    vg = gen((1, Tc, Hkv, D), 6040 + r)
    qc = [gen((1, Tc, Hq, D), 6050 + 100 * l + r) for l in range(cross_layers)]
    clk = _Clock(device)
    t_self, t_gather, t_cross = [], [], []
    out = None
    for it in range(warmup + steps):
        m0 = clk.mark()
        for l in range(self_layers):
            o_s = cp.swa_chunk(qs[l], ks[l], vs[l], W, comm, ops)
        m1 = clk.mark()
        k_all, v_all = cp.gather_global_kv(kg, vg, comm)
        m2 = clk.mark()
        for l in range(cross_layers):
            o_c = cp.cross_chunk(qc[l], k_all, v_all, s0, ops)
        m3 = clk.mark()
        if device.type == "cuda":
            torch.cuda.synchronize()
        if it >= warmup:
            t_self.append(clk.ms(m0, m1))
            t_gather.append(clk.ms(m1, m2))
            t_cross.append(clk.ms(m2, m3))
        out = (o_s, o_c)
    swa_fl = self_layers * 4.0 * Hq * D * sum(min(s0 + i + 1, W) for i in range(Tc))
    cross_fl = cross_layers * 4.0 * Hq * D * (Tc * s0 + Tc * (Tc + 1) / 2.0)
    rep = {"rank": r, "ms_self": sum(t_self) / steps, "ms_gather": sum(t_gather) / steps,
           "ms_cross": sum(t_cross) / steps, "flops_self": swa_fl, "flops_cross": cross_fl,
           "gather_bytes": 2.0 * world * Tc * Hkv * D * torch.tensor([], dtype=dtype).element_size()}
    rep["ms_step"] = rep["ms_self"] + rep["ms_gather"] + rep["ms_cross"]
    return rep, out


def run_chunk_parallel(args):
    """bench.py --chunk-parallel: the chunk-parallel prefill over NCCL, one
    rank per GPU (torchrun); prints one JSON line from rank 0 with the job's
    TFLOP/s (all ranks' FLOPs over the slowest rank's step time) and each
    rank's times, the all-gather's share among them."""
    import datetime
    import torch
    import torch.distributed as dist
    import shared_kv_decoder_b200 as yoco
    from shared_kv_decoder_b200 import chunk_parallel as cp
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29511")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), world_size=world,
                            rank=int(os.environ.get("RANK", "0")), device_id=dev)
    yoco.load()
    rep, _ = chunk_parallel_measure(cp.DistComm(), cp.KernelOps, dev, torch.bfloat16, args.steps,
                                    args.warmup, **CP)
    st = yoco.device_status()
    reps = [None] * world
    dist.all_gather_object(reps, rep)
    t = torch.tensor([float(st)], device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    worst = int(t.item())
    dist.barrier()
    dist.destroy_process_group()
    if worst != yoco.OK:
        sys.stderr.write(f"bench: device status {worst}; no number is reported\n")
        sys.exit(3)
    if int(os.environ.get("RANK", "0")) != 0:
        return
    step = max(x["ms_step"] for x in reps)
    flops = sum(x["flops_self"] + x["flops_cross"] for x in reps)
    out = {"metric": "chunk-parallel prefill TFLOP/s (self-decoder halo + one global-KV all-gather)",
           "value": flops / (step * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": step, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"one sequence of {world} x {CP['Tc']} tokens, one chunk per rank; "
                                  f"{CP['self_layers']} SWA layers (window {CP['W']}) + {CP['cross_layers']} "
                                  "cross layers, 32q/8kv D=128",
                      "parallelism": f"chunk-parallel over {world} ranks"},
           "gather_share": max(x["ms_gather"] for x in reps) / step,
           "ranks": reps, "device_status": worst}
    print(json.dumps(out), flush=True)


class DeviceStatusError(RuntimeError):
    pass


def check_device_status(where, dev):
    """Read (and clear) the library's device status word after a timed block;
    any non-OK status on any rank fails the run (every rank takes the same
    collective step here, on the error path too)."""
    import shared_kv_decoder_b200 as yoco
    st = yoco.device_status()
    worst = int(reduce_max_over_ranks([st], dev)[0])
    if worst != yoco.OK:
        raise DeviceStatusError(f"{where}: device status {worst} ({'this rank' if st else 'another rank'})")
    return st


def main():
    args = parse_args()
    if args.case:
        run_case(args)
        return
    if args.chunk_parallel:
        run_chunk_parallel(args)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import shared_kv_decoder_b200 as yoco
    yoco.load()
    try:
        out = measure(args, world, rank, local, dev)
    except DeviceStatusError as e:
        sys.stderr.write(f"bench: {e}; no number is reported\n")
        if world > 1:
            dist.destroy_process_group()
        sys.exit(3)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def measure(args, world, rank, local, dev):
    import torch
    import torch.distributed as dist
    import shared_kv_decoder_b200 as yoco
    peaks = load_peaks()
    W = make_workload(dev)
    graph_launches = capture_self_decoder_decode(W)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        W["flush"].zero_()
        run_step(W)
    torch.cuda.synchronize()
    check_device_status("warm-up steps", dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    launches0 = yoco.launch_count()
    evs = []
    for _ in range(args.steps):
        W["flush"].zero_()
        ev = new_events()
        ev["step"][0].record()
        run_step(W, ev)
        ev["step"][1].record()
        evs.append(ev)
    torch.cuda.synchronize()
    # kernels launched from the library's host calls, plus those each replay
    # of the self-decoder's decode graph launched (counted once at capture)
    launches = yoco.launch_count() - launches0 + args.steps * graph_launches
    clk = clocks.stop()
    status = check_device_status("timed steps", dev)
    if world > 1:
        dist.barrier()

    def pair(ev, name, i=0):
        return ev[name][i].elapsed_time(ev[name][i + 1])

    step_ms = [pair(e, "step") for e in evs]
    pre_l = [pair(e, "prefill_l", 2 * l) for e in evs for l in range(P["layers"])]
    dec_l = [pair(e, "decode_l", 2 * l) for e in evs for l in range(DEC["layers"])]
    pre_ms = [sum(pair(e, "prefill_l", 2 * l) for l in range(P["layers"])) for e in evs]
    dec_ms = [pair(e, "decode") for e in evs]
    L4, S4 = SWA["layers"], SWA["steps"]
    swa_pre_ms = [pair(e, "swa") for e in evs]
    swa_proj_l = [pair(e, "swa_proj", 2 * l) for e in evs for l in range(L4)]
    swa_att_l = [pair(e, "swa_att", 2 * l) for e in evs for l in range(L4)]
    swa_dec_ms = [pair(e, "swa_dec") for e in evs]
    gkv_ms = [pair(e, "gkv") for e in evs]

    mx = reduce_max_over_ranks([sum(step_ms), sum(pre_ms), sum(dec_ms), sum(swa_pre_ms), sum(swa_dec_ms)], dev)
    tot = {"step": mx[0], "pre": mx[1], "dec": mx[2], "swa_pre": mx[3], "swa_dec": mx[4]}

    f_layer = prefill_flops_per_layer(P["T"], P["Hq"], P["D"])
    value = world * args.steps * P["layers"] * f_layer / (tot["pre"] * 1e-3) / 1e12
    dec_bytes_layer = float(W["lens"].sum()) * DEC["Hkv"] * DEC["D"] * 2 * 2
    dec_tok_s = world * args.steps * DEC["B"] / (tot["dec"] * 1e-3)
    dec_gbs_layer = dec_bytes_layer / (statistics.mean(dec_l) * 1e-3) / 1e9
    pre_tflops_launch = f_layer / (statistics.mean(pre_l) * 1e-3) / 1e12
    B4, T4, W4, Hkv4, D4, d4, Hq4 = (SWA[k] for k in ("B", "T", "W", "Hkv", "D", "d", "Hq"))
    n4 = B4 * T4
    swa_proj_fl = 2.0 * n4 * d4 * 2 * Hkv4 * D4
    swa_att_fl = B4 * prefill_flops_per_layer(T4, Hq4, D4, 0, W4)
    swa_tile_fl = swa_tile_flops_per_layer(B4, T4, Hq4, D4, W4)
    swa_att_tf = swa_att_fl / (statistics.mean(swa_att_l) * 1e-3) / 1e12
    # one decode layer-step reads the layer's ring (K and V, B x W rows) and
    # its W_kv, reads the 4 new tokens' x, q and the bottom layer's new K/V,
    # and writes the new K/V (into the ring) and o
    ring_bytes = 2.0 * B4 * W4 * Hkv4 * D4 * 2
    wkv_bytes = 2.0 * Hkv4 * D4 * d4 * 2
    small_bytes = B4 * (d4 + Hq4 * D4 * 2 + 2 * Hkv4 * D4 * 3) * 2.0
    layer_step_bytes = ring_bytes + wkv_bytes + small_bytes
    layer_step_ms = tot["swa_dec"] / (args.steps * S4 * L4)
    swa_dec_gbs = layer_step_bytes / (layer_step_ms * 1e-3) / 1e9
    gkv_fl = 2.0 * P["T"] * P["d"] * 2 * P["Hkv"] * P["D"]

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot["step"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "model": "YOCO attention core (synthetic, random init)",
                   "global_batch": world, "seq_len": P["T"], "parallelism": "replicas",
                   "l2": "every part's inputs exceed L2; 256 MB rewritten between steps"},
        "decode": {"tokens_per_s": dec_tok_s, "hbm_gbs": dec_gbs_layer,
                   "frac_hbm": dec_gbs_layer / peaks["hbm"], "ms_per_decode_step": tot["dec"] / args.steps,
                   "bytes_per_layer": dec_bytes_layer},
        "swa": {"shape": f"B={B4} T={T4} window={W4} 32q/8kv D=128 d={d4}, {L4} layers, w_l ~ U(0,1)",
                "prefill_ms": tot["swa_pre"] / args.steps,
                "prefill_tokens_per_s": world * args.steps * n4 / (tot["swa_pre"] * 1e-3),
                "attention_ms_per_layer": statistics.mean(swa_att_l),
                "attention_tflops": swa_att_tf,
                "attention_tflops_tile": swa_tile_fl / (statistics.mean(swa_att_l) * 1e-3) / 1e12,
                "attention_flops_per_layer": swa_att_fl, "attention_tile_flops_per_layer": swa_tile_fl,
                "projection_ms_per_layer": statistics.mean(swa_proj_l),
                "projection_tflops": swa_proj_fl / (statistics.mean(swa_proj_l) * 1e-3) / 1e12,
                "decode_steps": S4, "decode_ms": tot["swa_dec"] / args.steps,
                "decode_tokens_per_s": world * args.steps * S4 * B4 / (tot["swa_dec"] * 1e-3),
                "decode_ms_per_layer_step": layer_step_ms, "decode_hbm_gbs": swa_dec_gbs,
                "decode_bytes_per_layer_step": layer_step_bytes,
                "note": "attention times include the ring fill; decode = 256 steps x 16 layers from one "
                        "CUDA graph, each layer-step = one yoco_swa_decode_step call: the 4 new tokens' "
                        "projection with the blend, then the clustered window decode (window attention, "
                        "merge with the new token, ring write)"},
        "gkv": {"ms": statistics.mean(gkv_ms), "tflops": gkv_fl / (statistics.mean(gkv_ms) * 1e-3) / 1e12},
        "roofline": {"kernel": "cross prefill (yoco_cross_prefill)", "bound": "tensor",
                     "achieved": pre_tflops_launch, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                     "frac": pre_tflops_launch / peaks["bf16_sus"], "traffic": traffic("prefill"),
                     "peak_src": f"{peaks['src']} bf16 sustained"},
        "roofline_decode": {"kernel": "cross decode (yoco_cross_decode)", "bound": "hbm",
                            "achieved": dec_gbs_layer, "peak": peaks["hbm"], "unit": "GB/s",
                            "frac": dec_gbs_layer / peaks["hbm"], "traffic": traffic("decode"),
                            "peak_src": f"{peaks['src']} hbm"},
        "roofline_swa_prefill": {"kernel": "sliding-window prefill (yoco_swa_prefill)", "bound": "tensor",
                                 "achieved": swa_att_tf, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                                 "frac": swa_att_tf / peaks["bf16_sus"], "traffic": traffic("swa_prefill"),
                                 "peak_src": f"{peaks['src']} bf16 sustained"},
        "roofline_swa_decode": {"kernel": "sliding-window decode layer-step (yoco_swa_decode_step: projection + window decode)",
                                "bound": "hbm", "achieved": swa_dec_gbs, "peak": peaks["hbm"], "unit": "GB/s",
                                "frac": swa_dec_gbs / peaks["hbm"], "traffic": traffic("swa_decode"),
                                "peak_src": f"{peaks['src']} hbm"},
        "gpu_launches": launches,
        "clocks": clk,
        "device_status": status,
    }
    # the self-decoder's inputs are not needed by the blocks below
    W["swa_graph"].reset()
    for k_ in ("x4", "q4", "x4d", "q4d", "k1", "v1", "k4", "v4", "o4"):
        W.pop(k_, None)
    torch.cuda.empty_cache()
    if not args.no_e2e:
        times, h2d, d2h = e2e_prefill(W, args.steps, args.warmup)
        check_device_status("e2e", dev)
        e2e_ms = reduce_max_over_ranks([sum(times)], dev)[0]
        out["e2e"] = {"value": world * len(times) * P["layers"] * f_layer / (e2e_ms * 1e-3) / 1e12,
                      "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if not args.no_long:
        out["long_context"] = long_context(W, peaks)
        check_device_status("long context", dev)
        torch.cuda.empty_cache()
    if not args.no_early_exit:
        out["early_exit"] = early_exit(W, 3)
        check_device_status("early exit", dev)
        out["gret"] = gret_layer(W, 3)
        check_device_status("gated retention", dev)
        out["decode_i8"] = decode_i8_step(W, 3)
        check_device_status("8-bit decode", dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(W, args.cpu_seconds)
    return out


if __name__ == "__main__":
    main()

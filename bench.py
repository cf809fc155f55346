"""Benchmark of one sparse spatial/temporal attention layer on B200.

A step is one pass of the whole hot path over one layer's inputs:
    profile heads, while a side stream makes token-major copies of q, k, v
    (every head) -> block-sparse attention in which temporal heads read the
    copies and write their output back frame-major (svg_sparse_attn_fused).
The permutation kernel is also timed on its own beside the step, and the
unfused layer (permute -> attention -> permute back) for comparison.
Workload (default): the largest layer, HunyuanVideo-720p-shaped, B=1 H=24
N=118800 (33 frames x 45x80 tokens) d=128 bf16, band |f - f'| <= 2, synthetic
biased-Gaussian q/k/v, 64 sampled queries.  --config picks another layer;
--config wan720 times the calibrated Wan 2.1 720p layer (per-head lists built
from four calibration inputs, the build timed separately).

Metric: effective TFLOPS of the layer = sum over heads of 4 * d * (query-key
pairs inside kept 128x128 tiles, ragged tiles counted by their valid rows and
columns) / step time.  tokens/s = B * N / step time is reported beside it.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
        python bench.py --impl reference ...    (the float64 CPU oracle)
Multi-GPU (torchrun): by default the heads of one layer are split into
contiguous ranges, one per rank (--shard heads; strong scaling: the whole
layer's work over the slowest rank's time); --shard replicas runs an
independent layer per rank instead (weak scaling).  No collective touches the
data path either way.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import svg_inputs as si  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "effective TFLOPS and tokens/s of sparse 3D attention per layer; % of bf16 TC peak"


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (read + write) of one attention launch, from ncu captures of the
# kernel built from the sources whose sha256 is recorded here: a 4-head slice
# of each layer, scaled by the head count, since each head's q, k, v are read
# and its o written once.  HunyuanVideo 720p: heads 2-5 (two spatial, two
# temporal), 370402048 + 101969152 bytes, x 24 / 4.  Wan 2.1 720p with the
# calibrated lists and the pairing order: heads 14-17 (two of each type),
# 243936000 + 59193600 bytes, x 40 / 4.  Reported only while the sources
# still match.
ATTN_SOURCES = ("attn_sm100.cu", "sm100.cuh", "attn.cuh", "common.cuh")
_ATTN_SHA = "3e36e93d3b8ea8d5059f4b6b6643b86a3d2c97b441c1e4d23108dc558d01b64e"
ATTN_TRAFFIC = {"hunyuan720": {"sha256": _ATTN_SHA, "bytes": (370402048 + 101969152) * 24 // 4},
                "wan720": {"sha256": _ATTN_SHA, "bytes": (243936000 + 59193600) * 40 // 4}}


def attn_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_video_svg_b200", "csrc")
    for name in ATTN_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic(workload):
    rec = ATTN_TRAFFIC.get(workload)
    if rec is None or attn_sources_sha256() != rec["sha256"]:
        return None
    return rec["bytes"]


def host_chunk(bh, target=4):
    """Heads per chunk of the host-streamed layer: the largest divisor of the
    rank's head count not above `target`."""
    return max(c for c in range(1, min(bh, target) + 1) if bh % c == 0)


def rank_seed(wl, rank):
    """With --shard replicas each rank runs its own independent layer (weak
    scaling) on this input seed."""
    return wl.seed + rank


def shard_heads(H, world, rank):
    """Contiguous head range of one rank when the heads of one layer are
    split over `world` GPUs: the first H mod world ranks take one head more."""
    base, extra = divmod(H, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def rank_heads(args, wl, rank, world):
    """(heads, sharded, input seed) of this rank: a --heads range (one GPU,
    small profiling captures), the rank's contiguous share of the layer's
    heads (--shard heads), or the whole layer (one GPU, or --shard replicas
    with an independent input per rank)."""
    if args.heads is not None:
        if world > 1:
            raise SystemExit("--heads runs on one GPU")
        a, b = (int(x) for x in args.heads.split(":"))
        if not 0 <= a < b <= wl.H:
            raise SystemExit(f"--heads {args.heads} outside 0:{wl.H}")
        return range(a, b), False, wl.seed
    if args.shard == "heads" and world > 1:
        if wl.H < world:
            raise SystemExit(f"{wl.H} heads cannot be split over {world} GPUs")
        return shard_heads(wl.H, world, rank), True, wl.seed
    return range(wl.H), False, rank_seed(wl, rank)


def sum_over_ranks(values, world, device):
    """Element-wise sum of per-rank values (every rank gets the result)."""
    if world == 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if world == 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate(job_flops, total_ms, steps, job_tokens):
    """Whole-job throughput: the work of all ranks (job_flops, job_tokens per
    step) over the slowest rank's time per step (total_ms over `steps`).
    Returns (TFLOPS, tokens/s, ms per step)."""
    ms = total_ms / steps
    return job_flops / (ms * 1e-3) / 1e12, job_tokens / (ms * 1e-3), ms


def workload_config(wl):
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "frames": wl.F, "tokens_per_frame": wl.P,
            "N": wl.N, "d": wl.d, "sampled_queries": wl.S, "spatial_width": wl.width}


def kept_pairs(indptr, indices, N, T=128):
    """Query-key pairs inside the kept tiles of one list (ragged tiles count
    their valid rows and columns)."""
    nb = len(indptr) - 1
    sizes = np.minimum(T, N - np.arange(nb) * T).astype(np.int64)
    total = 0
    for i in range(nb):
        total += int(sizes[i]) * int(sizes[indices[indptr[i]:indptr[i + 1]]].sum())
    return total


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"svg_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return parse_clock_samples(lines)


def parse_clock_samples(lines):
    """Summary of `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,
    noheader,nounits` lines: median SM clock, max SM clock and the throttle
    reasons seen Active in any sample."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

    def num(x):
        try:
            return float(x)
        except ValueError:
            return None
    sm = [num(r[1]) for r in rows if num(r[1]) is not None]
    mx = [num(r[2]) for r in rows if num(r[2]) is not None]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
            "samples": len(rows)}


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import sparse_attention_video_svg_b200 as svg

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = si.WORKLOADS[args.config]
    if wl.kind != "profiled":
        raise SystemExit(f"run_ours times profiled layers; {wl.name} is {wl.kind}")
    heads, sharded, seed = rank_heads(args, wl, rank, world)
    q, k, v, types = si.generate(wl, seed=seed, heads=heads)
    Hl = len(heads)
    idx = si.sample_queries(wl, seed=wl.seed)
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v)]
    del q, k, v
    qd, kd, vd = (h.to(dev) for h in host)
    idx_d = torch.from_numpy(idx).to(dev)
    F, P, w, N, d = wl.F, wl.P, wl.width, wl.N, wl.d
    lists = svg.geometric_lists(F, P, w, N, device=dev)
    bufs = svg.LayerBuffers(qd, wl.S)
    stream = torch.cuda.current_stream()

    # effective work from the modes the layer picks (deterministic for the input)
    _, mode, _ = svg.svg_layer(qd, kd, vd, F, P, w, idx_d, lists, bufs)
    torch.cuda.synchronize()
    modes = mode.cpu().numpy()
    nb = svg.n_tiles(N)
    ip = lists.indptr.cpu().numpy().reshape(3, nb + 1)
    ix = lists.indices.cpu().numpy()
    pairs = {kind: kept_pairs(ip[kind] - ip[kind][0], ix[ip[kind][0]:ip[kind][-1]], N)
             for kind in (0, 1)}
    flops = float(sum(4 * d * pairs[int(m)] for m in modes))   # per layer, this rank
    kept_frac = {kind: pairs[kind] / float(N * N) for kind in pairs}

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    K, W = args.steps, args.warmup

    def step():
        return svg.svg_layer(qd, kd, vd, F, P, w, idx_d, lists, bufs)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(K)]
    side = bufs.side
    for i in range(K):
        flush.fill_(i & 0xff)
        s0, p0, a0, s1 = ev[i]
        s0.record(stream)
        # the schedule svg_layer runs: V exponents on the side stream beside
        # the profiling, then token-major copies of the temporal heads
        side.wait_event(s0)
        svg.svg_v_exponents(vd, out=bufs.vexp, stream=side)
        side_done = torch.cuda.Event()
        side_done.record(side)
        svg.svg_profile_heads(qd, kd, vd, F, P, w, idx_d, mse_out=bufs.mse, mode_out=bufs.mode,
                              workspace=bufs.ws)
        p0.record(stream)
        for x, y in ((qd, bufs.qp), (kd, bufs.kp), (vd, bufs.vp)):
            svg.svg_permute_temporal_heads(x, F, P, bufs.mode, out=y)
        stream.wait_event(side_done)
        a0.record(stream)
        svg.svg_sparse_attn_fused(qd, kd, vd, F, P, bufs.mode, lists,
                                  layout=svg._lib.SVG_FUSE_OUTPUT,
                                  copies=(bufs.qp, bufs.kp, bufs.vp), out=bufs.o,
                                  v_exp=bufs.vexp)
        s1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    attn_ms = [e[2].elapsed_time(e[3]) for e in ev]
    prof_ms = [e[0].elapsed_time(e[1]) for e in ev]
    fwd_perm_ms = [e[1].elapsed_time(e[2]) for e in ev]  # temporal heads' copies after profiling
    total_ms = float(sum(step_ms))
    attn_avg = float(sum(attn_ms) / K)
    prof_avg = float(sum(prof_ms) / K)
    fwd_perm_avg = float(sum(fwd_perm_ms) / K)

    # the permutation kernels on their own (one token-major pass of q over
    # every head, L2 flushed before each) and the unfused layer
    tmp = [torch.empty_like(qd) for _ in range(4)]
    perm_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    unf_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    for i in range(K):
        flush.fill_(i & 0xff)
        perm_ev[i][0].record(stream)
        svg.svg_permute_token_major(qd, F, P, None, out=tmp[0])
        perm_ev[i][1].record(stream)
    for i in range(K):
        flush.fill_(i & 0xff)
        unf_ev[i][0].record(stream)
        svg.svg_profile_heads(qd, kd, vd, F, P, w, idx_d, mse_out=bufs.mse, mode_out=bufs.mode,
                              workspace=bufs.ws)
        for x, y in zip((qd, kd, vd), tmp):
            svg.svg_permute_token_major(x, F, P, bufs.mode, out=y)
        svg.svg_sparse_attn(tmp[0], tmp[1], tmp[2], bufs.mode, lists, out=tmp[3])
        svg.svg_permute_frame_major(tmp[3], F, P, bufs.mode, out=bufs.o)
        unf_ev[i][1].record(stream)
    torch.cuda.synchronize()
    perm_avg = float(sum(e[0].elapsed_time(e[1]) for e in perm_ev) / K)
    unf_avg = float(sum(e[0].elapsed_time(e[1]) for e in unf_ev) / K)
    del tmp

    # mask encodings of the layer's three lists ([CAL] 3.3): skip list and bitmap
    rows = 3 * nb
    ix_host = lists.indices.cpu().numpy()
    segs = [ix_host[ip[kk][r]:ip[kk][r + 1]] for kk in range(3) for r in range(nb)]
    ip_all = torch.from_numpy(np.cumsum([0] + [len(x) for x in segs]).astype(np.int32)).to(dev)
    ix_all = torch.from_numpy(np.concatenate(segs).astype(np.int32)).to(dev)
    enc = {}
    for kind, fn in (("intervals", lambda: svg.svg_lists_to_intervals(ip_all, ix_all, nb)),
                     ("bitmap", lambda: svg.svg_lists_to_bitmap(ip_all, ix_all, nb))):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            res = fn()
        e1.record(stream)
        torch.cuda.synchronize()
        enc[kind] = (e0.elapsed_time(e1) / 10 * 1e3, res)
    iptr_e, starts_e, _ = enc["intervals"][1]
    encodings = {"rows": rows, "csr_bytes": int(4 * (rows + 1 + ix_all.numel())),
                 "intervals_bytes": int(4 * (rows + 1 + 2 * starts_e.numel())),
                 "bitmap_bytes": int(enc["bitmap"][1].numel() * 4),
                 "int32_mask_bytes": int(rows * nb * 4),
                 "intervals_us": round(enc["intervals"][0], 2),
                 "bitmap_us": round(enc["bitmap"][0], 2),
                 "note": "host-synchronising size query included in intervals_us"}

    # QK-Norm + RoPE of q and k, writing the token-major copies in the same
    # pass, on its own; then the layer with it in front (the pass makes the
    # copies of q and k, only v is permuted on the side stream) against the
    # pass followed by the plain layer (which reorders q and k again)
    gq, gk = si.qk_norm_weights(wl)
    cos, sin = si.rope_tables(wl)
    to_dev = lambda a: torch.from_numpy(a).to(dev)
    qk = svg.QKTransform(to_dev(gq), to_dev(gk), 1e-6, to_dev(cos), to_dev(sin))
    qk_bufs = svg.LayerBuffers(qd, wl.S, qk=True)
    qn, kn = torch.empty_like(qd), torch.empty_like(kd)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        evs = []
        for i in range(K):
            flush.fill_(i & 0xff)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        return float(sum(a.elapsed_time(b) for a, b in evs) / K)

    qk_ms = timed(lambda: svg.svg_qk_norm_rope(qd, kd, qk, out=(qn, kn),
                                               tm_out=(qk_bufs.qp, qk_bufs.kp), frames=F,
                                               tokens_per_frame=P))
    qk_layer_ms = timed(lambda: svg.svg_layer(qd, kd, vd, F, P, w, idx_d, lists, qk_bufs, qk=qk))
    qk_modes = qk_bufs.mode.cpu().numpy()  # QK-Norm changes what profiling picks
    qk_then_layer_ms = timed(lambda: (svg.svg_qk_norm_rope(qd, kd, qk, out=(qn, kn)),
                                      svg.svg_layer(qn, kn, vd, F, P, w, idx_d, lists, bufs)))
    del qk_bufs, qn, kn

    # spatial-repetition heads ([CAL] 3.2): the row-similarity test on one
    # frame of every head, and the layer with every spatial head taken as
    # repeating (anchor tiles only, then the broadcast)
    ph, pw = wl.ph, wl.pw
    mid = torch.tensor([F // 2], dtype=torch.int32, device=dev)
    rs_ws = torch.empty(max(256, svg._lib.lib.svg_row_similarity_workspace_size(
        svg._lib.SVG_BF16, wl.B, Hl, ph, pw, 1)), dtype=torch.uint8, device=dev)
    sims = svg.svg_row_similarity(qd, kd, F, ph, pw, mid, workspace=rs_ws)
    rs_ms = timed(lambda: svg.svg_row_similarity(qd, kd, F, ph, pw, mid, out=sims,
                                                 workspace=rs_ws))
    sims_h = sims.cpu().numpy()
    rep_all = torch.from_numpy((modes == 0).astype(np.int32)).to(dev)  # every spatial head
    modes_d = torch.from_numpy(modes.astype(np.int32)).to(dev)  # this layer's profiled modes
    alists, ids = svg.svg_anchor_lists(lists, N, F, ph, pw, modes_d, rep_all,
                                       skip_list=svg._lib.SVG_MODE_TEMPORAL)
    rep_attn_ms = timed(lambda: svg.svg_sparse_attn_fused(
        qd, kd, vd, F, P, ids, alists, layout=svg._lib.SVG_FUSE_OUTPUT,
        copies=(bufs.qp, bufs.kp, bufs.vp), out=bufs.o))
    rep_layer_ms = timed(lambda: svg.svg_layer(qd, kd, vd, F, P, w, idx_d, lists, bufs,
                                               repeat=rep_all, frame_shape=(ph, pw)))
    aip = alists.indptr.cpu().numpy().reshape(6, nb + 1)
    aix = alists.indices.cpu().numpy()
    anchor_pairs = kept_pairs(aip[3] - aip[3][0], aix[aip[3][0]:aip[3][-1]], N)
    rep_attn_pairs_ms = timed(lambda: svg.svg_sparse_attn_fused(
        qd, kd, vd, F, P, ids, alists._replace(tile_order=None),
        layout=svg._lib.SVG_FUSE_OUTPUT, copies=(bufs.qp, bufs.kp, bufs.vp), out=bufs.o))

    # the fixed-scratch profiling entry point on the same inputs, alone
    noalloc_ms = timed(lambda: svg.svg_profile_heads_noalloc(
        qd, kd, vd, F, P, w, idx_d, mse_out=bufs.mse, mode_out=bufs.mode))

    # end to end through the public API with host buffers: q, k, v from pinned
    # host memory, o and the modes back, every step; chunks of heads stream
    # through two device slots so the copies overlap the layer
    out_host = torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory()
    mode_host = torch.empty(modes.shape, dtype=torch.int32).pin_memory()
    hc = host_chunk(wl.B * Hl)
    hbufs = svg.HostLayerBuffers(hc, N, d, wl.S, dev)
    for _ in range(2):
        svg.svg_layer_from_host(*host, F, P, w, idx_d, lists, out=out_host, mode_out=mode_host,
                                heads_per_chunk=hc, buffers=hbufs)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        svg.svg_layer_from_host(*host, F, P, w, idx_d, lists, out=out_host, mode_out=mode_host,
                                heads_per_chunk=hc, buffers=hbufs)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    del hbufs

    (total_ms, e2e_ms, attn_avg, prof_avg, perm_avg, unf_avg, fwd_perm_avg, qk_ms, qk_layer_ms,
     qk_then_layer_ms, rs_ms, rep_attn_ms, rep_layer_ms, rep_attn_pairs_ms,
     noalloc_avg) = max_over_ranks(
        [total_ms, e2e_ms, attn_avg, prof_avg, perm_avg, unf_avg, fwd_perm_avg, qk_ms,
         qk_layer_ms, qk_then_layer_ms, rs_ms, rep_attn_ms, rep_layer_ms, rep_attn_pairs_ms,
         noalloc_ms], world, dev)
    h2d = sum(h.numel() * 2 for h in host)
    d2h = out_host.numel() * 2 + mode_host.numel() * 4
    # the job's work per step: every rank's heads (one layer split over the
    # ranks, or one layer per rank)
    job_flops, job_h2d, job_d2h, n_spatial, n_temporal = sum_over_ranks(
        [flops, h2d, d2h, int((modes == 0).sum()), int((modes == 1).sum())], world, dev)
    job_tokens = wl.B * N * (1 if sharded else world)
    if rank != 0:
        return None

    peaks, src = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    value, tokens_s, step_ms_avg = aggregate(job_flops, total_ms, K, job_tokens)
    e2e_value, _, e2e_step_ms = aggregate(job_flops, e2e_ms, K, job_tokens)
    # the attention kernel of the slowest rank against its own work
    attn_tf = flops / (attn_avg * 1e-3) / 1e12
    hbm_gbs = float(peaks["hbm_gbs"])
    elems = wl.B * Hl * N * d
    perm_bytes = 2 * elems * 2      # one tensor read and written once
    prof_bytes = 2 * elems * 2      # K and V streamed once
    # q, k read once; q, k written frame-major and token-major; cos, sin once
    qk_bytes = 6 * elems * 2 + 2 * N * (d // 2) * 4
    # profile partial, merge, finalize; 3 permutes; V exponents (max, finalize);
    # attention (output reordering fused)
    launches_per_step = 3 + 3 + 2 + 1
    if sharded:
        parallelism = (f"heads of one layer split over {world} GPUs "
                       f"(contiguous ranges, rank 0 heads {heads.start}-{heads.stop - 1})")
    else:
        parallelism = f"independent layer per GPU x{world}" if world > 1 else "1 GPU"
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(step_ms_avg, 5),
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded biased-Gaussian q/k/v, no model weights)",
        "config": {**workload_config(wl),
                   **({"heads_subset": f"{heads.start}:{heads.stop}"}
                      if args.heads is not None else {}),
                   "modes": {"spatial": int(n_spatial), "temporal": int(n_temporal)},
                   "kept_fraction": {"spatial": round(kept_frac[0], 5),
                                     "temporal": round(kept_frac[1], 5)},
                   "l2": "flushed (256 MB write) before every timed step",
                   "parallelism": parallelism},
        "tokens_per_s": round(tokens_s, 1),
        "pct_of_bf16_peak": round(100 * value / world / peak_tf, 2),
        "attention_only": {"ms": round(attn_avg, 5), "effective_tflops": round(attn_tf, 3),
                           "kernel": "svg_sparse_attn_fused (copies, output fused)"},
        "temporal_copies_ms": round(fwd_perm_avg, 5),
        "mask_encodings": encodings,
        "unfused_layer_ms": round(unf_avg, 5),
        # the permutation kernel alone: one [B,H,N,d] tensor, every head
        # reordered, 2 * B*H*N*d * 2 bytes, L2 flushed before each launch
        "permute": {"ms": round(perm_avg, 5),
                    "gbs": round(perm_bytes / (perm_avg * 1e-3) / 1e9, 1),
                    "frac_of_hbm": round(perm_bytes / (perm_avg * 1e-3) / 1e9 / hbm_gbs, 4),
                    "hbm_peak_gbs": hbm_gbs},
        "qk_norm_rope": {"ms": round(qk_ms, 5),
                         "gbs": round(qk_bytes / (qk_ms * 1e-3) / 1e9, 1),
                         "frac_of_hbm": round(qk_bytes / (qk_ms * 1e-3) / 1e9 / hbm_gbs, 4),
                         "bytes": qk_bytes,
                         "note": "q, k -> QK-Norm + RoPE, frame-major and token-major copies"},
        "layer_with_qk_norm_rope_ms": round(qk_layer_ms, 5),
        "layer_with_qk_norm_rope_modes": {"spatial": int((qk_modes == 0).sum()),
                                          "temporal": int((qk_modes == 1).sum())},
        "qk_norm_rope_then_layer_ms": round(qk_then_layer_ms, 5),
        "repeat_heads": {
            "similarity_one_frame_ms": round(rs_ms, 5),
            "similarity": {"min": round(float(sims_h.min()), 4),
                           "max": round(float(sims_h.max()), 4),
                           "above_0.87": int((sims_h > 0.87).sum())},
            "spatial_kept_fraction_anchor_tiles": round(anchor_pairs / float(N * N), 5),
            "attention_ms_spatial_heads_repeating": round(rep_attn_ms, 5),
            "attention_ms_spatial_heads_repeating_index_pairs": round(rep_attn_pairs_ms, 5),
            "layer_ms_spatial_heads_repeating": round(rep_layer_ms, 5),
            "note": "anchors k=5 per frame; every spatial head forced to repeat for timing"},
        "profile": {"ms": round(prof_avg, 5),
                    "kv_gbs": round(prof_bytes / (prof_avg * 1e-3) / 1e9, 1),
                    "share_of_step": round(prof_avg / step_ms_avg, 4),
                    "noalloc_ms": round(noalloc_avg, 5),
                    "note": "ms in the step (V exponents on a side stream beside it); "
                            "noalloc_ms: the fixed-scratch entry point alone"},
        "roofline": {"kernel": "svg_sparse_attn_fused", "bound": "tensor",
                     "achieved": round(attn_tf, 3),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(attn_tf / peak_tf, 4),
                     "peak_source": f"{src} bf16 burst", "traffic": attn_traffic(wl.name)},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS",
                "h2d_bytes_per_step": int(job_h2d), "d2h_bytes_per_step": int(job_d2h),
                "ms_per_step": round(e2e_step_ms, 5),
                "api": f"svg_layer_from_host, {hc} heads per chunk"},
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return line


# ------------------------------------------------------- calibrated layer

def run_calibrated(args, rank, world, local_rank):
    """The calibrated Wan 2.1 720p layer ([CAL] 3.1): per-head key-block lists
    built once from the block energies of the calibration inputs (timed
    separately: energy per input, list build), then a step = block-sparse
    attention of every head on its own list (list_id = h, frame-major) on
    the timed input."""
    import torch
    import torch.distributed as dist

    import sparse_attention_video_svg_b200 as svg

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = si.WORKLOADS[args.config]
    heads, sharded, seed = rank_heads(args, wl, rank, world)
    Hl = len(heads)
    N, d = wl.N, wl.d
    nb = svg.n_tiles(N)
    stream = torch.cuda.current_stream()
    tseed = wl.calib_seeds[0]
    shift = seed - wl.seed  # replicas: every rank its own inputs

    def ev():
        return torch.cuda.Event(enable_timing=True)

    # calibration: block energies of every calibration input, then the lists
    E = torch.empty(len(wl.calib_seeds), Hl, nb, nb, dtype=torch.float32, device=dev)
    ews = torch.empty(max(256, svg._lib.lib.svg_block_energy_workspace_size(1, Hl, N)),
                      dtype=torch.uint8, device=dev)
    energy_ms = []
    for r, s in enumerate(wl.calib_seeds):
        q, k, _, _ = si.generate(wl, seed=s + shift, types_seed=tseed, heads=heads)
        qd, kd = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in (q, k))
        del q, k
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record(stream)
        svg.svg_block_energy(qd, kd, out=E[r], workspace=ews)
        e1.record(stream)
        torch.cuda.synchronize()
        energy_ms.append(e0.elapsed_time(e1))
        del qd, kd
    del ews
    svg.svg_build_block_mask_calibrated(E, wl.eps, wl.rho)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    lists = svg.svg_build_block_mask_calibrated(E, wl.eps, wl.rho)
    e1.record(stream)
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)
    del E
    ip = lists.indptr.cpu().numpy().reshape(Hl, nb + 1)
    ix = lists.indices.cpu().numpy()
    pairs = [kept_pairs(ip[h] - ip[h][0], ix[ip[h][0]:ip[h][-1]], N) for h in range(Hl)]
    flops = float(sum(4 * d * p for p in pairs))
    # the pairing order of the query tiles (once per list set, like the lists)
    svg.svg_pair_query_tiles(lists)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    lists = svg.svg_pair_query_tiles(lists)
    e1.record(stream)
    torch.cuda.synchronize()
    pairing_ms = e0.elapsed_time(e1)
    # merged-walk steps of the work items with and without the order (a
    # key block kept by both tiles of an item is one step)
    order = lists.tile_order.cpu().numpy().reshape(Hl, nb)
    rows = [[set(ix[ip[h][i]:ip[h][i + 1]].tolist()) for i in range(nb)] for h in range(Hl)]

    def steps_of(seq):
        return sum(len(rows[h][seq[h][i]] | (rows[h][seq[h][i + 1]] if i + 1 < nb else set()))
                   for h in range(Hl) for i in range(0, nb, 2))
    steps_index = steps_of([list(range(nb))] * Hl)
    steps_paired = steps_of(order.tolist())
    del rows

    q, k, v, _ = si.generate(wl, seed=seed, types_seed=tseed, heads=heads)
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v)]
    del q, k, v
    qd, kd, vd = (h.to(dev) for h in host)
    o = torch.empty_like(qd)
    list_id = torch.arange(Hl, dtype=torch.int32, device=dev)
    vexp = torch.empty(wl.B * Hl, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup

    def step():
        # the per-head V exponents (one read of v), then every head on its
        # list, query tiles paired by the order
        svg.svg_v_exponents(vd, out=vexp)
        svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, list_id, lists, layout=0, out=o,
                                  v_exp=vexp)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    evs = [(ev(), ev()) for _ in range(K)]
    for i in range(K):
        flush.fill_(i & 0xff)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = float(sum(a.elapsed_time(b) for a, b in evs))

    # end to end: q, k, v from pinned host memory, o back, every step; chunks
    # of heads stream through two device slots so the copies overlap the work
    out_host = torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory()
    hc = host_chunk(wl.B * Hl)
    hbufs = svg.HostLayerBuffers(hc, N, d, 1, dev)
    for _ in range(2):
        svg.svg_attention_from_host(*host, list_id, lists, out=out_host, heads_per_chunk=hc,
                                    buffers=hbufs)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(K):
        svg.svg_attention_from_host(*host, list_id, lists, out=out_host, heads_per_chunk=hc,
                                    buffers=hbufs)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    del hbufs

    energy_avg = float(sum(energy_ms) / len(energy_ms))
    total_ms, e2e_ms, energy_avg, build_ms = max_over_ranks(
        [total_ms, e2e_ms, energy_avg, build_ms], world, dev)
    h2d = sum(h.numel() * 2 for h in host)
    d2h = out_host.numel() * 2
    job_flops, job_h2d, job_d2h, job_pairs = sum_over_ranks(
        [flops, h2d, d2h, float(sum(pairs))], world, dev)
    job_tokens = wl.B * N * (1 if sharded else world)
    if rank != 0:
        return None
    peaks, src = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    value, tokens_s, ms = aggregate(job_flops, total_ms, K, job_tokens)
    e2e_value, _, e2e_step_ms = aggregate(job_flops, e2e_ms, K, job_tokens)
    attn_tf = flops / (total_ms / K * 1e-3) / 1e12
    job_heads = wl.H if sharded else Hl * world
    energy_flops = 2 * 2 * float(N) * N * d * Hl  # two dense Q K^T passes per head
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOPS", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded biased-Gaussian q/k/v, no model weights)",
        "config": {**workload_config(wl),
                   **({"heads_subset": f"{heads.start}:{heads.stop}"}
                      if args.heads is not None else {}),
                   "lists": f"calibrated per head: eps {wl.eps}, rho {wl.rho}, inputs "
                            f"{list(wl.calib_seeds)}, timed on seed {wl.seed}",
                   "kept_fraction": round(job_pairs / (float(N) * N * job_heads), 5),
                   "l2": "flushed (256 MB write) before every timed step",
                   "parallelism": (f"heads of one layer split over {world} GPUs" if sharded else
                                   f"independent layer per GPU x{world}" if world > 1 else
                                   "1 GPU")},
        "tokens_per_s": round(tokens_s, 1),
        "pct_of_bf16_peak": round(100 * value / world / peak_tf, 2),
        "attention_only": {"ms": round(total_ms / K, 5), "effective_tflops": round(attn_tf, 3),
                           "kernel": "svg_v_exponents + svg_sparse_attn_fused (list_id = h, "
                                     "tiles paired by svg_pair_query_tiles)"},
        "calibration": {"energy_ms_per_input": round(energy_avg, 3),
                        "energy_tflops": round(energy_flops / (energy_avg * 1e-3) / 1e12, 1),
                        "build_lists_ms": round(build_ms, 3),
                        "pairing_ms": round(pairing_ms, 3),
                        "item_steps": {"index_pairs": int(steps_index),
                                       "paired_order": int(steps_paired)},
                        "inputs": len(wl.calib_seeds),
                        "note": "offline, not in the step"},
        "roofline": {"kernel": "svg_sparse_attn_fused", "bound": "tensor",
                     "achieved": round(attn_tf, 3),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(attn_tf / peak_tf, 4),
                     "peak_source": f"{src} bf16 burst", "traffic": attn_traffic(wl.name)},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS",
                "h2d_bytes_per_step": int(job_h2d), "d2h_bytes_per_step": int(job_d2h),
                "ms_per_step": round(e2e_step_ms, 5),
                "api": f"svg_attention_from_host, {hc} heads per chunk"},
        "gpu_launches": 3 * K,   # V exponents (max, finalize), attention
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return line


# ------------------------------------------------------------- oracle timing

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline_calibrated(wl, budget_s=15.0):
    """The float64 oracle on a bounded sample of the calibrated layer: for
    query tiles of two heads, the energy rows of the tile on every
    calibration input, the voted list row, then block-sparse attention of
    the tile on the timed input.  The value counts the attention alone (the
    calibration is offline); its time is reported beside it."""
    from oracle import svg_oracle as O

    heads = range(2)
    tseed = wl.calib_seeds[0]
    cal = [si.generate(wl, seed=s, types_seed=tseed, heads=heads)[:2] for s in wl.calib_seeds]
    q, k, v, _ = si.generate(wl, seed=wl.seed, types_seed=tseed, heads=heads)
    N = wl.N
    nb = O.n_tiles(N)
    order = np.random.default_rng(0).permutation(nb)
    t_cal = t_att = 0.0
    flops = 0.0
    units = 0
    t_start = time.perf_counter()
    for h in heads:
        qh, kh, vh = (si.as_float64(t[0, h]) for t in (q, k, v))
        cal_h = [(si.as_float64(cq[0, h]), si.as_float64(ck[0, h])) for cq, ck in cal]
        for i in order:
            t0 = time.perf_counter()
            Es = [O.block_energy(cq, ck, row_blocks=[int(i)]) for cq, ck in cal_h]
            ip1, ix1 = O.calibrate_lists(Es, wl.eps, wl.rho)
            t1 = time.perf_counter()
            ip = np.zeros(nb + 1, np.int64)
            ip[i + 1:] = len(ix1)
            rows = O.tile_rows(int(i), N)
            O.block_sparse_rows(qh, kh, vh, rows, ip, ix1)
            t2 = time.perf_counter()
            t_cal += t1 - t0
            t_att += t2 - t1
            flops += 4.0 * wl.d * len(rows) * sum(min(128, N - j * 128) for j in ix1)
            units += 1
            if t2 - t_start > budget_s:
                break
        if time.perf_counter() - t_start > budget_s:
            break
    return {"value": flops / t_att / 1e12, "unit": "TFLOPS", "cores": oracle_threads(),
            "kind": "oracle",
            "sample": f"{wl.name}: {units} query tiles of 2 heads: calibrated list rows "
                      f"({len(wl.calib_seeds)} inputs, {t_cal:.1f} s, not in the value) and "
                      f"block-sparse attention (float64 NumPy, {t_att:.1f} s)"}


def cpu_baseline(wl, budget_s=15.0, seed=None):
    """The float64 oracle on a bounded sample of the same layer: profiling and
    block-sparse attention for as many (head, query tile) units as fit the
    budget, converted to the same effective-TFLOPS unit."""
    from oracle import svg_oracle as O

    if wl.kind == "calibrated":
        return cpu_baseline_calibrated(wl, budget_s)
    seed = wl.seed if seed is None else seed
    one = wl.scaled(wl.name, H=2)
    q, k, v, types = si.generate(one, seed=seed)
    idx = si.sample_queries(wl)
    F, P, w, N = wl.F, wl.P, wl.width, wl.N
    lists = {kind: O.geometric_block_lists(kind, F, P, w, N) for kind in (0, 1)}
    t0 = time.perf_counter()
    flops = 0.0
    units = 0
    heads_profiled = 0
    for h in range(one.H):
        qh, kh, vh = (si.as_float64(t[0, h]) for t in (q, k, v))
        ms, mt, md = O.profile_head(qh, kh, vh, idx, F, P, w)
        heads_profiled += 1
        ip, ix = lists[md]
        if md == O.MODE_TEMPORAL:
            qh, kh, vh = (O.permute_token_major(t, F, P) for t in (qh, kh, vh))
        nb = len(ip) - 1
        for i in range(nb):
            rows = O.tile_rows(i, N)
            O.block_sparse_rows(qh, kh, vh, rows, ip, ix)
            cols = sum(min(128, N - j * 128) for j in ix[ip[i]:ip[i + 1]])
            flops += 4.0 * wl.d * len(rows) * cols
            units += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": oracle_threads(),
            "kind": "oracle",
            "sample": f"{wl.name}: {heads_profiled} head(s) profiled, {units} query tiles of "
                      f"block-sparse attention (float64 NumPy), {dt:.1f} s"}


def run_reference(args, world=1):
    wl = si.WORKLOADS[args.config]
    K, W = args.steps, args.warmup
    budget = max(1.0, args.cpu_budget / max(1, K + W))
    for _ in range(W):
        cpu_baseline(wl, budget_s=budget)
    vals, wall = [], []
    for _ in range(K):
        t0 = time.perf_counter()
        vals.append(cpu_baseline(wl, budget_s=budget))
        wall.append(time.perf_counter() - t0)
    value = statistics.mean(v["value"] for v in vals)
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(1e3 * statistics.mean(wall), 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded biased-Gaussian q/k/v, no model weights)",
        "config": {**workload_config(wl),
                   **({"heads_subset": f"{heads.start}:{heads.stop}"}
                      if args.heads is not None else {}), "oracle": "rank 0 host cores only"},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": vals[-1]["cores"],
                         "kind": "oracle", "sample": vals[-1]["sample"]},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="hunyuan720",
                    choices=[n for n in si.ORDER if n != "tiny"])
    ap.add_argument("--heads", default=None, metavar="A:B",
                    help="run only heads A..B-1 of the layer (small cases for ncu captures)")
    ap.add_argument("--shard", default="heads", choices=["heads", "replicas"],
                    help="multi-GPU: split one layer's heads (default) or one layer per GPU")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    if si.WORKLOADS[args.config].kind == "calibrated":
        line = run_calibrated(args, rank, world, local_rank)
    else:
        line = run_ours(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

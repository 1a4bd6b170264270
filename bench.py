"""Benchmark of the DashAttention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole prefill hot path (stage 0 pooling, stage 1
routing, stage 2 sparse attention) over the 32K-token GQA bf16 workload
(B=1, 32/8 heads, d=128, block 64, alpha 1.5, ~75% block sparsity).  The
printed ``value`` is prefill tokens/s (all ranks); the same line carries a
``decode`` object: µs per decode step for 64 sequences at 64K..128K context
(block 64, 2048 blocks), with its HBM roofline.  Inputs are resident in HBM
and larger than L2 (126 MB), so no flush is needed between timed steps.

``--impl reference`` times the fp64 CPU oracle (the reference for this
build) on a bounded sample of the same workload on the host cores.

Under torchrun every rank runs its own independent sequence (weak scaling,
no data-path collective); times are the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gen import full_inputs, get_config, kv_values, make_plan, q_values, sample_rows  # noqa: E402

METRIC = "sparse-attn tokens/s (prefill) & decode us/step at 128K ctx; % of roofline"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
CSRC = os.path.join(ROOT, "sparse_hierarchical_attention_mean_b200", "csrc")


# --------------------------------------------------------------------------- helpers


def peaks() -> dict:
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_sha(files: list[str]) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, files: list[str]):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current source."""
    sha = source_sha(files)
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for name in sorted(os.listdir(pdir)):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(pdir, name)).read()
        if f"kernel: {kernel}" not in text:
            continue
        m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
        m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        if m_sha and m_tr and m_sha.group(1) == sha:
            return float(m_tr.group(1))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dash_clocks_{os.getpid()}.csv")
        self.t_mark = None
        self.t_end = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def mark(self):
        """Start of the timed region (samples from here on are the ones reported)."""
        self.t_mark = time.time()

    def __exit__(self, *exc):
        self.t_end = time.time()
        time.sleep(0.05)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        import datetime

        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        # samples inside the timed region; the warm-up (same work) if it was too short to catch one
        timed = [r for r in rows if self.t_mark is not None and self.t_mark <= r[0] <= (self.t_end or 1e30)]
        window = "timed"
        if not timed:
            timed = [r for r in rows if r[1] > 0.5 * max((x[1] for x in rows), default=0.0)]
            window = "warm-up and timed (timed region shorter than the sampling interval)"
        if not timed:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = set()
        for r in timed:
            for n, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median([r[1] for r in timed])), "sm_max_mhz": max(r[2] for r in timed),
                "reasons": sorted(reasons), "samples": len(timed), "window": window}


# --------------------------------------------------------------------------- distributed


def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU under torchrun; NCCL on GPUs, gloo for CPU-only runs."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg, rank: int) -> int:
    """Each rank processes its own independent sequence (weak scaling)."""
    return cfg.seed + rank


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_max * 1e-3)


# --------------------------------------------------------------------------- prefill (ours)


def prefill_work(cfg, cnt: torch.Tensor):
    """Selected stage-2 FLOPs from the routing counts cnt [B, Hkv, S] (causal):
    4 d G (block |support| + diagonal tokens) summed over the rows."""
    S, block, d, G = cfg.seq, cfg.block, cfg.head_dim, cfg.group
    pos = torch.arange(S, device=cnt.device)
    diag = (pos - (pos // block) * block + 1).double()  # causal diagonal tokens per row
    sel_tokens = cnt.double() * block + diag  # [B, Hkv, S]
    return 4.0 * d * G * float(sel_tokens.sum())


def union_flops(cfg, idx: torch.Tensor, cnt: torch.Tensor) -> float:
    """FLOPs the tile-pair stage-2 kernel executes: each tile of 128 / G positions (128 rows)
    runs every block in the union of its rows' lists plus its own blocks (64-token steps up
    to its last position), for all of its rows."""
    B, Hkv, S, T = idx.shape
    P = 128 // cfg.group
    n_tiles = -(-S // P)
    blk = cfg.block
    union_blocks = 0.0
    own_tokens = 0.0
    ar = torch.arange(T, device=idx.device)
    chunk = max(1, 16384 // P)  # tiles per pass (bounds the temporary mask)
    for t0 in range(0, n_tiles, chunk):
        t1 = min(n_tiles, t0 + chunk)
        lo, hi = t0 * P, min(S, t1 * P)
        sub_idx, sub_cnt = idx[:, :, lo:hi], cnt[:, :, lo:hi]
        mask = torch.zeros((B, Hkv, (t1 - t0) * P, T + 1), dtype=torch.bool, device=idx.device)
        tgt = torch.where(ar < sub_cnt[..., None], sub_idx.long(), T)
        mask[:, :, : hi - lo].scatter_(3, tgt, True)
        tiles = mask[..., :T].view(B, Hkv, t1 - t0, P, T).any(3)
        for tl in range(t0, t1):  # own blocks are counted below, once
            a, b = tl * P, min(S, tl * P + P) - 1
            tiles[:, :, tl - t0, a // blk:b // blk + 1] = False
        union_blocks += float(tiles.sum())
        del mask, tgt, tiles
    for tl in range(n_tiles):
        a, b = tl * P, min(S, tl * P + P) - 1
        for c in range(a // blk, b // blk + 1):
            last = min(b, (c + 1) * blk - 1)
            own_tokens += -(-(last - c * blk + 1) // 64) * 64
    tokens = union_blocks * blk + B * Hkv * own_tokens
    return 4.0 * cfg.head_dim * 128 * tokens


def measure_forward(dash, cfg, steps, warmup, world, rank, clocks=False):
    """Times one prefill workload through dash_attn_fwd (the whole forward, CUDA events around
    `steps` back-to-back calls, max over ranks), then the same work stage by stage, and the
    stage-2 entry point alone (the dominant kernel).  Work counts come from the routing lists
    the timed forward left in its workspace."""
    inp = full_inputs(cfg, device="cuda", seed=rank_seed(cfg, rank))
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    B, S, H, d = q.shape
    out = torch.empty_like(q)
    ws = torch.empty(dash.fwd_workspace_size(q, k, cfg.block), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        dash.fwd(q, k, v, w, cfg.alpha, cfg.block, cfg.causal, out=out, workspace=ws)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(torch.cuda.current_device()) if clocks else None
    if clk:
        clk.__enter__()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if clk:
        clk.mark()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__(None, None, None)
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, world)
    status = dash.device_status(ws)

    # the routing the timed forward used (views into its workspace)
    lists = dash.fwd_lists(ws, q, k, cfg.block)
    summ, idx, logp, cnt = lists["summaries"], lists["idx"], lists["logp"], lists["cnt"]
    flops = prefill_work(cfg, cnt)
    uflops = union_flops(cfg, idx, cnt)
    pos = torch.arange(S, device="cuda")
    cand_row = (pos // cfg.block).double()
    per_head_cand = float(cand_row.sum()) * B
    per_head_sel = cnt.double().sum(dim=(0, 2))  # [Hkv]
    head_sparsity = (1.0 - per_head_sel / per_head_cand).tolist()
    sparsity = 1.0 - float(per_head_sel.sum()) / (per_head_cand * k.shape[2])

    # stage by stage through the stage entry points, writing into the same buffers
    T = idx.shape[-1]
    sws = torch.empty(dash.sparse_workspace_size(q, k, cfg.block, T), dtype=torch.uint8, device="cuda")
    rws = torch.empty(dash.route_workspace_size(q, k.shape[2], T, False), dtype=torch.uint8, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    seg = np.zeros(3)

    def stages(record):
        if record:
            evs[0].record(stream)
        dash.summarize(k, w, cfg.block, summaries=summ)
        if record:
            evs[1].record(stream)
        dash.route(q, summ, cfg.alpha, cfg.block, cfg.causal, idx=idx, logp=logp, cnt=cnt, workspace=rws)
        if record:
            evs[2].record(stream)
        dash.sparse(q, k, v, idx, logp, cnt, cfg.block, cfg.causal, out=out, workspace=sws)
        if record:
            evs[3].record(stream)

    for _ in range(warmup):
        stages(False)
    torch.cuda.synchronize()
    for _ in range(steps):
        stages(True)
        torch.cuda.synchronize()
        seg += [evs[i].elapsed_time(evs[i + 1]) for i in range(3)]
    seg /= steps

    # the dominant kernel alone: stage 2 (pair-list kernel + tcgen05 attention kernel)
    # launched back to back on the same stream, CUDA events around the loop
    for _ in range(warmup):
        dash.sparse(q, k, v, idx, logp, cnt, cfg.block, cfg.causal, out=out, workspace=sws)
    torch.cuda.synchronize()
    evs[0].record(stream)
    for _ in range(steps):
        dash.sparse(q, k, v, idx, logp, cnt, cfg.block, cfg.causal, out=out, workspace=sws)
    evs[1].record(stream)
    torch.cuda.synchronize()
    sparse_ms = max_over_ranks(evs[0].elapsed_time(evs[1]) / steps, world)
    del sws, rws, lists, summ, idx, logp, cnt
    return {"inp": inp, "out": out, "ws": ws, "ms": ms, "tokens": B * S, "status": status,
            "seg_ms": seg.tolist(), "sparse_ms": sparse_ms, "flops": flops, "union_flops": uflops,
            "sparsity": sparsity, "head_sparsity": head_sparsity,
            "achieved_tflops": flops / (sparse_ms * 1e-3) / 1e12, "clocks": clk.summary() if clk else None}


def run_prefill(dash, cfg, steps, warmup, world, rank, pk, do_backward=True):
    m = measure_forward(dash, cfg, steps, warmup, world, rank, clocks=True)
    q, k, v, w = m["inp"]["q"], m["inp"]["k"], m["inp"]["v"], m["inp"]["w_s"]
    traffic = profiled_traffic("sparse_prefill_tc_kernel", ["attn_prefill_tc.cu", "tc.cuh", "sparse_common.cuh",
                                                            "common.cuh"])
    # End to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory and reads its output back.  Copies
    # run on their own streams, double-buffered, so step i+1's upload and
    # step i-1's download overlap step i's kernels.
    e2e_ms, h2d, d2h = run_e2e(dash, cfg, q, k, v, w, m["ws"], steps, warmup, world)
    ws = m.pop("ws")
    del ws
    bwd = run_backward(dash, cfg, q, k, v, w, m["out"], min(steps, 5), warmup, m["flops"], world) \
        if do_backward else None
    m.update({"traffic": traffic, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h, "backward": bwd})
    del m["inp"], m["out"]
    return m


def prefill_object(m, cfg, pk, world, extra=None):
    """Summary of one measured prefill workload (tokens/s, stages, sparsity, stage-2 roofline)."""
    peak = pk["bf16_tflops"]
    obj = {
        "tokens_per_s": job_throughput(m["tokens"], world, m["ms"]), "ms_per_step": m["ms"],
        "stage_ms": {"pool": m["seg_ms"][0], "route": m["seg_ms"][1], "sparse_attention": m["seg_ms"][2]},
        "sparsity": m["sparsity"], "union_inflation": m["union_flops"] / m["flops"],
        "roofline": {"kernel": "stage-2 entry point (pair lists + sparse_prefill_tc_kernel) back to back",
                     "bound": "tensor", "ms_per_launch": m["sparse_ms"], "achieved": m["achieved_tflops"],
                     "peak": peak, "unit": "TFLOP/s", "frac": m["achieved_tflops"] / peak, "traffic": None,
                     "selected_flops": m["flops"], "peak_source": f"{pk['source']} bf16 (burst)"},
        "device_status": m["status"],
    }
    if extra:
        obj.update(extra)
    return obj


def run_long_prefill(dash, steps, warmup, world, rank, pk):
    cfg = get_config("long_prefill")
    m = measure_forward(dash, cfg, steps, warmup, world, rank)
    hs = m["head_sparsity"]
    obj = prefill_object(m, cfg, pk, world, {
        "workload": "long prefill: B=1, S=131072, 32/8 heads, d=128, bf16, causal, block 128 (1024 blocks), "
                    "alpha 1.5; KV heads 0-3 diffuse (no plant), 4-7 needle heads (1-16 planted blocks per topic)",
        "sparsity_per_kv_head": hs,
        "sparsity_diffuse_heads": float(np.mean(hs[:4])), "sparsity_needle_heads": float(np.mean(hs[4:])),
        "steps": steps,
    })
    del m
    torch.cuda.empty_cache()
    return obj


def run_sweep(dash, steps, warmup, world, rank, pk):
    from gen import sweep_configs

    points = []
    for cfg in sweep_configs():
        m = measure_forward(dash, cfg, steps, warmup, world, rank)
        o = prefill_object(m, cfg, pk, world, {"alpha": cfg.alpha, "key_strength": cfg.key_strength})
        o["roofline"]["peak_source"] = f"{pk['source']} bf16 (burst); f16 has the same dense rate"
        points.append(o)
        del m
        torch.cuda.empty_cache()
    return {"workload": "alpha / sparsity sweep: B=4, 16/16 heads, d=64, f16, S=16384, causal, block 64, "
                        "16 topics; alpha in {1.25, 1.5, 2}, key plant strength in {0, 1, 2, 4}",
            "steps": steps, "points": points}


def run_backward(dash, cfg, q, k, v, w, out, steps, warmup, fwd_flops, world):
    """The backward pass (dash_attn_bwd) on the same inputs, timed with CUDA events.

    Algorithmic work: 2.5x the forward's selected FLOPs (the scores S = QK^T
    recomputed, dP = dout V^T, and the three gradient products dV = P^T dout,
    dK = dS^T Q, dQ = dS K, against the forward's two products).
    """
    gen = torch.Generator(device="cuda").manual_seed(7)
    dout = torch.randn(q.shape, generator=gen, device="cuda", dtype=torch.float32).to(q.dtype)
    ws = torch.empty(dash.bwd_workspace_size(q, k, cfg.block), dtype=torch.uint8, device="cuda")
    grads = {"dq": torch.empty(q.shape, dtype=torch.float32, device="cuda"),
             "dk": torch.empty(k.shape, dtype=torch.float32, device="cuda"),
             "dv": torch.empty(v.shape, dtype=torch.float32, device="cuda"),
             "dw_s": torch.empty((q.shape[-1], q.shape[-1]), dtype=torch.float32, device="cuda")}
    stream = torch.cuda.current_stream()

    def step():
        dash.bwd(q, k, v, w, out, dout, cfg.alpha, cfg.block, True, grads=grads, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, world)
    status = dash.device_status(ws)
    del ws
    return {"ms": ms, "flops": 2.5 * fwd_flops, "steps": steps, "status": status}


def run_e2e(dash, cfg, q, k, v, w, ws, steps, warmup, world):
    hq, hk, hv = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
    hout = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    dev = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)) for _ in range(2)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, comp_done, out_free = [ev() for _ in range(2)], [ev() for _ in range(2)], [ev() for _ in range(2)]
    for e in comp_done + out_free:
        e.record(comp)

    def e2e_step(i):
        sl = i & 1
        dq, dk, dv, dout = dev[sl]
        up.wait_event(comp_done[sl])  # the slot's previous step no longer reads its inputs
        with torch.cuda.stream(up):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
        in_ready[sl].record(up)
        comp.wait_event(in_ready[sl])
        comp.wait_event(out_free[sl])  # the slot's previous output has been read back
        dash.fwd(dq, dk, dv, w, cfg.alpha, cfg.block, True, out=dout, workspace=ws)
        comp_done[sl].record(comp)
        down.wait_event(comp_done[sl])
        with torch.cuda.stream(down):
            hout[sl].copy_(dout, non_blocking=True)
        out_free[sl].record(down)

    for i in range(max(1, warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(up)
    for i in range(steps):
        e2e_step(i)
    down.wait_stream(comp)
    down.wait_stream(up)
    t1.record(down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    h2d = (q.numel() + k.numel() + v.numel()) * q.element_size()
    d2h = q.numel() * q.element_size()
    return e2e_ms, h2d, d2h


# --------------------------------------------------------------------------- decode (ours)


def run_decode(dash, cfg, steps, warmup, world, rank):
    inp = full_inputs(cfg, device="cuda", seed=rank_seed(cfg, rank))
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    B, _, H, d = q.shape
    Hkv = k.shape[2]
    T = -(-cfg.seq // cfg.block)
    summ = torch.zeros((B, Hkv, T, d), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dash.summarize(k, w, cfg.block, seqlens=sl, summaries=summ)
    torch.cuda.synchronize()
    e0.record(stream)
    dash.summarize(k, w, cfg.block, seqlens=sl, summaries=summ)
    e1.record(stream)
    torch.cuda.synchronize()
    summarize_ms = e0.elapsed_time(e1)
    # the same cache with learned summary queries (seeded q_bar per KV head)
    qbar = torch.from_numpy(np.random.default_rng(11).normal(size=(Hkv, d)) * 3.0).float().cuda()
    summ_q = torch.zeros_like(summ)
    dash.summarize(k, w, cfg.block, seqlens=sl, summaries=summ_q, qbar=qbar)
    torch.cuda.synchronize()
    e0.record(stream)
    dash.summarize(k, w, cfg.block, seqlens=sl, summaries=summ_q, qbar=qbar)
    e1.record(stream)
    torch.cuda.synchronize()
    summarize_sdpa_ms = e0.elapsed_time(e1)
    del summ_q
    pool_bytes = float(sl.double().sum()) * Hkv * d * k.element_size() + float(summ.numel()) * 4
    out = torch.empty_like(q)
    ws = torch.empty(dash.decode_workspace_size(q, k, cfg.block, T), dtype=torch.uint8, device="cuda")

    def step():
        dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block, out=out, workspace=ws)

    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clk.mark()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    us = max_over_ranks(e0.elapsed_time(e1) / steps * 1e3, world)
    status = dash.device_status(ws)

    rt = dash.route(q, summ, cfg.alpha, cfg.block, True, seqlens=sl)
    cnt = rt["cnt"][:, :, 0].double()  # [B, Hkv]
    L = sl.double()
    pos = L - 1
    n_cand = torch.floor(pos / cfg.block)
    diag = pos - n_cand * cfg.block + 1
    bytes_summ = float((n_cand * d * 4).sum()) * Hkv
    bytes_kv = float((cnt * cfg.block * d * 4).sum()) + float((diag * d * 4).sum()) * Hkv
    bytes_q = 2.0 * B * H * d * 2
    total = bytes_summ + bytes_kv + bytes_q
    sparsity = 1.0 - float(cnt.sum()) / float(n_cand.sum() * Hkv)
    return {"us": us, "bytes": total, "bytes_summaries": bytes_summ, "sparsity": sparsity,
            "summarize_ms": summarize_ms, "summarize_sdpa_ms": summarize_sdpa_ms, "pool_bytes": pool_bytes,
            "status": status, "clocks": clk.summary()}


def run_cp_decode(dash, cfg, steps, warmup, rank, ranks=4):
    """Context-parallel decode on the decode workload, `ranks` block-aligned shards of every
    sequence's cache run one after another on this GPU (what the ranks of a context-parallel
    group do at once): shard scores, their sum (the all-reduce), lists, shard attention, and
    the log-sum-exp merge of the stacked partials (the all-gather).  The shards are views of
    the cache; each has its own summaries, built once outside the timed steps."""
    inp = full_inputs(cfg, device="cuda", seed=rank_seed(cfg, rank))
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    B, lmax, Hkv, d = k.shape
    G, blk = cfg.group, cfg.block
    t_cap = -(-lmax // blk)
    bounds = [((lmax // blk) * r // ranks) * blk for r in range(ranks)] + [lmax]
    shards = []
    for r in range(ranks):
        lo, hi = bounds[r], bounds[r + 1]
        ks, vs = k[:, lo:hi], v[:, lo:hi]
        sl_r = (sl - lo).clamp(0, hi - lo).to(torch.int32)
        shards.append((lo, hi, ks, vs, dash.summarize(ks, w, blk, seqlens=sl_r)))
    H = q.shape[2]
    scores = torch.zeros((B, Hkv, G, t_cap), dtype=torch.float32, device="cuda")
    part_scores = torch.zeros_like(scores)
    parts = torch.empty((ranks, B, H, d + 2), dtype=torch.float32, device="cuda")
    ws = torch.empty(dash.cp_attend_workspace_size(B, H, Hkv, d, blk, t_cap), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    attend_ms = 0.0

    def step(record):
        scores.zero_()
        for lo, hi, ks, vs, summ_r in shards:
            part_scores.zero_()
            dash.cp_scores(q, summ_r, lo // blk, hi // blk, sl, lmax, cfg.alpha, blk, part_scores)
            scores.add_(part_scores)
        lists = dash.cp_lists(q, Hkv, scores, sl, lmax, cfg.alpha, blk)
        if record:
            ev[2].record(stream)
        for r, (lo, hi, ks, vs, _) in enumerate(shards):
            dash.cp_attend_ex(q, ks, vs, lo, sl, lmax, lists, blk, part=parts[r], workspace=ws)
        if record:
            ev[3].record(stream)
        dash.cp_merge(parts, out)
        return lists

    for _ in range(warmup):
        step(False)
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(steps):
        ev[0].record(stream)
        lists = step(True)
        ev[1].record(stream)
        torch.cuda.synchronize()
        total += ev[0].elapsed_time(ev[1])
        attend_ms += ev[2].elapsed_time(ev[3])
    # the CUDA-core shard attention (no workspace) on the same lists, for comparison
    core_ms = 0.0
    for _ in range(steps):
        ev[2].record(stream)
        for r, (lo, hi, ks, vs, _) in enumerate(shards):
            dash.cp_attend(q, ks, vs, lo, sl, lmax, lists, blk, part=parts[r])
        ev[3].record(stream)
        torch.cuda.synchronize()
        core_ms += ev[2].elapsed_time(ev[3])
    # bytes the shard attention reads: the selected and diagonal K/V (each read once over the shards)
    cnt = lists["cnt"].double()
    pos = sl.double() - 1
    diag = pos - torch.floor(pos / blk) * blk + 1
    kv_bytes = float((cnt * blk * d * 4).sum()) + float((diag * d * 4).sum()) * Hkv
    attend_us = attend_ms / steps * 1e3
    core_us = core_ms / steps * 1e3
    return {"ranks": ranks, "us_per_step": total / steps * 1e3, "attend_us": attend_us,
            "attend_gbs": kv_bytes / (attend_us * 1e-6) / 1e9, "kv_bytes": kv_bytes,
            "attend_kernel": "split-KV tensor-core path (dash_attn_cp_attend_ex)",
            "attend_cuda_cores_us": core_us, "attend_cuda_cores_gbs": kv_bytes / (core_us * 1e-6) / 1e9}


def cp_object(cpd, pk) -> dict:
    return {
        "workload": f"decode workload above, each sequence's cache split into {cpd['ranks']} block-aligned "
                    "shards run one after another on this GPU (shard scores, their sum, lists, shard "
                    "attention, log-sum-exp merge)",
        "us_per_step_all_shards": cpd["us_per_step"], "shard_attention_us": cpd["attend_us"],
        "shard_attention": {"bound": "hbm", "achieved": cpd["attend_gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": cpd["attend_gbs"] / pk["hbm_gbs"], "bytes": cpd["kv_bytes"],
                            "kernel": cpd["attend_kernel"], "peak_source": f"{pk['source']} HBM copy"},
        "shard_attention_cuda_cores": {"us": cpd["attend_cuda_cores_us"], "achieved": cpd["attend_cuda_cores_gbs"],
                                       "unit": "GB/s", "frac": cpd["attend_cuda_cores_gbs"] / pk["hbm_gbs"]},
    }


# --------------------------------------------------------------------------- oracle timing


def oracle_sample_time(cfg, n_rows: int, budget_s: float, seed: int = 0, groups=None, row_offset: int = 0) -> dict:
    """Times the oracle on a bounded sample of the prefill workload on this host, one thread.

    For each sampled KV group (default: all): pooling of the whole sequence
    once, then the routing and sparse attention of ``n_rows`` evenly spread
    query positions (shifted by ``row_offset``).  Returns the full-sequence
    time (all KV groups and positions) extrapolated from the sample, and
    tokens/s.
    """
    from threadpoolctl import threadpool_limits

    from oracle.dash_oracle import block_summaries, forward_row

    plan = make_plan(cfg, seed)
    G = cfg.group
    rows = (np.linspace(cfg.block, cfg.seq - 1 - cfg.block, n_rows).astype(int) + row_offset % cfg.block).tolist()
    pool_t = row_t = 0.0
    n_done = 0
    t_start = time.perf_counter()
    groups = list(range(cfg.kv_heads)) if groups is None else list(groups)
    with threadpool_limits(1):
        for g in groups:
            k = kv_values(cfg, plan, "k", 0, range(cfg.seq), [g], as_float32=True)[:, 0].double().numpy()
            v = kv_values(cfg, plan, "v", 0, range(cfg.seq), [g], as_float32=True)[:, 0].double().numpy()
            q = q_values(cfg, plan, 0, rows, range(g * G, (g + 1) * G), as_float32=True).double().numpy()
            t0 = time.perf_counter()
            summ = block_summaries(k, plan.w_s.double().numpy(), cfg.block, cfg.seq)
            t1 = time.perf_counter()
            pool_t += t1 - t0
            for i, pos in enumerate(rows):
                forward_row(q[i], k, v, summ, pos, cfg.seq, cfg.block, cfg.alpha, True)
                n_done += 1
                if time.perf_counter() - t_start > budget_s and i >= 1:
                    break
            row_t += time.perf_counter() - t1
    per_row = row_t / max(n_done, 1)  # one position of one KV group (G heads)
    full_s = pool_t / len(groups) * cfg.kv_heads + per_row * cfg.seq * cfg.kv_heads
    return {"full_s": full_s, "tokens_per_s": cfg.seq / full_s, "rows": n_done, "wall_s": time.perf_counter() - t_start,
            "pool_s": pool_t, "row_s": row_t, "n_groups": len(groups),
            "sample": f"{n_done} (position, KV group) rows spread over the {cfg.seq}-token sequence + pooling of "
                      f"{len(groups)} of {cfg.kv_heads} KV heads, extrapolated to {cfg.seq} positions x "
                      f"{cfg.kv_heads} groups"}


def _oracle_worker(args):
    cfg, n_rows, budget_s, seed, g, offset = args
    return oracle_sample_time(cfg, n_rows, budget_s, seed, groups=[g], row_offset=offset)


def host_info() -> dict:
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


class OraclePool:
    """The oracle run by one single-threaded process per host core, up to 64 (spawned, so no worker
    inherits a CUDA context).  Each process times its own sample (the oracle as it stands),
    all at once, so memory-bandwidth contention between cores is part of the measurement."""

    def __init__(self, workers: int | None = None):
        import multiprocessing as mp

        self.n = workers or max(1, min(64, (os.cpu_count() or 2) - 1))
        self.pool = mp.get_context("spawn").Pool(self.n)

    def sample(self, cfg, n_rows: int, budget_s: float, seed: int, step: int = 0) -> dict:
        tasks = [(cfg, n_rows, budget_s, seed, (step * self.n + i) % cfg.kv_heads, 7 * (step * self.n + i))
                 for i in range(self.n)]
        parts = self.pool.map(_oracle_worker, tasks, chunksize=1)
        rows = sum(p["rows"] for p in parts)
        row_s = sum(p["row_s"] for p in parts)
        pool_s = sum(p["pool_s"] for p in parts) / len(parts)
        # the whole job spread over the n processes: per-row and per-group costs measured under load
        full_s = (pool_s * cfg.kv_heads + row_s / rows * cfg.seq * cfg.kv_heads) / self.n
        return {"full_s": full_s, "tokens_per_s": cfg.seq / full_s, "rows": rows,
                "sample": f"{rows} (position, KV group) rows and {len(parts)} KV-head poolings timed at once on "
                          f"{self.n} processes (one thread each), extrapolated to {cfg.seq} positions x "
                          f"{cfg.kv_heads} groups shared over the {self.n} processes"}

    def close(self):
        self.pool.close()
        self.pool.join()


# --------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences in the decode workload (64 = full)")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--skip-long", action="store_true", help="skip the 128K long-prefill workload")
    ap.add_argument("--skip-sweep", action="store_true", help="skip the alpha / sparsity sweep")
    ap.add_argument("--skip-cp", action="store_true", help="skip the context-parallel decode emulation")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--seq", type=int, default=None,
                    help="prefill sequence length override (smaller cases for profiling; default 32768)")
    args = ap.parse_args()
    warmup = max(3, args.warmup)
    cfg = get_config("prefill")
    if args.seq is not None:
        cfg = cfg.with_(seq=args.seq)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        pool = OraclePool()
        per_step = []
        samples = None
        for i in range(warmup + args.steps):
            # each step: every process samples 2 rows of one KV group (rotating) and its pooling
            r = pool.sample(cfg, n_rows=2, budget_s=30.0, seed=cfg.seed, step=i)
            if i >= warmup:
                per_step.append(r["full_s"])
                samples = r
        pool.close()
        full_s = float(np.mean(per_step))
        value = cfg.seq / full_s
        info = host_info()
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": warmup, "ms_per_step": full_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"prefill GQA bf16 inputs (B=1, S={cfg.seq}, 32/8 heads, d=128, block 64, "
                                   "alpha 1.5)",
                       "global_batch": 1, "seq_len": cfg.seq,
                       "parallelism": f"host oracle, {pool.n} processes x 1 thread"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.n, "kind": "oracle",
                             "sample": samples["sample"] + "; each step one such sample", **info},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    import sparse_hierarchical_attention_mean_b200 as dash

    dash.load()
    world, rank, _ = dist_setup(args.gpus)
    pk = peaks()
    pre = None if args.skip_prefill else run_prefill(dash, cfg, args.steps, warmup, world, rank, pk,
                                                         not args.skip_backward)
    dec = cpd = None
    dcfg = get_config("decode").with_(batch=args.decode_batch)
    if not args.skip_decode:
        dec = run_decode(dash, dcfg, max(20, args.steps), warmup, world, rank)
        torch.cuda.empty_cache()
        if not args.skip_cp:
            cpd = run_cp_decode(dash, dcfg, max(5, min(args.steps, 10)), warmup, rank)
            torch.cuda.empty_cache()

    long_obj = sweep_obj = None
    if not args.skip_long and not args.skip_prefill:
        long_obj = run_long_prefill(dash, max(3, min(args.steps, 5)), warmup, world, rank, pk)
    if not args.skip_sweep and not args.skip_prefill:
        sweep_obj = run_sweep(dash, max(3, min(args.steps, 5)), warmup, world, rank, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        c1 = oracle_sample_time(cfg, n_rows=6, budget_s=args.cpu_budget / 2)
        pool = OraclePool()
        cn = pool.sample(cfg, n_rows=3, budget_s=args.cpu_budget / 2, seed=cfg.seed)
        pool.close()
        cpu = {"value": cn["tokens_per_s"], "unit": "tokens/s", "cores": pool.n, "kind": "oracle",
               "sample": cn["sample"], **host_info(),
               "one_thread": {"value": c1["tokens_per_s"], "unit": "tokens/s", "cores": 1, "sample": c1["sample"],
                              "wall_s": round(c1["wall_s"], 1)}}

    if rank != 0:
        barrier(world)
        finish(world)
        return
    if pre is None:
        print(json.dumps({"decode_only": True, "us_per_step": None if dec is None else dec["us"],
                          "decode": None if dec is None else decode_object(dec, dcfg, pk),
                          "cp_decode": None if cpd is None else cp_object(cpd, pk)}), flush=True)
        barrier(world)
        finish(world)
        return
    value = job_throughput(pre["tokens"], world, pre["ms"])
    peak_tf = pk["bf16_tflops"]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": warmup,
        "ms_per_step": pre["ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"prefill GQA: B=1, S={cfg.seq}, 32 q / 8 kv heads, d=128, bf16, causal, "
                               "block 64, alpha 1.5, topic-planted keys (~75% block sparsity)",
                   "global_batch": world, "seq_len": cfg.seq, "parallelism": f"dp{world} (independent sequences)",
                   "l2": "inputs larger than L2 (q 268 MB, k+v 134 MB); no flush"},
        "sparsity": pre["sparsity"],
        "stage_ms": {"pool": pre["seg_ms"][0], "route": pre["seg_ms"][1], "sparse_attention": pre["seg_ms"][2]},
        "roofline": {
            "kernel": "sparse_prefill_tc_kernel, timed through the stage-2 entry point (with its union- and "
                      "pair-list kernels, ~4%) launched back to back",
            "ms_per_launch": pre["sparse_ms"],
            "bound": "tensor",
            "achieved": pre["achieved_tflops"],
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": pre["achieved_tflops"] / peak_tf,
            "traffic": pre["traffic"],
            "peak_source": f"{pk['source']} bf16 (burst)",
            "selected_flops": pre["flops"],
            "union_inflation": pre["union_flops"] / pre["flops"],
        },
        "e2e": {"value": job_throughput(pre["tokens"], world, pre["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": pre["h2d"], "d2h_bytes_per_step": pre["d2h"]},
        "gpu_launches": 5 * args.steps,  # per forward: pool, summary split, routing, pair lists, attention
        "clocks": pre["clocks"],
        "device_status": pre["status"],
        "cpu_baseline": cpu,
    }
    if dec is not None:
        line["decode"] = decode_object(dec, dcfg, pk)
    if cpd is not None:
        line["cp_decode"] = cp_object(cpd, pk)
    if long_obj is not None:
        line["long_prefill"] = long_obj
    if sweep_obj is not None:
        line["sweep"] = sweep_obj
    if pre["backward"] is not None:
        bw = pre["backward"]
        ach = bw["flops"] / (bw["ms"] * 1e-3) / 1e12
        line["backward"] = {
            "workload": "gradients of the prefill workload above (dq, dk, dv fp32 and dW_s), dout ~ N(0, 1)",
            "ms": bw["ms"], "steps": bw["steps"], "device_status": bw["status"],
            "roofline": {"kernels": "the whole backward call: pooling, routing, the stage-2 log-sum-exp pass, "
                                    "row masks, bwd_row_tc and bwd_key_tc (tcgen05), bwd_route, bwd_ws",
                         "bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s", "frac": ach / peak_tf,
                         "traffic": None, "algorithmic_flops": bw["flops"],
                         "peak_source": f"{pk['source']} bf16 (burst)"},
        }
    print(json.dumps(line), flush=True)
    barrier(world)
    finish(world)


def decode_object(dec, dcfg, pk):
    ach = dec["bytes"] / (dec["us"] * 1e-6) / 1e9
    return {
        "workload": f"decode: {dcfg.batch} seqs, 32/8 heads, d=128, bf16, cache 131072, L ~ U[65536, 131072], "
                    "block 64",
        "us_per_step": dec["us"], "sparsity": dec["sparsity"],
        "summary_cache": {"bytes": dec["pool_bytes"], "mean_ms": dec["summarize_ms"],
                          "mean_gbs": dec["pool_bytes"] / (dec["summarize_ms"] * 1e-3) / 1e9,
                          "learned_query_ms": dec["summarize_sdpa_ms"],
                          "learned_query_gbs": dec["pool_bytes"] / (dec["summarize_sdpa_ms"] * 1e-3) / 1e9,
                          "peak_gbs": pk["hbm_gbs"]},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / pk["hbm_gbs"], "traffic": None, "bytes_per_step": dec["bytes"],
                     "peak_source": f"{pk['source']} HBM copy"},
        "clocks": dec["clocks"], "device_status": dec["status"], "gpu_launches_per_step": 4,
    }


def finish(world):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()

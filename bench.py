"""Benchmark of the NABLA hot path on B200.

One step = one pass of the whole forward hot path over one batch of synthetic
input: the mask builder (pooling, reduced scores, softmax, CDF selection,
index lists, work list) followed by block-sparse attention forward over the
kept tiles.  Default workload: the 720p-shaped problem (B=1, H=40, S=75,600,
D=128, bf16, thr 0.8).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nabla|reference]

N > 1 runs under torch.distributed.run, one process per GPU; every rank
processes its own independent problem of the same shape (weak scaling, no
collective on the data path) and the reported time is the maximum over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NABLA attn ms/call + achieved TFLOP/s at S=75,600, H=40, D=128 bf16; mask-build GB/s"
WORKLOAD_ID = 3
# kernels of this library per step: pool, score GEMM, select, work list
# (mask builder, no CSC transpose) and the attention forward
LAUNCHES_PER_STEP = 5
THR = 0.8

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture, keyed by the SHA-256 of the kernel source it was taken on;
# reported only while the source is unchanged.
NCU_TRAFFIC = {
    # 4-head capture of the 720p shape at thr 0.8: 301.6 MB, scaled x10 to 40 heads
    "attn_fwd_tc.cu": ("bc42bc8e5f502ccf8f42ff8185e5efa74da747e0c6fee1a7d40adc9c6b74438a", 3.016e9),
    # full-size capture of the projection leg (one pass): DRAM read 7.96 GB + write 2.50 GB
    "qkv_tc.cu": ("2bf31b7e64ef472bc2670ca245436e66ceafb3494d6951646151ea3385f8ff90", 10.46e9),
}
# the mask builder's four launches, captured together at full size (one pass
# each): pool 1.55 GB + 184 MB, score GEMM 98 + 165 MB, selection 323 + 95 MB,
# work list 7 MB; keyed by the three sources they come from
NCU_BUILDER_TRAFFIC = ({"pool.cu": "ca97bc086ac16466e6d5db392101528fccf729ca4dfb3b099cfc0c5a87fad7b6",
                        "score_tc.cu": "21f70fb96eaedfe6a16ebc1c608ea74616280707caf240b4744f22c3cd28cc5a",
                        "mask_kernels.cu": "b7a03e632ccf5e26dd4f61360ca8d46eab111746af8de1b68aff913884ac51aa"},
                       2.422e9)


def _sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def _builder_traffic():
    files, bytes_ = NCU_BUILDER_TRAFFIC
    for f, h in files.items():
        path = os.path.join(ROOT, "block_sparse_attention_nabla_b200", "csrc", f)
        if not os.path.exists(path) or _sha(path) != h:
            return None
    return bytes_


def _traffic(kernel_file: str):
    ent = NCU_TRAFFIC.get(kernel_file)
    if not ent:
        return None
    path = os.path.join(ROOT, "block_sparse_attention_nabla_b200", "csrc", kernel_file)
    return ent[1] if os.path.exists(path) and _sha(path) == ent[0] else None


def _peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region
    runs: nvidia-smi is started (and has printed its first line) before the
    region, every line carries its timestamp, and the summary keeps the lines
    that fall between mark_start() and mark_end()."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
            deadline = time.time() + 5.0
            while time.time() < deadline and os.path.getsize(self.file.name) == 0:
                time.sleep(0.05)  # sampling is live before the region starts
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        import datetime
        self.file.flush()
        rows = [l.split(",") for l in open(self.file.name).read().strip().splitlines() if l.strip()]
        os.unlink(self.file.name)
        parsed = []
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 10:
                continue
            ts = None
            for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
                try:
                    ts = datetime.datetime.strptime(r[0], fmt).timestamp()
                    break
                except ValueError:
                    pass
            try:
                parsed.append((ts, float(r[2]), float(r[3]), r[6:10]))
            except ValueError:
                continue
        inside = [p for p in parsed if p[0] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 - 0.05 <= p[0] <= self.t1 + 0.05]
        use = inside or parsed
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for p in use:
            for n, v in zip(names, p[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm = [p[1] for p in use]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(p[2] for p in use) if use else None,
                "reasons": sorted(reasons), "samples": len(inside),
                **({} if inside else {"note": "no sample fell inside the timed region; all samples used"})}


def rank_workload(w, rank: int):
    """Every rank times its own independent problem of the same shape (weak
    scaling): rank r > 0 draws its inputs from seed + 1000 r."""
    return w.scaled(seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(values, dist=None, device=None) -> list:
    """Element-wise maximum of per-rank timings over all ranks (the slowest
    rank sets the job's time); unchanged without a process group."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: the kept-tile flops of all ranks' problems over
    the max-over-ranks step time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def cpu_baseline(x: dict, thr: float, budget_s: float = 12.0, heads_total: int | None = None) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the
    full mask of one head, then masked attention for as many query blocks of
    that head as fit in the time budget.  Value in the metric's unit (TFLOP/s on
    kept tiles, i.e. 4 * 64 * 64 * D flops per kept tile)."""
    import numpy as np
    from oracle import nabla_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count()
    q, k, v = x["q"][:, :1], x["k"][:, :1], x["v"][:, :1]
    D = q.shape[-1]
    t0 = time.perf_counter()
    M, C, _ = orc.nabla_mask(q, k, thr)
    t_mask = time.perf_counter() - t0
    nb = M.shape[-1]
    order = np.random.default_rng(0).permutation(nb)
    done_tiles, spent, nblk = 0, 0.0, 0
    step = 2
    while spent < budget_s and nblk < nb:
        sel = order[nblk:nblk + step]
        Ms = np.zeros_like(M)
        Ms[0, 0, sel] = M[0, 0, sel]
        t0 = time.perf_counter()
        orc.masked_attention(q, k, v, Ms)
        spent += time.perf_counter() - t0
        done_tiles += int(Ms.sum())
        nblk += step
        step = min(step * 2, 64)
    flops = done_tiles * 4 * 64 * 64 * D
    mask_bytes = q.numel() * q.element_size() * 2
    heads = heads_total or x["q"].shape[0] * x["q"].shape[1]
    full_s = heads * (t_mask + spent / nblk * nb)
    return {"value": flops / spent / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "full_config_extrapolated_s": full_s,
            "full_config_note": "one head's mask time plus its attention time per query block, scaled "
                                "linearly to every query block and head of the problem",
            "sample": f"head 0 of {tuple(x['q'].shape)}: full fp64 mask ({t_mask:.2f} s, "
                      f"{mask_bytes / t_mask / 1e9:.3f} GB/s of Q+K), masked attention for {nblk} of {nb} "
                      f"query blocks ({done_tiles} kept tiles, {spent:.2f} s)",
            "host_cpus": os.cpu_count()}


def cpu_baseline_legs(main_rate_tflops: float, sweep=None, table1=None) -> dict:
    """The fp64 oracle, as it stands, timed beside the other legs on bounded
    samples of their workloads (a few seconds each), each extrapolated to the
    leg's full problem and labelled; part of the CPU-baseline leg."""
    import numpy as np
    import synth
    from oracle import nabla_oracle as orc
    out = {}
    # backward at the pretraining shape: one (b, h) in full
    w = synth.WORKLOADS[4]
    x = synth.make_inputs(w, heads=[0])
    sl = (slice(0, 1), slice(0, 1))
    M, _, _ = orc.nabla_mask(x["q"][sl], x["k"][sl], w.thresholds[0])
    t0 = time.perf_counter()
    orc.masked_attention_bwd(x["q"][sl], x["k"][sl], x["v"][sl], x["do"][sl], M)
    t = time.perf_counter() - t0
    kept = int(M.sum())
    out["training_backward"] = {
        "tflops": kept * 10 * 64 * 64 * w.D / t / 1e12, "full_config_extrapolated_s": t * w.B * w.H,
        "sample": f"(b, h) = (0, 0) of the pretraining shape: fp64 backward under its mask ({kept} kept tiles, "
                  f"{t:.2f} s), scaled to {w.B * w.H} heads"}
    # Eq. 1 projection with the pooling: 256 tokens of the 720p shape, C = 5120
    S_s, S_full, C, H, D = 256, 75600, 5120, 40, 128
    pi = synth.make_projection_inputs(1, S_s, C, H, D, seed=3)
    t0 = time.perf_counter()
    Q, K, V = orc.qkv_project(pi["x"], pi["wt"], H, D)
    orc.block_pool(orc.round_bf16(Q)), orc.block_pool(orc.round_bf16(K))
    t = time.perf_counter() - t0
    out["projection"] = {
        "tflops": 2.0 * S_s * C * 3 * H * D / t / 1e12, "full_config_extrapolated_s": t * S_full / S_s,
        "sample": f"{S_s} tokens of X [1, {S_full}, {C}] x W [{C}, 3 x {H * D}] in fp64 with the block means "
                  f"of Q and K ({t:.2f} s), scaled to {S_full} tokens"}
    # fractal reorder: the 720p latent with 64 fp32 channels (256-byte rows),
    # scaled by row bytes to the 5120 bf16 channels of the GPU leg
    T, Hl, Wl, P, ch = 21, 45, 80, 8, 64
    a = np.random.default_rng(0).standard_normal((1, T * Hl * Wl, ch)).astype(np.float32)
    t0 = time.perf_counter()
    orc.fractal_reorder(a, T, Hl, Wl, P)
    t = time.perf_counter() - t0
    out["fractal_reorder"] = {
        "full_config_extrapolated_s": t * (5120 * 2) / (ch * 4),
        "sample": f"[1, {T}x{Hl}x{Wl}, {ch}] fp32 rows gathered ({t:.3f} s), scaled by bytes to {5120} "
                  f"bf16 channels"}
    # block fidelity: four query blocks of head 0 at the 720p shape
    w3 = synth.WORKLOADS[WORKLOAD_ID]
    x3 = synth.make_inputs(w3, heads=[0])
    blocks = [0, 300, 700, w3.nb - 1]
    t0 = time.perf_counter()
    orc.block_mass_rows(x3["q"], x3["k"], 0, 0, blocks)
    t = time.perf_counter() - t0
    out["block_fidelity"] = {
        "full_config_extrapolated_s": t / len(blocks) * w3.nb * w3.H,
        "sample": f"block mass of {len(blocks)} query blocks of head 0 ({t:.2f} s), scaled to "
                  f"{w3.nb} blocks x {w3.H} heads"}
    # the sweeps and Table 1 run the main leg's kernels on other masks: their
    # oracle time follows from the main leg's oracle rate on kept tiles
    def derived(rows):
        return [{"thr": r.get("thr"), "method": r.get("method"),
                 "oracle_s_extrapolated": r["attn_tflops"] * r["attn_ms"] * 1e-3 / main_rate_tflops}
                for r in rows]
    if sweep:
        out["sweep"] = {"note": "kept-tile flops / the main leg's oracle rate", "cases": derived(sweep["cases"])}
    if table1:
        out["table1"] = {"note": "kept-tile flops / the main leg's oracle rate", "cases": derived(table1["cases"])}
    return out


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[WORKLOAD_ID]
    x = synth.make_inputs(w, heads=[0])
    budget = 4.0
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are not run
    vals = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(x, THR, budget_s=budget, heads_total=w.B * w.H))
    elapsed = time.perf_counter() - t_all
    v = statistics.median(r["value"] for r in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w, args.gpus), "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def measure_training(dev, warmup: int, steps: int) -> dict:
    """The training leg: mask (with the transposed lists), forward and backward
    at the pretraining shape (B=2, H=16, S=16,384, D=128, bf16, thr 0.8), each
    timed with CUDA events on the launching stream.  The forward runs in
    residual mode (o_res: the backward takes rowsum(dO * O) from o + o_res);
    the plain forward (no residual) is timed beside it for its cost.  Backward
    flops are the algorithmic 10 * 64 * 64 * D per kept tile (five GEMMs)."""
    import torch

    import block_sparse_attention_nabla_b200 as nabla
    import synth
    w = synth.WORKLOADS[4]
    x = synth.make_inputs(w)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, S, D = q.shape
    ws = nabla.workspace(q, want_bwd=True)
    mask = nabla.Mask.empty(B, H, S, dev, transpose=True)
    o, lse = torch.empty_like(q), torch.empty(B, H, S, dtype=torch.float32, device=dev)
    o_res = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        nabla.build_mask(q, k, w.thresholds[0], out=mask, ws=ws, transpose=True)
        if ev:
            ev[1].record(stream)
        nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws, o_res=o_res)
        if ev:
            ev[2].record(stream)
        nabla.attn_bwd(q, k, v, o, do, lse, mask, dq=dq, dk=dk, dv=dv, ws=ws, o_res=o_res)
        if ev:
            ev[3].record(stream)
        nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws)
        if ev:
            ev[4].record(stream)

    for _ in range(max(warmup, 1)):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    if nabla.workspace_status(ws) != 0:
        raise SystemExit("device status word reports a timeout in the training leg")
    mask_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    fwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    fwd_plain_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
    kept = int(mask.cnt.to(torch.int64).sum().item())
    nb = mask.cnt.shape[-1]
    peaks = _peaks()
    bwd_tflops = kept * 10 * 64 * 64 * D / (bwd_ms * 1e-3) / 1e12
    fwd_tflops = kept * 4 * 64 * 64 * D / (fwd_ms * 1e-3) / 1e12
    return {"workload": f"{w.name}: B={B} H={H} S={S} D={D} bf16, thr {w.thresholds[0]}, fwd + bwd with dO",
            "kept_fraction": kept / (B * H * nb * nb), "kept_tiles": kept, "steps": steps,
            "mask_ms": mask_ms, "fwd_ms": fwd_ms, "fwd_tflops": fwd_tflops,
            "fwd_mode": "residual (o_res written; P V with P in two bf16 terms)",
            "fwd_plain_ms": fwd_plain_ms, "fwd_plain_tflops": kept * 4 * 64 * 64 * D / (fwd_plain_ms * 1e-3) / 1e12,
            "bwd_ms": bwd_ms, "bwd_tflops": bwd_tflops,
            "bwd_roofline": {"bound": "tensor", "kernels": "bwd_stats + dkdv_tc + dq_tc (attn_bwd_tc.cu)",
                             "achieved": bwd_tflops, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                             "frac": bwd_tflops / peaks["bf16_sus"],
                             "algorithmic": "kept tiles x 10*64*64*D flops per call (executed: 14*64*64*D)"},
            "gpu_launches_per_step": 10}


def builder_bytes(B: int, H: int, S: int, D: int, elem: int, kept_tiles: int) -> int:
    """Algorithmic bytes of one mask build: Q and K read once, and the bitmask,
    the counts, the kept key-block indices and the work list written."""
    nb = -(-S // 64)
    W = -(-nb // 32)
    return 2 * B * H * S * D * elem + B * H * nb * (W * 4 + 4) + kept_tiles * 4 + B * H * -(-nb // 2) * 8


def oracle_sample_ms(x: dict, thr: float, budget_s: float) -> dict:
    """The fp64 oracle, as it stands, on head 0 of inputs x: its full mask, then
    masked attention for as many query blocks as fit in budget_s, extrapolated
    to all heads and query blocks of the workload (labelled as such)."""
    import numpy as np
    from oracle import nabla_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count()
    B, H, S, D = x["q"].shape
    q, k, v = x["q"][:1, :1], x["k"][:1, :1], x["v"][:1, :1]
    t0 = time.perf_counter()
    M, _, _ = orc.nabla_mask(q, k, thr)
    t_mask = time.perf_counter() - t0
    nb = M.shape[-1]
    order = np.random.default_rng(0).permutation(nb)
    spent, done = 0.0, 0
    step = 2
    while spent < budget_s and done < nb:
        sel = order[done:done + step]
        Ms = np.zeros_like(M)
        Ms[0, 0, sel] = M[0, 0, sel]
        t0 = time.perf_counter()
        orc.masked_attention(q, k, v, Ms)
        spent += time.perf_counter() - t0
        done += len(sel)
        step = min(step * 2, 64)
    attn_ms = spent / done * nb * B * H * 1e3
    mask_ms = t_mask * B * H * 1e3
    return {"mask_ms": mask_ms, "attn_ms": attn_ms, "cores": threads, "host_cpus": os.cpu_count(),
            "sample": f"head 0: full fp64 mask ({t_mask:.2f} s), attention for {done} of {nb} query blocks "
                      f"({spent:.2f} s); both extrapolated linearly to {B * H} heads"
                      + ("" if done < nb or B * H > 1 else " (complete)")}


def measure_config(nabla, dev, wid: int, warmup: int, steps: int, oracle_budget_s: float = 3.0) -> dict:
    """One workload at every threshold it names: per threshold the kept
    fraction, mask-build ms and GB/s (algorithmic bytes, builder_bytes), and
    attention ms and TFLOP/s on kept tiles (CUDA events on the launching
    stream), each as a fraction of the measured peaks; next to them the fp64
    oracle's time for the same workload on the host's cores (bounded sample,
    extrapolated)."""
    import torch
    import synth
    w = synth.WORKLOADS[wid]
    x = synth.make_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    B, H, S, D = q.shape
    elem = q.element_size()
    ws = nabla.workspace(q)
    mask = nabla.Mask.empty(B, H, S, dev, transpose=False)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    peaks = _peaks()
    rows = []
    for thr in w.thresholds:
        def one(ev=None):
            if ev:
                ev[0].record(stream)
            nabla.build_mask(q, k, thr, out=mask, ws=ws, transpose=False)
            if ev:
                ev[1].record(stream)
            nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws)
            if ev:
                ev[2].record(stream)

        for _ in range(max(warmup, 1)):
            one()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in evs:
            one(e)
        torch.cuda.synchronize()
        if nabla.workspace_status(ws) != 0:
            raise SystemExit(f"device status word reports a timeout in the {w.name} leg")
        kept = int(mask.cnt.to(torch.int64).sum().item())
        nb = mask.cnt.shape[-1]
        mask_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        tflops = kept * 4 * 64 * 64 * D / (attn_ms * 1e-3) / 1e12
        gbs = builder_bytes(B, H, S, D, elem, kept) / (mask_ms * 1e-3) / 1e9
        row = {"thr": thr, "kept_fraction": kept / (B * H * nb * nb), "kept_tiles": kept,
               "mask_ms": mask_ms, "mask_gbs": gbs, "mask_frac_hbm": gbs / peaks["hbm"],
               "attn_ms": attn_ms, "attn_tflops": tflops}
        if w.dtype == "bf16":
            row["attn_frac_bf16_sustained"] = tflops / peaks["bf16_sus"]
        else:
            # CUDA-core fp32 path: nominal fp32 FMA rate of 148 SMs x 128 lanes x 2 flops at 1.965 GHz
            row["attn_frac_fp32_nominal"] = tflops / (148 * 128 * 2 * 1.965e9 / 1e12)
        rows.append(row)
    out = {"workload": f"{w.name}: B={B} H={H} S={S} D={D} {w.dtype}, {w.T}x{w.Hl}x{w.Wl} tokens",
           "steps": steps, "cases": rows,
           "oracle": oracle_sample_ms(x, w.thresholds[0], oracle_budget_s)}
    del q, k, v
    return out


def measure_sweep(nabla, q, k, v, coords, warmup: int, steps: int, with_sta: bool = True,
                  inputs: str = "same inputs as the main line") -> dict:
    """The sparsity sweep at the 720p shape (thresholds 0.5 ... 1.0, the last
    the dense path) and, with_sta, the threshold-0.8 mask OR-ed with the STA
    window of 3 x 3 x 3 tiles: per case the kept fraction, mask-build and
    attention ms/call and the attention TFLOP/s on kept tiles (CUDA events on
    the launching stream)."""
    import torch
    B, H, S, D = q.shape
    ws = nabla.workspace(q)
    mask = nabla.Mask.empty(B, H, S, q.device, transpose=False)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream()
    rows = []
    cases = [(t, False) for t in (0.5, 0.7, 0.8, 0.9, 0.95, 1.0)] + ([(0.8, True)] if with_sta else [])
    for thr, sta in cases:
        kw = dict(sta_coords=coords, sta_window=(3, 3, 3)) if sta else {}

        def one(ev=None):
            if ev:
                ev[0].record(stream)
            nabla.build_mask(q, k, thr, out=mask, ws=ws, transpose=False, **kw)
            if ev:
                ev[1].record(stream)
            nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws)
            if ev:
                ev[2].record(stream)

        for _ in range(max(warmup, 1)):
            one()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in evs:
            one(e)
        torch.cuda.synchronize()
        if nabla.workspace_status(ws) != 0:
            raise SystemExit("device status word reports a timeout in the sweep")
        kept = int(mask.cnt.to(torch.int64).sum().item())
        nb = mask.cnt.shape[-1]
        attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        rows.append({"thr": thr, "sta": "3x3x3 tiles" if sta else None,
                     "kept_fraction": kept / (B * H * nb * nb),
                     "mask_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in evs), "attn_ms": attn,
                     "attn_tflops": kept * 4 * 64 * 64 * D / (attn * 1e-3) / 1e12})
    dense = next(r for r in rows if r["thr"] == 1.0)
    for r in rows:
        r["speedup_vs_dense"] = dense["attn_ms"] / r["attn_ms"]
    return {"workload": f"720p shape B={B} H={H} S={S} D={D} bf16, {inputs}",
            "steps": steps, "cases": rows}


def measure_sweep_sigma06(nabla, dev, warmup: int, steps: int) -> dict:
    """The same sweep on the 720p inputs drawn with block means and locality
    anchors of standard deviation 0.6 (same seed: the same noise, block
    structure scaled by 1.2), whose masks are as sparse as Table 1's NABLA
    rows (about 92 % at thr 0.7, 82 % at thr 0.8)."""
    import synth
    w = synth.WORKLOADS[7]
    x = synth.make_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    out = measure_sweep(nabla, q, k, v, None, warmup, steps, with_sta=False,
                        inputs=f"{w.name}: block means and anchors of std {w.sigma}, seed {w.seed}")
    del q, k, v
    return out


# Table 1 of the pages (§4.1): sparsity and whole-model inference time of
# Wan 2.1 14B at 720p on 4 x H100, printed beside this library's numbers for
# context only (another machine, another metric).
PAGES_TABLE1 = {"Baseline": (0.0, 8.35), "STA(18,40,40)": (79.45, 4.00), "NABLA(0.7)": (80.13, 4.02),
                "NABLA(0.5)+STA(11,40,40)": (81.0, 3.58), "STA(18,24,24)": (91.28, 3.08),
                "NABLA(0.4)": (92.5, 3.07), "NABLA(0.2)+STA(11,24,24)": (92.27, 3.13)}


def measure_table1(nabla, dev, warmup: int, steps: int, heads: int | None = None) -> dict:
    """The seven configurations of Table 1 on the padded 720p layout (21 x 48 x
    80 = 80,640 tokens, 21 x 6 x 10 tiles): the dense baseline (thr 1.0), STA
    alone (nabla_build_sta_mask), NABLA alone and NABLA + STA.  Per case the
    sparsity, mask-build and attention ms/call (CUDA events on the launching
    stream), attention TFLOP/s on kept tiles and the attention speed-up over
    the baseline."""
    import torch
    import synth
    w = synth.WORKLOADS[6]
    if heads:
        w = w.scaled(H=heads)
    x = synth.make_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    coords = nabla.sta_block_coords(w.T, w.Hl, w.Wl, w.P, w.S).to(dev)
    B, H, S, D = q.shape
    ws = nabla.workspace(q)
    mask = nabla.Mask.empty(B, H, S, dev, transpose=False)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    rows = []
    for name, thr, window in synth.TABLE1:
        tiles = synth.sta_tiles(window) if window else None

        def build():
            if thr is None:
                nabla.build_sta_mask(tuple(q.shape), coords, tiles, out=mask, transpose=False)
            else:
                nabla.build_mask(q, k, thr, sta_coords=coords if tiles else None, sta_window=tiles, out=mask,
                                 ws=ws, transpose=False)

        def one(ev=None):
            if ev:
                ev[0].record(stream)
            build()
            if ev:
                ev[1].record(stream)
            nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws)
            if ev:
                ev[2].record(stream)

        for _ in range(max(warmup, 1)):
            one()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in evs:
            one(e)
        torch.cuda.synchronize()
        if nabla.workspace_status(ws) != 0:
            raise SystemExit("device status word reports a timeout in the Table 1 leg")
        nb = mask.cnt.shape[-1]
        kept = int(mask.cnt.to(torch.int64).sum().item())
        attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        pages = PAGES_TABLE1[name]
        rows.append({"method": name, "thr": thr, "sta_window_tokens": window, "sta_window_tiles": tiles,
                     "kept_fraction": kept / (B * H * nb * nb), "sparsity_pct": 100.0 * (1 - kept / (B * H * nb * nb)),
                     "mask_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in evs), "attn_ms": attn,
                     "attn_tflops": kept * 4 * 64 * 64 * D / (attn * 1e-3) / 1e12,
                     "pages_sparsity_pct": pages[0], "pages_inference_min_4xH100": pages[1]})
    base = rows[0]["attn_ms"]
    for r in rows:
        r["attn_speedup_vs_baseline"] = base / r["attn_ms"]
    return {"workload": f"table1_720p_padded: B={B} H={H} S={S} D={D} bf16, 21x48x80 tokens (frames padded "
                        f"45 -> 48 rows), tiles 21x6x10",
            "steps": steps, "note": "pages_* = Table 1 of the pages (Wan 2.1 14B, 4 x H100, whole-model "
                                    "inference minutes): context only", "cases": rows}


def measure_fidelity(nabla, q, k) -> dict:
    """The per-block fidelity check at the 720p shape: the true token-level
    block mass of dense attention (block_mass_kernel, two dense passes of
    S = Q K^T: 4 S^2 D flops per head) and the kept mass (recall) of the CDF
    masks at thr 0.5 and 0.8 against fixed-budget Top-k masks with the same
    mean number of blocks per row."""
    import torch
    B, H, S, D = q.shape
    ws = torch.zeros(256, dtype=torch.uint8, device=q.device)
    A = nabla.block_mass(q, k, ws=ws)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    nabla.block_mass(q, k, out=A, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    if nabla.workspace_status(ws) != 0:
        raise SystemExit("device status word reports a timeout in the block-mass kernel")
    ms = e0.elapsed_time(e1)
    rows = []
    for thr in (0.5, 0.8):
        cdf = nabla.build_mask(q, k, thr, transpose=False)
        budget = int(round(cdf.cnt.float().mean().item()))
        tk = nabla.build_mask_topk(q, k, budget, transpose=False)
        rc = nabla.mask_recall(A, cdf, tuple(q.shape))
        rt = nabla.mask_recall(A, tk, tuple(q.shape))
        nb = cdf.cnt.shape[-1]
        rows.append({"thr": thr, "topk_budget": budget,
                     "kept_fraction_cdf": cdf.cnt.float().mean().item() / nb,
                     "kept_fraction_topk": tk.cnt.float().mean().item() / nb,
                     "recall_cdf_mean": rc.mean().item(), "recall_cdf_min": rc.min().item(),
                     "recall_topk_mean": rt.mean().item(), "recall_topk_min": rt.min().item(),
                     "rows_cdf_better": (rc > rt).float().mean().item()})
    flops = 4.0 * B * H * S * S * D
    return {"workload": f"720p shape B={B} H={H} S={S} D={D} bf16, same inputs as the main line",
            "block_mass_ms": ms, "block_mass_tflops": flops / (ms * 1e-3) / 1e12,
            "kernel": "block_mass_kernel<128> (fidelity.cu)", "cases": rows}


def measure_reorder(nabla, dev, warmup: int, steps: int) -> dict:
    """Fractal token reordering (§3.1.1) of [B, T*H*W, C] activations at the
    720p latent (T=21, H=45, W=80, P=8) with C = 5120 bf16 channels, forward and
    inverse; HBM-bound: every row read once and written once (2 x 774 MB per
    call; inputs larger than L2)."""
    import torch
    T, H, W, P, C = 21, 45, 80, 8, 5120
    x = torch.randn(1, T * H * W, C, device=dev, dtype=torch.bfloat16)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    res = {}
    peaks = _peaks()
    for inv in (False, True):
        for _ in range(max(warmup, 1)):
            nabla.fractal_reorder(x, T, H, W, P, inverse=inv, out=y)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            nabla.fractal_reorder(x, T, H, W, P, inverse=inv, out=y)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        gbs = 2 * x.numel() * x.element_size() / (ms * 1e-3) / 1e9
        res["inverse" if inv else "forward"] = {"ms": ms, "gbs": gbs, "frac_hbm": gbs / peaks["hbm"]}
    return {"workload": f"[1, {T}x{H}x{W}, {C}] bf16, P={P}", "bytes_per_call": 2 * x.numel() * x.element_size(),
            "kernel": "reorder_kernel (reorder.cu)", **res}


def measure_projection(nabla, dev, warmup: int, steps: int, heads: int | None = None) -> dict:
    """Eq. 1 projection with the block pooling fused (NEXT-4): Q, K, V = X W
    at the 720p shape (B=1, S=75,600, C=5120, H=40, D=128) from hidden states
    with per-block means and N(0, 1/C) weights drawn on the GPU.  Reports the
    fused kernel (tensor-bound: 2 S C (3 H D) flops; timed alone, so against
    the burst bf16 peak), a library GEMM of the same product for context, and
    the mask build from the fused means against the build that pools Q and K
    itself.  heads (profiling only) keeps C and S and projects onto fewer heads."""
    import torch
    import synth
    B, H, S, D, C = 1, heads or 40, 75600, 128, 5120
    d = synth.make_projection_inputs(B, S, C, H, D, seed=3, device=dev)
    x, wt = d["x"], d["wt"]
    q, k, v, ws = nabla.qkv_project(x, wt, H, D)
    mask = nabla.build_mask_pooled(q.shape, THR, ws, transpose=False)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(max(warmup, 1)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    flops = 2.0 * B * S * C * 3 * H * D
    proj_ms = timed(lambda: nabla.qkv_project(x, wt, H, D, q, k, v, ws), steps)
    if nabla.workspace_status(ws) != 0:
        raise SystemExit("device status word reports a timeout in the projection leg")
    pooled_ms = timed(lambda: nabla.build_mask_pooled(q.shape, THR, ws, out=mask, transpose=False), steps)
    ws2 = nabla.workspace(q)
    direct_ms = timed(lambda: nabla.build_mask(q, k, THR, out=mask, ws=ws2, transpose=False), steps)
    out = torch.empty(B * S, 3 * H * D, dtype=torch.bfloat16, device=dev)
    lib_ms = timed(lambda: torch.matmul(x.reshape(B * S, C), wt.reshape(3 * H * D, C).t(), out=out), steps)
    if nabla.workspace_status(ws) != 0 or nabla.workspace_status(ws2) != 0:
        raise SystemExit("device status word reports a timeout in the projection leg")
    peaks = _peaks()
    tflops = flops / (proj_ms * 1e-3) / 1e12
    res = {"workload": f"X [{B}, {S}, {C}] x W [{C}, 3 x {H * D}] bf16 -> Q, K, V [{B}, {H}, {S}, {D}] "
                       f"+ block means of Q, K; thr {THR} for the builds",
           "kernel": "qkv_project_kernel (qkv_tc.cu)", "ms": proj_ms, "tflops": tflops,
           "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16"], "unit": "TFLOP/s",
                        "frac": tflops / peaks["bf16"],
                        "peak_note": f"{peaks['source']} burst bf16 (kernel timed alone)",
                        "traffic": _traffic("qkv_tc.cu") if H == 40 else None,
                        "algorithmic": "2 * B * S * C * 3 * H * D flops per launch"},
           "library_gemm_ms": lib_ms, "library_gemm_tflops": flops / (lib_ms * 1e-3) / 1e12,
           "library_gemm_note": "torch.matmul (cuBLAS) of the same product into [B*S, 3*H*D], no pooling",
           "mask_build_from_fused_means_ms": pooled_ms, "mask_build_from_q_k_ms": direct_ms}
    del x, wt, q, k, v, ws, ws2, out, mask
    torch.cuda.empty_cache()
    return res


def _config(w, n) -> dict:
    return {"workload": f"{w.name}: B={w.B} H={w.H} S={w.S} D={w.D} bf16, {w.T}x{w.Hl}x{w.Wl} tokens, "
                        f"thr {THR}, no STA",
            "B": w.B, "H": w.H, "S": w.S, "D": w.D, "thr": THR, "sta": None,
            "global_batch": w.B * n, "seq_len": w.S,
            "parallelism": f"{n} independent problems, one per GPU" if n > 1 else "single GPU",
            "l2": "inputs larger than L2 (Q, K, V = 2.32 GB per problem)"}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="nabla", choices=["nabla", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-training", action="store_true", help="skip the forward + backward training leg")
    ap.add_argument("--no-sweep", action="store_true", help="skip the threshold sweep and the STA case")
    ap.add_argument("--only-training", action="store_true",
                    help="run only the training leg and print its object (profiling; not a bench line)")
    ap.add_argument("--only-reorder", action="store_true",
                    help="run only the fractal-reorder leg and print its object (profiling; not a bench line)")
    ap.add_argument("--only-table1", action="store_true",
                    help="run only the Table 1 configurations (padded 720p layout) and print their JSON")
    ap.add_argument("--only-sweep", action="store_true",
                    help="run only the two threshold sweeps and print their JSON (not a bench line)")
    ap.add_argument("--only-fidelity", action="store_true",
                    help="run only the block-fidelity leg and print its object (profiling; not a bench line)")
    ap.add_argument("--only-projection", action="store_true",
                    help="run only the fused projection leg and print its object (profiling; not a bench line)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the head count (smaller cases for ncu captures; not a bench line)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return

    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_attention_nabla_b200 as nabla
    import synth

    if args.only_training:
        import torch
        torch.cuda.set_device(0)
        print(json.dumps(measure_training(torch.device("cuda", 0), args.warmup, max(1, args.steps))), flush=True)
        return
    if args.only_reorder:
        torch.cuda.set_device(0)
        print(json.dumps(measure_reorder(nabla, torch.device("cuda", 0), args.warmup, max(1, args.steps))), flush=True)
        return
    if args.only_table1:
        torch.cuda.set_device(0)
        print(json.dumps(measure_table1(nabla, torch.device("cuda", 0), max(1, args.warmup), max(1, args.steps),
                                        args.heads)), flush=True)
        return
    if args.only_sweep:
        torch.cuda.set_device(0)
        dev0 = torch.device("cuda", 0)
        ws_ = synth.WORKLOADS[WORKLOAD_ID]
        xs = synth.make_inputs(ws_)
        qs, ks, vs = (xs[n].to(dev0) for n in ("q", "k", "v"))
        first = measure_sweep(nabla, qs, ks, vs, nabla.sta_block_coords(ws_.T, ws_.Hl, ws_.Wl, ws_.P, ws_.S).to(dev0), max(1, args.warmup),
                              max(1, args.steps))
        del qs, ks, vs
        print(json.dumps({"sweep": first, "sweep_sigma06": measure_sweep_sigma06(
            nabla, dev0, max(1, args.warmup), max(1, args.steps))}), flush=True)
        return
    if args.only_projection:
        torch.cuda.set_device(0)
        print(json.dumps(measure_projection(nabla, torch.device("cuda", 0), max(1, args.warmup),
                                            max(1, args.steps), args.heads)), flush=True)
        return
    if args.only_fidelity:
        torch.cuda.set_device(0)
        wf = synth.WORKLOADS[WORKLOAD_ID]
        if args.heads:
            wf = wf.scaled(H=args.heads)
        xf = synth.make_inputs(wf)
        print(json.dumps(measure_fidelity(nabla, xf["q"].cuda(), xf["k"].cuda())), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    w = synth.WORKLOADS[WORKLOAD_ID]
    if args.heads:
        w = w.scaled(H=args.heads, name=f"{w.name}_h{args.heads}")
    wr = rank_workload(w, rank)
    x = synth.make_inputs(wr)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    B, H, S, D = q.shape
    ws = nabla.workspace(q)
    mask = nabla.Mask.empty(B, H, S, dev, transpose=False)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        nabla.build_mask(q, k, THR, out=mask, ws=ws, transpose=False)
        if ev:
            ev[1].record(stream)
        nabla.attn_fwd(q, k, v, mask, o=o, lse=lse, ws=ws)
        if ev:
            ev[2].record(stream)

    # the clock sampler starts before the warm-up (so that its start-up adds no
    # idle gap before the timed region) and keeps the samples of the region
    with ClockSampler(local) as clocks:
        for _ in range(max(args.warmup, 0)):
            step()
        torch.cuda.synchronize()
        if nabla.workspace_status(ws) != 0:
            raise SystemExit("device status word reports a timeout in warm-up")

        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks.mark_start()
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    mask_ms = [e[0].elapsed_time(e[1]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    if nabla.workspace_status(ws) != 0:
        raise SystemExit("device status word reports a timeout")

    total_ms, attn_avg, mask_avg = max_over_ranks(
        [total_ms, statistics.mean(attn_ms), statistics.mean(mask_ms)], dist if world > 1 else None, dev)

    kept_tiles = int(mask.cnt.to(torch.int64).sum().item())
    nb = mask.cnt.shape[-1]
    kept_frac = kept_tiles / (B * H * nb * nb)
    # tiles the kernel executes: a unit of two query blocks computes the union
    # of their kept lists at M = 128, i.e. two 64 x 64 tiles per union entry
    union_tiles = 2 * int(mask.work[:, 1].to(torch.int64).sum().item())
    flops = kept_tiles * 4 * 64 * 64 * D                     # per problem, tile basis
    ms_step = total_ms / args.steps
    value = job_tflops(world, flops, ms_step)
    attn_tflops = flops / (attn_avg * 1e-3) / 1e12
    mask_bytes = builder_bytes(B, H, S, D, q.element_size(), kept_tiles)
    mask_gbs = mask_bytes / (mask_avg * 1e-3) / 1e9
    peaks = _peaks()

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(nabla, q, k, v, o, lse, mask, ws, stream, args, world, dist, dev, flops)

    training = None
    if world == 1 and not args.no_training:
        training = measure_training(dev, args.warmup, max(1, min(args.steps, 5)))

    reorder = None
    if world == 1 and not args.no_sweep:
        reorder = measure_reorder(nabla, dev, 3, 10)

    projection = None
    if world == 1 and not args.no_sweep:
        projection = measure_projection(nabla, dev, 3, 10)

    fidelity = None
    if world == 1 and not args.no_sweep:
        fidelity = measure_fidelity(nabla, q, k)

    sweep = None
    if world == 1 and not args.no_sweep:
        sweep = measure_sweep(nabla, q, k, v, nabla.sta_block_coords(w.T, w.Hl, w.Wl, w.P, w.S).to(dev), 1, 2)

    sweep06 = None
    if world == 1 and not args.no_sweep:
        sweep06 = measure_sweep_sigma06(nabla, dev, 1, 2)

    table1 = None
    if world == 1 and not args.no_sweep:
        table1 = measure_table1(nabla, dev, 1, 2)

    configs = None
    if world == 1 and not args.no_sweep:
        configs = {"tiny_fp32": measure_config(nabla, dev, 1, 3, 5),
                   "fwd_480p": measure_config(nabla, dev, 2, 2, 5)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": _config(w, world),
            "attn_ms_per_call": attn_avg, "attn_tflops_actual": attn_tflops,
            "attn_frac_of_bf16_peak": attn_tflops / peaks["bf16_sus"],
            "mask_build_ms": mask_avg, "mask_build_gbs": mask_gbs, "mask_build_frac_hbm": mask_gbs / peaks["hbm"],
            "kept_fraction": kept_frac, "kept_tiles": kept_tiles,
            "executed_tiles": union_tiles, "union_efficiency": kept_tiles / union_tiles,
            "attn_tflops_executed": union_tiles * 4 * 64 * 64 * D / (attn_avg * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "fwd_tc_kernel<128> (attn_fwd_tc.cu)",
                         "achieved": attn_tflops, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                         "frac": attn_tflops / peaks["bf16_sus"],
                         "peak_note": f"{peaks['source']} sustained bf16 (kernel timed inside a long step); "
                                      f"burst {peaks['bf16']}",
                         "traffic": _traffic("attn_fwd_tc.cu"),
                         "algorithmic": "kept tiles x 4*64*64*D flops per launch"},
            "mask_roofline": {"bound": "hbm", "kernels": "pool + score GEMM + select + work list",
                              "achieved": mask_gbs, "peak": peaks["hbm"], "unit": "GB/s",
                              "frac": mask_gbs / peaks["hbm"], "bytes_per_call": mask_bytes,
                              "ms_per_call": mask_avg,
                              "traffic": _builder_traffic() if (H, S) == (40, 75600) else None,
                              "algorithmic": "Q + K read once; bitmask, counts, kept indices, work list written"},
            "e2e": e2e,
            "configs": configs,
            "training": training,
            "sweep": sweep,
            "sweep_sigma06": sweep06,
            "table1": table1,
            "fractal_reorder": reorder,
            "projection": projection,
            "fidelity": fidelity,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline({n: x[n][:, :1] for n in ("q", "k", "v")}, THR,
                                                heads_total=B * H)
            try:
                line["cpu_baseline"]["legs"] = cpu_baseline_legs(line["cpu_baseline"]["value"], sweep, table1)
            except Exception as e:  # a host-side sample must not cost the bench line
                line["cpu_baseline"]["legs"] = {"error": f"{type(e).__name__}: {e}"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(nabla, q, k, v, o, lse, mask, ws, stream, args, world, dist, dev, flops):
    """Same step through the public API with every step's inputs copied in
    from pinned host memory and its output copied back, all inside the timed
    region.  Uploads and downloads run on two more streams with double-buffered
    device tensors, so step i + 1's inputs travel while step i computes and
    step i's output travels while step i + 1 computes; the compute stream runs
    the steps in order.  The region starts before the first upload and ends
    after the last download."""
    import torch
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    bufs = [[torch.empty_like(t) for t in (q, k, v)] for _ in range(2)]
    outs = [torch.empty_like(o) for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n = max(2, args.steps)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    copied, done, fetched = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    down.wait_event(e0)
    for i in range(n):
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(done[i - 2])            # step i - 2 finished reading buffer b
            for dst, src in zip(bufs[b], (hq, hk, hv)):
                dst.copy_(src, non_blocking=True)
            copied[i].record(up)
        stream.wait_event(copied[i])
        if i >= 2:
            stream.wait_event(fetched[i - 2])         # output buffer b copied back
        dq_, dk_, dv_ = bufs[b]
        m2 = nabla.build_mask(dq_, dk_, THR, out=mask, ws=ws, transpose=False)
        nabla.attn_fwd(dq_, dk_, dv_, m2, o=outs[b], lse=lse, ws=ws)
        done[i].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(done[i])
            ho.copy_(outs[b], non_blocking=True)
            fetched[i].record(down)
    up.wait_event(fetched[n - 1])
    e1.record(up)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n
    e2e_ms = max_over_ranks([e2e_ms], dist if world > 1 else None, dev)[0]
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size()
    return {"value": job_tflops(world, flops, e2e_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n,
            "overlap": "uploads and downloads on two more streams, inputs and outputs double-buffered"}


if __name__ == "__main__":
    main()

"""Benchmark: block-sparse attention layer path on B200, one JSON line on rank 0.

A step is one pass of the whole hot path over one layer of the video-DiT-small-like
workload (B=1 per GPU, 12 heads, head dim 128, latent grid 21x30x52 = 32,760 tokens padded to
32,768, 1x8x16 tiles, 128x128 blocks, +-1 latent-frame window + 4 rotating anchor blocks):
tile reorder of Q, K and V, CSR build for denoising step s = k mod 50, block-sparse
attention, inverse reorder of O.  Inputs (302 MB of Q/K/V, larger than the 126 MB L2) are
resident in HBM before the timed region.

  value      effective TFLOP/s over active blocks (4*Bs^2*d per active block pair and head)
             for the whole step, summed over ranks, divided by the max-over-ranks time.
  roofline   the attention kernel alone (CUDA events on its launch stream).
  e2e        the same metric through the public API with pinned host buffers: H2D of
             Q/K/V and D2H of O and LSE inside the timed region.
  cpu_baseline  the FP64 oracle on a bounded, time-limited sample of the same workload.

``--impl reference`` times the oracle itself as the reference arm (rank 0 only).
Multi-GPU (torchrun): every rank runs its own batch element (``--shard batch``, weak
scaling), or one layer is split into contiguous head ranges (``--shard heads``, strong
scaling, the mask replicated).  Neither has a collective on the data path: a barrier and a
max-reduce of the timings only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synthetic import WORKLOADS, Workload, make_qkv, mask_variants  # noqa: E402

METRIC = "block-sparse attn effective TFLOP/s (active blocks) & % bf16 TC peak; ms/layer"
WORKLOAD = "small"
ATTN_SRC = os.path.join(ROOT, "block_sparse_attention_lva_b200", "csrc", "attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "bsa_fwd_small_traffic.json")
ATTN_KERNEL = "bsa_fwd_kernel<128,128>"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _workload_for_rank(rank: int) -> Workload:
    w = WORKLOADS[WORKLOAD]
    return Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def _config_dict(w: Workload, spec: dict, n_gpus: int, shard: str = "batch") -> dict:
    if shard == "heads":
        return {"workload": f"video-DiT-small-like: one layer (B=1, {w.H} heads) split by heads over {n_gpus} GPU(s), "
                            f"d={w.d}, latent grid {w.T}x{w.Hg}x{w.Wg}={w.n_valid} tokens padded to {w.n_pad}, "
                            f"tiles 1x8x16, {w.block_size}x{w.block_size} blocks, +-1 latent-frame window + 4 rotating "
                            f"anchor blocks, denoising step = step index mod 50",
                "global_batch": w.B, "heads": w.H, "head_dim": w.d, "seq_len": w.n_pad, "block": w.block_size,
                "step_contents": "per rank, its contiguous head range: reorder of stacked QKV + CSR build (3 "
                                 "launches, the mask replicated) + attention with the inverse reorder fused into "
                                 "its epilogue; no collective on the data path",
                "l2": "inputs larger than L2 at 1-2 GPUs (302 MB Q/K/V in all), no flush",
                "parallelism": f"heads{n_gpus} (contiguous head ranges of one layer)"}
    return {"workload": f"video-DiT-small-like: B=1 per GPU, {w.H} heads, d={w.d}, latent grid "
                        f"{w.T}x{w.Hg}x{w.Wg}={w.n_valid} tokens padded to {w.n_pad}, tiles 1x8x16, "
                        f"{w.block_size}x{w.block_size} blocks, +-1 latent-frame window + 4 rotating "
                        f"anchor blocks, denoising step = step index mod 50",
            "global_batch": n_gpus * w.B, "heads": w.H, "head_dim": w.d, "seq_len": w.n_pad,
            "block": w.block_size, "step_contents": "reorder of stacked QKV + CSR build (3 launches) + attention with the inverse reorder fused into its epilogue",
            "l2": "inputs larger than L2 (302 MB Q/K/V per GPU), no flush",
            "parallelism": f"dp{n_gpus} (independent batch elements)"}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def _traffic_per_launch():
    """DRAM bytes per attention launch from the committed ncu summary, if it matches the source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    sha = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()
    return d.get("bytes_per_launch") if d.get("attn_cu_sha256") == sha else None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_over_ranks(times, work, device, distributed: bool):
    """Max over ranks of each time, sum over ranks of the work (the only cross-rank traffic)."""
    t = torch.tensor(list(times), dtype=torch.float64, device=device)
    wk = torch.tensor([float(work)], dtype=torch.float64, device=device)
    if distributed:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(wk, op=dist.ReduceOp.SUM)
    return t.tolist(), wk.item()


def _flops_per_nnz(w: Workload) -> float:
    return 4.0 * w.block_size * w.block_size * w.d


def _nnz_table(layer, steps):
    """Active block pairs of the mask at each denoising step (read back outside timing)."""
    table = {}
    for s in steps:
        layer.build_mask(s)
        table[s] = int(layer.nnz.item())
    return table


def run_lva(args):
    import torch.distributed as dist

    import block_sparse_attention_lva_b200 as lva

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    spec = mask_variants(WORKLOADS[WORKLOAD])[0]
    n_steps_cycle = len(spec["steps"])
    if args.shard == "heads":
        # one layer, split into contiguous head ranges: every rank draws only its own heads
        w = WORKLOADS[WORKLOAD]
        h0, h1 = lva.head_range(w.H, ws, rank)
        heads = list(range(h0, h1))
    else:
        # every rank its own batch element (its own seed)
        w = _workload_for_rank(rank)
        heads = list(range(w.H))
    H_local = len(heads)
    q, k, v = make_qkv(w, heads=heads)
    # Q, K, V as one stacked raster buffer (as a fused QKV projection produces them).
    qkv = torch.stack([q, k, v]).to(dev)
    qd, kd, vd = qkv[0], qkv[1], qkv[2]
    layer = lva.VideoBlockSparseAttention(w.B, H_local, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                          scale=w.scale, device=dev)
    nnz = _nnz_table(layer, range(n_steps_cycle))
    fpn = _flops_per_nnz(w) * w.B * H_local      # mask_heads = 1: every head shares the CSR
    stream = torch.cuda.current_stream(dev)

    def step(kidx, ev=None):
        s = kidx % n_steps_cycle
        layer.reorder_in(qd, kd, vd)
        layer.build_mask(s)
        if ev is not None:
            ev[0].record(stream)
        layer.attend_to_raster()       # attention with the inverse reorder fused in
        if ev is not None:
            ev[1].record(stream)

    def barrier():
        if ws > 1:
            dist.barrier()

    for kk in range(args.warmup):
        step(kk)
    torch.cuda.synchronize()
    status, detail = lva.lva_device_error()
    if status != 0:
        raise RuntimeError(f"kernel error word {status} ({detail}) during warm-up")

    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    base = args.warmup
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for kk in range(args.steps):
            step(base + kk, attn_ev[kk])
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms_total = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in attn_ev]
    flops = sum(nnz[(base + kk) % n_steps_cycle] for kk in range(args.steps)) * fpn
    status, detail = lva.lva_device_error()
    if status != 0:
        raise RuntimeError(f"kernel error word {status} ({detail}) during timing")

    # ---------------- e2e through the public API with pinned host buffers
    qkvh = torch.stack([q, k, v]).pin_memory()
    oh = torch.empty((w.B, H_local, w.n_valid, w.d), dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((w.B, H_local, w.n_pad), dtype=torch.float32).pin_memory()

    last_done = [None]

    def e2e_step(kidx):
        # the public host-buffer call: copies of each head group overlap the other groups'
        # reorder + attention, and consecutive steps overlap through double-buffered device
        # buffers (see VideoBlockSparseAttention.forward_host); the timed region ends after
        # the last step's copies back have landed in host memory
        last_done[0] = layer.forward_host(qkvh, oh, lh, step=kidx % n_steps_cycle, wait=False)

    for kk in range(args.warmup):
        e2e_step(kk)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for kk in range(args.steps):
        e2e_step(base + kk)
    stream.wait_event(last_done[0])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1)
    h2d = qkvh.numel() * qkvh.element_size()
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    # ---------------- reduce over ranks (max time, summed work)
    (ms_total, ms_e2e, attn_ms_mean), flops_all = reduce_over_ranks(
        [ms_total, ms_e2e, float(np.mean(attn_ms))], flops, dev, ws > 1)

    if rank == 0:
        burst, sustained, hbm, peak_kind = _peaks()
        attn_flops_launch = flops / args.steps                   # this rank's mean per launch
        achieved = attn_flops_launch / (attn_ms_mean * 1e-3) / 1e12
        traffic = _traffic_per_launch()
        line = {
            "metric": METRIC, "value": flops_all / (ms_total * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_total / args.steps, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 Q/K/V)",
            "config": _config_dict(w, spec, ws, args.shard),
            "attn_ms_per_layer": attn_ms_mean,
            "active_block_pairs_per_head": {"min": min(nnz.values()), "max": max(nnz.values()),
                                             "density": float(np.mean(list(nnz.values()))) / w.nb ** 2},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                         "frac": achieved / burst, "traffic": traffic,
                         "peak_kind": f"{peak_kind} bf16 dense cuBLAS, burst",
                         "frac_of_sustained": achieved / sustained,
                         "sustained_note": "the sustained cuBLAS figure was measured at a lower SM clock "
                                           "under the power cap; the clocks below are those of this run",
                         "kernel": ATTN_KERNEL},
            "clocks": clocks.summary(),
            "e2e": {"value": flops_all / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e2e / args.steps},
            "gpu_launches": 5 * args.steps,
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, spec, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def _oracle_sample(w, spec, q, k, v, perm, seconds, seed):
    """Runs the oracle on seeded random (head, query block) items until `seconds` pass."""
    from oracle.attention import attention_blocked
    from oracle.mask import window_anchor_mask
    from oracle.reorder import reorder_forward

    rng = np.random.default_rng(seed)
    P = w.B * w.H
    tile = [torch.from_numpy(reorder_forward(x.view(torch.int16).reshape(P, w.n_valid, w.d).numpy(), perm, w.n_pad))
            .view(torch.bfloat16).reshape(w.B, w.H, w.n_pad, w.d) for x in (q, k, v)]
    s = int(rng.integers(0, len(spec["steps"])))
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"], spec["anchors"], s)
    flops, items = 0.0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds or items < 4:
        h, i = int(rng.integers(0, w.H)), int(rng.integers(0, w.nb))
        attention_blocked(tile[0][:, h:h + 1], tile[1][:, h:h + 1], tile[2][:, h:h + 1], m, w.block_size,
                          w.n_valid, w.scale, query_blocks=[(0, 0, i)])
        flops += int(m[i].sum()) * _flops_per_nnz(w)
        items += 1
    return flops, time.perf_counter() - t0, items


def _oracle_mask_for(w, spec, step=0):
    """Dense block mask [H_m, nb, nb] of a mask specification, from the oracle."""
    from oracle.mask import all_mask, lvsa_frame_mask, two_stage_mask, window_anchor_mask
    from synthetic import static_calibrated_mask
    kind = spec["kind"]
    if kind == "window_anchor":
        return window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"],
                                  spec["anchors"], step)[None]
    if kind == "two_stage":
        return two_stage_mask(w.nb, spec["group"])[None]
    if kind == "all":
        return all_mask(w.nb)[None]
    if kind == "lvsa_frames":
        return lvsa_frame_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["anchors"], step,
                               spec["budget"])[None]
    if kind == "static":
        return static_calibrated_mask(w, spec["density"]).astype(bool)
    raise ValueError(kind)


def run_oracle_report(args, gpu_ms):
    """The FP64 oracle timed per (workload, mask) on a seeded sample of (head, query block)
    items -- the first and last query block of every head, then random ones -- for about
    ``args.cpu_seconds`` / 4 each, extrapolated to the whole launch by active block pairs."""
    from oracle.attention import attention_blocked
    from oracle.reorder import reorder_forward, tile_permutation
    budget = max(2.0, args.cpu_seconds / 4)
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    for name in ("tiny", "small", "static", "large", "long"):
        w = WORKLOADS[name]
        q, k, v = make_qkv(w)
        perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
        P = w.B * w.H
        tile = [torch.from_numpy(reorder_forward(x.view(torch.int16).reshape(P, w.n_valid, w.d).numpy(), perm,
                                                 w.n_pad)).view(torch.bfloat16).reshape(w.B, w.H, w.n_pad, w.d)
                for x in (q, k, v)]
        for spec in mask_variants(w):
            m = _oracle_mask_for(w, spec)
            total_pairs = int(m.sum()) * (w.H if m.shape[0] == 1 else 1) * w.B
            rng = np.random.default_rng(11)
            order = [(h, 0) for h in range(w.H)] + [(h, w.nb - 1) for h in range(w.H)]
            flops, items = 0.0, 0
            t0 = time.perf_counter()
            while (time.perf_counter() - t0 < budget or items < 4) and items < w.H * w.nb:
                h, i = order[items] if items < len(order) else (int(rng.integers(0, w.H)), int(rng.integers(0, w.nb)))
                hm = h if m.shape[0] > 1 else 0
                attention_blocked(tile[0][:, h:h + 1], tile[1][:, h:h + 1], tile[2][:, h:h + 1], m[hm:hm + 1],
                                  w.block_size, w.n_valid, w.scale, query_blocks=[(0, 0, i)])
                flops += int(m[hm, i].sum()) * _flops_per_nnz(w)
                items += 1
            secs = time.perf_counter() - t0
            rate = flops / secs
            full_s = total_pairs * _flops_per_nnz(w) / rate
            line = {"report": "oracle", "workload": name, "mask": spec["label"], "sample_items": items,
                    "sample_s": secs, "oracle_tflops": rate / 1e12, "cores": _threads(), "cpu_model": model,
                    "full_launch_s_extrapolated": full_s}
            ms = gpu_ms.get((name, spec["label"]))
            if ms:
                line["gpu_attn_ms"] = ms
                line["speedup_vs_oracle"] = full_s * 1e3 / ms
            print(json.dumps(line), flush=True)


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, spec, seconds):
    from oracle.reorder import tile_permutation
    q, k, v = make_qkv(w)
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    flops, secs, items = _oracle_sample(w, spec, q, k, v, perm, seconds, seed=7)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{items} random (head, query block) items of the same workload (one denoising step's "
                      f"mask), {secs:.1f} s of FP64 numpy/BLAS work; the whole step is attention-dominated"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    from oracle.reorder import tile_permutation
    w = _workload_for_rank(0)
    spec = mask_variants(WORKLOADS[WORKLOAD])[0]
    q, k, v = make_qkv(w)
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    per_step = args.reference_seconds
    for kk in range(args.warmup):
        _oracle_sample(w, spec, q, k, v, perm, per_step / 4, seed=100 + kk)
    tot_f, tot_s, tot_items = 0.0, 0.0, 0
    for kk in range(args.steps):
        f, s, n = _oracle_sample(w, spec, q, k, v, perm, per_step, seed=kk)
        tot_f, tot_s, tot_items = tot_f + f, tot_s + s, tot_items + n
    value = tot_f / tot_s / 1e12
    sample = (f"each step: random (head, query block) items of the same workload for ~{per_step:.0f} s "
              f"({tot_items} items over {args.steps} steps)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V)", "config": _config_dict(w, spec, ws),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _time_cuda(fn, reps=20, warmup=5, flush=None):
    """Median ms of `fn` over `reps` launches (CUDA events on the current stream).  With
    ``flush`` (a device buffer larger than L2), the buffer is rewritten before every timed
    launch, outside the timed interval, so each launch starts with a cold L2."""
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.add_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.median(ts))


def run_report(args):
    """One JSON line per (workload, mask): attention ms / TFLOP/s / fraction of peak, reorder
    and mask-build GB/s; then the density sweep fit time = a + b * active pairs."""
    import block_sparse_attention_lva_b200 as lva
    from synthetic import static_calibrated_mask
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    burst, sustained, hbm, peak_kind = _peaks()
    names = args.report.split(",")
    l2_flush = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MB > 126 MB L2
    gpu_ms = {}
    for name in names:
        if name in ("stress", "squad", "calib", "oracle"):
            continue
        w = WORKLOADS[name]
        q, k, v = make_qkv(w)
        qkv_dev = torch.stack([q, k, v]).to(dev)
        qkv_stacked = (qkv_dev[0], qkv_dev[1], qkv_dev[2])
        qd, kd, vd = qkv_stacked
        del q, k, v
        sweep = []
        for spec in mask_variants(w):
            static = static_calibrated_mask(w) if spec["kind"] == "static" else None
            layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                                  static_mask=static, scale=w.scale, device=dev)
            layer(qd, kd, vd, step=0)
            torch.cuda.synchronize()
            nnz = int(layer.nnz.item())
            pairs = nnz * (w.B * w.H if layer.mask_heads == 1 else w.B)
            flops = pairs * _flops_per_nnz(w)
            ms = _time_cuda(layer.attend)
            # roofline bound of this launch: tensor work at the burst peak vs algorithmic
            # bytes (Q, K, V read once, O written once, LSE) at the measured copy bandwidth
            algo_bytes = w.B * w.H * (4 * w.n_pad * w.d * 2 + 4 * w.n_pad)
            t_tensor, t_hbm = flops / (burst * 1e9), algo_bytes / (hbm * 1e6)
            bound_ms = max(t_tensor, t_hbm)
            # the whole layer path: stacked reorder + CSR + attention with the fused inverse
            ms_layer = _time_cuda(lambda: (layer.reorder_in(*qkv_stacked), setattr(layer, "_built_step", None),
                                           layer.build_mask(0), layer.attend_to_raster()))
            ms_flushed = _time_cuda(layer.attend, reps=10, flush=l2_flush) if name == "small" else None
            layer._built_step = None
            ms_mask = _time_cuda(lambda: (setattr(layer, "_built_step", None), layer.build_mask(0)))
            mask_bytes = (layer.mask_heads * w.nb * w.nb if spec["kind"] == "static" else 0) \
                + 4 * (layer.mask_heads * w.nb + 1) + 4 * nnz
            ms_reorder = _time_cuda(lambda: lva.lva_reorder_tokens(
                qd.view(w.B * w.H, w.n_valid, w.d), layer.q_t.view(w.B * w.H, w.n_pad, w.d),
                (w.T, w.Hg, w.Wg), w.tile, w.n_pad))
            reorder_bytes = w.B * w.H * (w.n_valid + w.n_pad) * w.d * 2
            status, detail = lva.lva_device_error()
            line = {"report": name, "mask": spec["label"], "active_pairs": pairs,
                    "density": nnz / (layer.mask_heads * w.nb * w.nb), "attn_ms": ms,
                    "tflops": flops / ms / 1e9, "frac_of_sustained": flops / ms / 1e9 / sustained,
                    "frac_of_burst": flops / ms / 1e9 / burst,
                    "bound": "tensor" if t_tensor >= t_hbm else "hbm", "bound_ms": bound_ms,
                    "frac_of_bound": bound_ms / ms, "algorithmic_bytes": algo_bytes,
                    "kv_l2_reread_bytes": pairs * 2 * w.block_size * w.d * 2,
                    "layer_path_ms": ms_layer, "attn_ms_l2_flushed": ms_flushed,
                    "mask_build_us": ms_mask * 1e3,
                    "mask_gbs": mask_bytes / ms_mask / 1e6, "reorder_ms": ms_reorder,
                    "reorder_gbs": reorder_bytes / ms_reorder / 1e6, "hbm_peak_gbs": hbm,
                    "peak_kind": peak_kind, "kernel_error": status}
            print(json.dumps(line), flush=True)
            gpu_ms[(name, spec["label"])] = ms
            if spec["kind"] in ("window_anchor", "all"):
                sweep.append((pairs, ms, nnz / (layer.mask_heads * w.nb * w.nb)))
            del layer
            torch.cuda.empty_cache()
        if len(sweep) >= 3:
            x = np.array([p for p, _, _ in sweep], dtype=np.float64)
            y = np.array([m for _, m, _ in sweep], dtype=np.float64)
            A = np.stack([np.ones_like(x), x], axis=1)
            (a, b), *_ = np.linalg.lstsq(A, y, rcond=None)
            r2 = 1 - np.sum((y - (a + b * x)) ** 2) / np.sum((y - y.mean()) ** 2)
            d = np.array([dd for _, _, dd in sweep])
            i10 = int(np.argmin(np.abs(d - 0.10)))
            print(json.dumps({"report": name, "density_sweep": [{"density": float(dd), "ms": float(m)} for _, m, dd in sweep],
                              "fit_ms": {"intercept": float(a), "per_pair_us": float(b * 1e3), "r2": float(r2),
                                         "intercept_share_of_10pct": float(a / y[i10])}}), flush=True)
        del qd, kd, vd, qkv_dev, qkv_stacked
        torch.cuda.empty_cache()
    # SQuad's exact two-stage operator: 12 heads, 131,072 tokens (64 frames of 32 x 64),
    # windows of 512 tokens (m = 256 windows): local pass, window transpose, global pass.
    if "squad" in names:
        H, n, d, win = 12, 131072, 128, 512
        g = torch.Generator(device=dev).manual_seed(9)
        qkv = torch.randn((3, 1, H, n, d), generator=g, device=dev).to(torch.bfloat16)
        op = lva.SquadTwoPass(1, H, n, d, win, device=dev)
        ms = _time_cuda(lambda: op(qkv[0], qkv[1], qkv[2]))
        nbk = n // 128
        pairs = H * nbk * (win // 128 + (n // win) // 128)
        flops = pairs * 4.0 * 128 * 128 * d
        print(json.dumps({"report": "squad_two_pass", "heads": H, "tokens": n, "window": win,
                          "active_pairs": pairs, "ms": ms, "tflops": flops / ms / 1e9,
                          "frac_of_burst": flops / ms / 1e9 / burst,
                          "note": "2 attention launches, no transposes: the global pass gathers the window-transposed rows through 3D tensor maps and stores O in the input order; FLOPs of both passes"}),
              flush=True)
        del qkv, op
        torch.cuda.empty_cache()
    # Static-mask calibration on the small workload (12 heads, 32,768 tokens, 256 x 256 blocks):
    # the dense pass for LSE, the block energies of all 786,432 block pairs, the selection of
    # 3,072 energy rows and the aggregation of 4 samples.
    if "calib" in names:
        from synthetic import make_qk_calibration
        w = WORKLOADS["small"]
        q, k = make_qk_calibration(w, prompt=0)
        qd, kd = q.to(dev), k.to(dev)
        cal = lva.StaticMaskCalibrator(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size,
                                       scale=w.scale, device=dev)
        cal.energies(qd, kd)
        ms_dense = _time_cuda(lambda: lva.lva_block_sparse_lse(
            cal.q_t, cal.k_t, cal.lse, w.n_valid, w.block_size, cal.row_ptr, cal.col_idx, 1, cal.scale))
        ms_energy = _time_cuda(lambda: lva.lva_block_energy(
            cal.q_t, cal.k_t, cal.lse, cal.energy, w.n_valid, w.block_size, cal.row_ptr, cal.col_idx, 1,
            cal.scale))
        mask = torch.empty(cal.energy.shape, dtype=torch.uint8, device=dev)
        ms_select = _time_cuda(lambda: lva.lva_select_blocks(cal.energy, mask, 0.8))
        samples = mask.unsqueeze(0).repeat(4, 1, 1, 1, 1).reshape(4, w.H, w.nb, w.nb).contiguous()
        out = torch.empty((w.H, w.nb, w.nb), dtype=torch.uint8, device=dev)
        ms_agg = _time_cuda(lambda: lva.lva_aggregate_masks(samples, out, 0.5))
        ms_total = _time_cuda(lambda: cal.add_prompt(qd, kd, 0.8))
        cal.samples.clear()
        status, detail = lva.lva_device_error()
        pairs = w.B * w.H * w.nb * w.nb
        qk_flops = pairs * 2.0 * w.block_size * w.block_size * w.d
        exps = pairs * float(w.block_size * w.block_size)
        print(json.dumps({"report": "calibration", "workload": "small (12 heads, 32,768 tokens)",
                          "block_pairs": pairs, "dense_lse_ms": ms_dense, "energy_ms": ms_energy,
                          "energy_qk_tflops": qk_flops / ms_energy / 1e9,
                          "energy_qk_frac_of_sustained": qk_flops / ms_energy / 1e9 / sustained,
                          "energy_exp_per_s": exps / ms_energy * 1e3,
                          "select_ms": ms_select, "select_rows": w.B * w.H * w.nb,
                          "aggregate_ms": ms_agg, "aggregate_bytes": 5 * w.H * w.nb * w.nb,
                          "add_prompt_ms": ms_total, "selected_density_eps0.8": float(mask.float().mean()),
                          "kernel_error": status}), flush=True)
        del qd, kd, cal, samples, out, mask
        torch.cuda.empty_cache()
    # mask-builder stress size: static mask, 40 heads x 4096 x 4096 blocks (671 MB read), or
    # --stress-heads heads of 4096 x 4096 blocks
    if "stress" in names or args.report_stress:
        hm, nb = args.stress_heads, 4096
        g = torch.Generator(device=dev).manual_seed(5)
        dense = (torch.rand((hm, nb, nb), generator=g, device=dev) < 0.3).to(torch.uint8)
        params = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128, 128, hm)
        row_ptr = torch.empty(hm * nb + 1, dtype=torch.int32, device=dev)
        col_idx = torch.empty(lva.lva_block_mask_max_nnz(params), dtype=torch.int32, device=dev)
        nnz = torch.empty(1, dtype=torch.int32, device=dev)
        ws = torch.empty(lva.lva_block_mask_workspace_bytes(params), dtype=torch.uint8, device=dev)
        ms_two_read = _time_cuda(lambda: lva.lva_build_block_mask(params, dense, row_ptr, col_idx, nnz))
        ms = _time_cuda(lambda: lva.lva_build_block_mask_ws(params, dense, row_ptr, col_idx, nnz, ws))
        n = int(nnz.item())
        # algorithmic bytes: the dense mask read once, row_ptr and col_idx written once
        byts = hm * nb * nb + 4 * (hm * nb + 1) + 4 * n
        print(json.dumps({"report": "mask_stress", "mask_heads": hm, "nb": nb, "nnz": n,
                          "ms_workspace_build": ms, "gbs": byts / ms / 1e6, "frac_of_hbm": byts / ms / 1e6 / hbm,
                          "ms_two_read_build": ms_two_read, "gbs_two_read": byts / ms_two_read / 1e6,
                          "algorithmic_bytes": byts, "workspace_bytes": ws.numel(), "hbm_peak_gbs": hbm}),
              flush=True)
        del dense, col_idx, ws
        torch.cuda.empty_cache()
    if "oracle" in names:
        run_oracle_report(args, gpu_ms)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lva", choices=["lva", "reference"])
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="batch: every rank its own batch element (weak scaling); heads: one layer split into "
                         "contiguous head ranges (strong scaling)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--report", default="", help="comma list of workloads (tiny,small,static,large,long,stress,squad,calib,oracle): "
                    "per-mask kernel timings and the density sweep fit instead of the bench line")
    ap.add_argument("--report-stress", action="store_true")
    ap.add_argument("--stress-heads", type=int, default=40, help="mask heads of the 4096 x 4096-block stress build")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.report:
        run_report(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_lva(args)


if __name__ == "__main__":
    main()

"""Benchmark of the score -> select -> compact path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over the resident cache: the fold of
the offset average into per-head weights, scoring of every key, top-B
selection per (layer, head, sequence) and the out-of-place compaction of K
and V (four C-ABI calls, four kernels).  Default workload: a Qwen3-8B-shaped
cache of 36 layers x 8 KV heads x 32768 keys (batch 1, contiguous), B = 2048.

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
every rank compresses its own cache (independent problems, no collective on
the data path), time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

KEY_BYTES = 256            # one bf16 key of head_dim 128, read once by the scorer
MOVE_BYTES = 4 * 256       # a kept K row and V row, each read and written by the gather
SPEC_HBM_GBS = 8000.0      # B200 HBM3e, nominal
L2_BYTES = 126 * 2 ** 20   # B200 L2
FLUSH_BYTES = 512 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Each rank compresses its own cache: a different seed per rank."""
    return seed + rank


def max_over_ranks(ms: float, world_size: int, device) -> float:
    """The job's time is the slowest rank's (device-timed) time."""
    if world_size <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# scoring kernel of each variant: (kernel name, its sources, committed traffic record)
SCORE_KERNELS = {
    "mean": ("score_kernel", ("common.cuh", "score.cuh"), "score_keys_traffic.txt"),
    "max": ("score_max_kernel", ("common.cuh", "score.cuh", "score_max.cuh"), "score_max_traffic.txt"),
    "pos": ("score_pos_tma_kernel", ("common.cuh", "score.cuh", "score_max.cuh", "score_pos.cuh",
                                     "score_pos_tma.cuh"), "score_pos_traffic.txt"),
}
POS_SPREAD = 4             # pre-RoPE variant: keys keep 1 in 4 of the original positions

METRICS = {
    "mean": "keys scored+selected/s (fold + score + top-B select + K/V compaction)",
    "max": ("keys scored (max over offsets)+selected/s (per-offset fold + tensor-core score + top-B select + "
            "K/V compaction)"),
    "pos": ("keys scored (per-key distance, pre-RoPE)+selected/s (fold + score at positions + top-B select + "
            "K/V compaction)"),
}


def score_kernel_fingerprint(variant="mean"):
    """Hash of the scoring kernel's sources: ncu traffic is only reported while it matches."""
    h = hashlib.sha256()
    for name in SCORE_KERNELS[variant][1]:
        with open(os.path.join(ROOT, "rope_aware_key_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, variant="mean"):
    """Per-launch DRAM bytes of the scoring kernel from the committed ncu summary, if current."""
    p = os.path.join(ROOT, "profiles", SCORE_KERNELS[variant][2])
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_sources") != score_kernel_fingerprint(variant) or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def wait_first(self, limit_s=5.0):
        """Wait (bounded) for the first sample: nvidia-smi's start-up then lies
        outside the timed region."""
        t = time.time()
        while self.proc is not None and not self.samples and time.time() - t < limit_s:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not rows:
            rows = [p for (_, p) in self.samples[-5:]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        smax = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.strip().lower() == "active"})
        pw = [num(r[4]) for r in rows if num(r[4]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200 import build as tri_build
    if tri_build.needs_build():
        log("building libtri_evict.so (missing or older than its sources)")
        tri_build.build()
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = gen.WORKLOADS[args.workload]
    assert wl.layout in ("contig", "ragged"), "the bench compresses contiguous or ragged caches out of place"
    B = wl.budget

    t = time.time()
    cache = gen.make_cache(wl, seed=rank_seed(args.seed, rank), device=dev)
    torch.cuda.synchronize()
    log(f"[rank {rank}] generated {args.workload} in {time.time() - t:.1f}s")
    d = (tri.desc_contig(cache.k, cache.v) if wl.layout == "contig"
         else tri.desc_ragged(cache.k, cache.v, cache.cu_seqlens.cpu().tolist()))
    keys = sum(cache.lens) * wl.num_layers * wl.num_kv_heads
    moved = sum(min(B, n) for n in cache.lens) * wl.num_layers * wl.num_kv_heads
    qc = cache.query_center.reshape(-1, wl.head_dim).to(dev).contiguous()
    if args.variant == "max":
        w = torch.empty((qc.shape[0], len(wl.offsets), wl.head_dim), dtype=torch.float32, device=dev)
    else:
        w = torch.empty_like(qc)
    stride = tri.score_row_stride(d)
    scores = torch.empty((d.units, stride), dtype=torch.float32, device=dev)
    kept = torch.empty((d.units, B), dtype=torch.int32, device=dev)
    cnt = torch.empty((d.units,), dtype=torch.int32, device=dev)
    k_out = torch.empty((d.units, B, wl.head_dim), dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    stream = torch.cuda.current_stream(dev)
    ws_buf = None
    if args.path == "compress":
        assert args.variant == "mean", "--path compress runs the folded score"
        ws_buf = torch.empty(tri.workspace_size(d, B), dtype=torch.uint8, device=dev)
    positions = qpos = None
    if args.variant == "pos":
        positions, qpos = gen.key_positions(cache, seed=rank_seed(args.seed, rank), stride=stride,
                                            spread=POS_SPREAD)

    def step(ev=None, st=None):
        st = st or stream
        if ev is not None:
            ev[0].record(st)
        if args.variant == "max":
            tri.fold_offset_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=st)
        else:
            tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=st)
        if ev is not None:
            ev[1].record(st)
        if args.path == "compress":
            # one call: the single-kernel step when the units fit one wave of clusters, else three kernels
            tri.compress(d, w, B, tri.COMPACT_OUT_OF_PLACE, kept, cnt, k_out, v_out, ws_buf, stream=st)
            if ev is not None:
                for e in ev[2:]:
                    e.record(st)
            return
        if args.variant == "max":
            tri.score_keys_max(d, w, scores, stream=st)
        elif args.variant == "pos":
            tri.score_keys_at_positions(d, w, wl.theta, qpos, positions, tri.PAIRING_HALF, scores, stream=st)
        else:
            tri.score_keys(d, w, scores, stream=st)
        if ev is not None:
            ev[2].record(st)
        tri.select_topk(d, scores, B, kept, cnt, stream=st)
        if ev is not None:
            ev[3].record(st)
        tri.compact_kv(d, kept, cnt, B, tri.COMPACT_OUT_OF_PLACE, k_out, v_out, stream=st)
        if ev is not None:
            ev[4].record(st)

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    sampler = ClockSampler(gpu_index)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = tri.read_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    # The timed steps replay the step as one CUDA graph (its launches issued
    # with no host work in between); --eager times plain launches instead.
    graph = None
    launches_per_step = 4
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        before = tri.kernel_launches()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            step(st=torch.cuda.current_stream(dev))
        launches_per_step = tri.kernel_launches() - before
        graph.replay()
        torch.cuda.synchronize()

    # Caches that L2 could hold a good part of are timed step by step with L2
    # flushed in between (a 512 MB fill, outside the events); larger ones back to back.
    kv_bytes = cache.k.numel() * 2 + cache.v.numel() * 2
    flush = kv_bytes < 4 * L2_BYTES
    flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if flush else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)] if flush else None
    sampler.wait_first()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = tri.kernel_launches()
    t0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        if flush:
            flush_buf.fill_(i)
            step_evs[i][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        if flush:
            step_evs[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if ws > 1:
        torch.distributed.barrier()
    launches = launches_per_step * args.steps if graph is not None else tri.kernel_launches() - launches0
    ms = start.elapsed_time(end) if not flush else sum(a.elapsed_time(b) for a, b in step_evs)
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    # Per-kernel times: plain launches with events between the kernels, queued
    # behind a GPU sleep so that the host is far ahead when they run.
    nb = min(args.steps, 100)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nb)]
    torch.cuda._sleep(int(4e7 + nb * 4e5))
    for i in range(nb):
        if flush:
            flush_buf.fill_(i)
        step(evs[i])
    torch.cuda.synchronize()
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])   # ms: fold, score, select, compact
    st = tri.read_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the timed steps")

    ms_max = max_over_ranks(ms, ws, dev)
    ms_step = ms_max / args.steps
    value = keys * ws * args.steps / (ms_max / 1e3)

    # roofline of the dominant kernel (scoring; or the one-call step) and of the whole step
    peak, peak_kind = measured_hbm_peak()
    score_ms = float(per[:, 1].mean())
    score_bytes = keys * (KEY_BYTES + (4 if args.variant == "pos" else 0))   # + the positions read
    if args.path == "compress":
        score_bytes = keys * KEY_BYTES + moved * MOVE_BYTES
    achieved = score_bytes / (score_ms / 1e3) / 1e9
    step_bytes = keys * KEY_BYTES + moved * MOVE_BYTES
    step_gbs = step_bytes / (ms_step / 1e3) / 1e9
    traffic = ncu_traffic(args.workload, args.variant)

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    e2e = run_e2e(args, tri, cache, d, wl, qc, w, kept, cnt, k_out, v_out, stream, keys, ws, positions, qpos)

    result = None
    if rank == 0:
        cpu = cpu_baseline(wl, args) if ws == 1 and not args.no_cpu_baseline else None
        result = {
            "metric": METRICS[args.variant],
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 keys/values, fp32 scores (fp64 fold)", "data": "synthetic (seeded generator)",
            "config": {"workload": f"{args.workload}: {wl.num_layers} layers x {wl.num_kv_heads} KV heads x "
                                   f"{max(cache.lens)} keys, batch {wl.batch}, {wl.layout}, B={B}, "
                                   f"theta={wl.theta:g}, |D|={len(wl.offsets)}",
                       "keys_per_gpu": keys, "budget": B, "parallelism": f"independent caches x{ws}",
                       "l2": ("K and V of %.3f GB each vs a 126 MB L2: L2 flushed (512 MB fill) before every "
                              "timed step, each step timed alone" if flush else
                              "inputs larger than L2 (K and V of %.2f GB each vs 126 MB); no flush")
                             % (keys * KEY_BYTES / 1e9)},
            "step_breakdown_ms": ({"fold": float(per[:, 0].mean()), "score": score_ms,
                                   "select": float(per[:, 2].mean()), "compact": float(per[:, 3].mean())}
                                  if args.path == "calls" else
                                  {"fold": float(per[:, 0].mean()), "compress": score_ms}),
            "hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_gbs,
                    "frac_of_measured": step_gbs / peak, "frac_of_8tbps_spec": step_gbs / SPEC_HBM_GBS},
            "roofline": {"kernel": (SCORE_KERNELS[args.variant][0] if args.path == "calls" else
                                    f"tri_compress ({launches_per_step - 1} kernel(s))"), "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic if args.path == "calls" else None,
                         "algorithmic_bytes_per_launch": score_bytes},
            "clocks": clocks,
            "gpu_launches": int(launches),
            "timing": ("CUDA graph of the step, replayed" if graph is not None else "plain launches") +
                      "; step_breakdown_ms from plain launches queued ahead of the GPU",
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
    if ws > 1:
        torch.distributed.destroy_process_group()
    return result


def run_e2e(args, tri, cache, d, wl, qc, w, kept, cnt, k_out, v_out, stream, keys, ws, positions=None, qpos=None):
    """Same step with the cache in pinned host memory: H2D of K and V, the four
    calls, D2H of the kept indices, counts and compacted K/V, every step.

    The results of step i go back on a second stream while step i+1's inputs
    come in (PCIe moves both directions at once): the outputs are double
    buffered, step i+1 overwrites K and V only after step i's compaction has
    read them (stream order), and a buffer is reused only after its copy-out
    has finished.  The timed region ends after the last copy-out."""
    steps = max(1, min(args.steps, args.e2e_steps))
    hk = torch.empty(cache.k.shape, dtype=cache.k.dtype, pin_memory=True)
    hv = torch.empty(cache.v.shape, dtype=cache.v.dtype, pin_memory=True)
    hk.copy_(cache.k)
    hv.copy_(cache.v)
    hkept = torch.empty(kept.shape, dtype=kept.dtype, pin_memory=True)
    hcnt = torch.empty(cnt.shape, dtype=cnt.dtype, pin_memory=True)
    hko = torch.empty(k_out.shape, dtype=k_out.dtype, pin_memory=True)
    hvo = torch.empty(v_out.shape, dtype=v_out.dtype, pin_memory=True)
    hq = qc.cpu().pin_memory()
    hpos = positions.cpu().pin_memory() if positions is not None else None
    B = kept.shape[1]
    scores = torch.empty((d.units, tri.score_row_stride(d)), dtype=torch.float32, device=qc.device)
    ws_e2e = torch.empty(tri.workspace_size(d, B), dtype=torch.uint8, device=qc.device) \
        if args.path == "compress" else None
    outs = [(kept, cnt, k_out, v_out),
            (torch.empty_like(kept), torch.empty_like(cnt), torch.empty_like(k_out), torch.empty_like(v_out))]
    out_stream = torch.cuda.Stream(device=qc.device)
    computed = [torch.cuda.Event(), torch.cuda.Event()]
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    state = {"i": 0}

    def one():
        j = state["i"] % 2
        state["i"] += 1
        kp, cn, ko, vo = outs[j]
        cache.k.copy_(hk, non_blocking=True)
        cache.v.copy_(hv, non_blocking=True)
        qc.copy_(hq, non_blocking=True)
        if hpos is not None:
            positions.copy_(hpos, non_blocking=True)
        stream.wait_event(copied[j])            # buffer j's previous copy-out is done
        if args.path == "compress":
            tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
            tri.compress(d, w, B, tri.COMPACT_OUT_OF_PLACE, kp, cn, ko, vo, ws_e2e, stream=stream)
        else:
            if args.variant == "max":
                tri.fold_offset_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
                tri.score_keys_max(d, w, scores, stream=stream)
            elif args.variant == "pos":
                tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
                tri.score_keys_at_positions(d, w, wl.theta, qpos, positions, tri.PAIRING_HALF, scores,
                                            stream=stream)
            else:
                tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
                tri.score_keys(d, w, scores, stream=stream)
            tri.select_topk(d, scores, B, kp, cn, stream=stream)
            tri.compact_kv(d, kp, cn, B, tri.COMPACT_OUT_OF_PLACE, ko, vo, stream=stream)
        computed[j].record(stream)
        out_stream.wait_event(computed[j])
        with torch.cuda.stream(out_stream):
            hkept.copy_(kp, non_blocking=True)
            hcnt.copy_(cn, non_blocking=True)
            hko.copy_(ko, non_blocking=True)
            hvo.copy_(vo, non_blocking=True)
        copied[j].record(out_stream)

    one()
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        one()
    stream.wait_stream(out_stream)              # the last copy-out is inside the timed region
    end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), ws, qc.device)
    h2d = hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 4 + (hpos.numel() * 4 if hpos is not None else 0)
    d2h = hkept.numel() * 4 + hcnt.numel() * 4 + hko.numel() * 2 + hvo.numel() * 2
    return {"value": keys * ws * steps / (ms / 1e3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "host_memory": "pinned",
            "overlap": "results of step i copied back on a second stream while step i+1's inputs are copied in"}


# ---------------------------------------------------------------- the oracle as a CPU baseline

def oracle_unit_pipeline(orc, keys_bits, vals_bits, qc, wl, B, threads, variant="mean"):
    """The oracle's own path for one unit: literal per-offset average (or
    maximum), keep-highest, gather."""
    if variant == "pos":
        # a compacted pre-RoPE unit: sorted distinct positions in [0, POS_SPREAD * n), query at POS_SPREAD * n
        n = keys_bits.shape[0]
        rng = np.random.default_rng(n)
        p = np.sort(rng.choice(POS_SPREAD * n, size=n, replace=False))
        s = orc.score_at_positions(keys_bits, qc, wl.theta, wl.offsets, p, POS_SPREAD * n, 0, threads)
    else:
        score = orc.score_max_literal if variant == "max" else orc.score_literal
        s = score(keys_bits, qc, wl.theta, wl.offsets, wl.delta0, 0, threads)
    kept = orc.select(s, B)
    orc.gather_rows(keys_bits, kept)
    orc.gather_rows(vals_bits, kept)
    return len(s)


def cpu_sample(wl, n_keys, seed):
    """A bounded sample of the workload drawn on the CPU: one unit's first n_keys keys."""
    sw = gen.scaled(wl, num_layers=1, num_kv_heads=1, batch=1, layout="contig", seq_len=n_keys)
    c = gen.make_cache(sw, seed=seed, device="cpu")
    kb = c.k[0, 0, 0].contiguous().view(torch.int16).numpy().view(np.uint16)
    vb = c.v[0, 0, 0].contiguous().view(torch.int16).numpy().view(np.uint16)
    return kb, vb, c.query_center[0, 0].numpy()


def cpu_baseline(wl, args, budget_s=None):
    import oracle as orc
    orc.build()
    threads = orc.default_threads()
    budget_s = args.cpu_seconds if budget_s is None else budget_s
    n = min(max(wl.seq_len, wl.len_hi, 4096), 32768)
    kb, vb, qc = cpu_sample(wl, n, args.seed)
    B = min(wl.budget, n)
    done = 0
    t0 = time.time()
    reps = 0
    while True:
        done += oracle_unit_pipeline(orc, kb, vb, qc, wl, B, threads, args.variant)
        reps += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": done / dt, "unit": "keys/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} x one unit of {n} keys (literal {'max' if args.variant == 'max' else 'average'} "
                      f"{'at per-key distances ' if args.variant == 'pos' else ''}over "
                      f"|D|={len(wl.offsets)} offsets, "
                      f"select B={B}, gather K and V), fp64, {dt:.1f}s"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle as orc
    orc.build()
    wl = gen.WORKLOADS[args.workload]
    threads = orc.default_threads()
    # size each step so that the whole run stays within about two minutes
    probe_n = 1024
    kb, vb, qc = cpu_sample(wl, probe_n, args.seed)
    t = time.time()
    oracle_unit_pipeline(orc, kb, vb, qc, wl, min(wl.budget, probe_n), threads, args.variant)
    rate = probe_n / max(time.time() - t, 1e-6)
    per_step_s = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    n = int(min(32768, max(256, rate * per_step_s)))
    kb, vb, qc = cpu_sample(wl, n, args.seed)
    B = min(wl.budget, n)
    for _ in range(args.warmup):
        oracle_unit_pipeline(orc, kb, vb, qc, wl, B, threads, args.variant)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_unit_pipeline(orc, kb, vb, qc, wl, B, threads, args.variant)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    kind = {"mean": "literal average", "max": "literal max", "pos": "literal average at per-key distances"}
    sample = (f"each step: one unit of {n} keys of the {args.workload} workload ({kind[args.variant]} over "
              f"|D|={len(wl.offsets)} offsets, select B={B}, gather K and V), fp64")
    return {"impl": "reference", "metric": METRICS[args.variant],
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
            "config": {"workload": args.workload, "keys_per_step": n, "budget": B},
            "cpu_baseline": {"value": value, "unit": "keys/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def relaunch_per_gpu(n: int) -> int:
    """Run this same command under torch.distributed.run with n processes on
    this node (rendezvous on 127.0.0.1, a free port); returns its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    log("launching " + " ".join(cmd[2:]))
    try:
        return subprocess.call(cmd, timeout=3600)      # last bound; the process group times out first
    except subprocess.TimeoutExpired:
        return 124


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3_full", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time plain launches instead of a CUDA graph of the step")
    ap.add_argument("--path", default="calls", choices=["calls", "compress"],
                    help="calls: fold, score, select, compact as four calls (default); compress: fold + tri_compress")
    ap.add_argument("--variant", default="mean", choices=["mean", "max", "pos"],
                    help="mean: the folded offset average (default); max: the max over the offsets; "
                         "pos: the offset average at per-key distances (pre-RoPE cache with positions)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    ws = dist_env()[0]
    if args.impl == "ours" and args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started by hand with --gpus N: one process per GPU, the launch torchrun gives
        raise SystemExit(relaunch_per_gpu(args.gpus))
    if args.impl == "ours" and ws != args.gpus:
        log(f"--gpus {args.gpus} but {ws} rank(s) were launched: reporting {ws}")
    res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

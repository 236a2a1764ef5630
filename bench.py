"""Benchmark of the score -> select -> compact path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over the resident cache: the fold of
the offset average into per-head weights, scoring of every key, top-B
selection per (layer, head, sequence) and the out-of-place compaction of K
and V (four C-ABI calls, four kernels).  Default workload: a Qwen3-8B-shaped
cache of 36 layers x 8 KV heads x 32768 keys (batch 1, contiguous), B = 2048.

The paged workload (--workload qwen25_paged: 28 layers x 4 KV heads, 64
sequences of 8192..32768 tokens in 16-token pages) is a serving cache that is
pruned once per window of generated tokens: one initial event (every
sequence down to B in place), then steady rounds, each appending 128 tokens
per sequence (untimed, as a decoder would) and re-compressing every
2176-key row down to B in place (the fold and one tri_compress call, whose
selection kernel also fills each row's holes).  A step there is one steady
round (default 8 timed rounds); the initial event is reported beside it.

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
every rank compresses its own cache (--shard replicas, the default), or the
ranks split one cache by whole layers (--shard layers); either way there is
no collective on the data path, and time = max over ranks.
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
PAGED_ROUNDS = 8           # timed steady rounds of the paged workload
PAGED_APPEND = 128         # tokens a sequence generates between two pruning events
PAGED_BREAKDOWN_ROUNDS = 3  # extra rounds that also time the scorer on its own

METRICS = {
    "mean": "keys scored+selected/s (fold + score + top-B select + K/V compaction)",
    "max": ("keys scored (max over offsets)+selected/s (per-offset fold + tensor-core score + top-B select + "
            "K/V compaction)"),
    "pos": ("keys scored (per-key distance, pre-RoPE)+selected/s (fold + score at positions + top-B select + "
            "K/V compaction)"),
}


def flush_l2(buf, sink):
    """Evict L2 between timed events: write a buffer larger than L2, then read
    it back (into `sink`, a 0-dim int64 tensor), so that the lines the write
    left dirty are written back here rather than inside the next event."""
    buf.fill_(1)
    torch.sum(buf, dim=0, dtype=torch.int64, out=sink)


def score_kernel_fingerprint(variant="mean"):
    """Hash of the scoring kernel's sources: ncu traffic is only reported while it matches."""
    h = hashlib.sha256()
    for name in SCORE_KERNELS[variant][1]:
        with open(os.path.join(ROOT, "rope_aware_key_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(workload, variant="mean"):
    """The committed ncu traffic record of a variant's scorer on a workload."""
    if gen.WORKLOADS[workload].layout == "paged":
        return f"{'score_max' if variant == 'max' else 'score_keys'}_paged_{workload}_traffic.txt"
    return SCORE_KERNELS[variant][2]


def ncu_traffic(workload, variant="mean"):
    """Per-launch DRAM bytes of the scoring kernel from the committed ncu summary, if current."""
    p = os.path.join(ROOT, "profiles", traffic_record(workload, variant))
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_sources") != score_kernel_fingerprint(variant) or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and throttle reasons sampled in the background while
    the timed region runs: through NVML every 0.5 ms (so that a timed region
    of 10 ms, 20 steps of the headline, gets about 20 samples), or, without
    NVML, nvidia-smi every 100 ms.  Each sample is a row
    [time, index, sm MHz, max sm MHz, power W, reasons, hw_slowdown,
     hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap]."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, uuid: str = None, period_s: float = 0.0005):
        self.samples = []
        self.proc = None
        self.source = None
        self.period_s = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self._nvml, self._h, self._index = pynvml, h, gpu_index
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.period_s = 0.1
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _poll(self):
        nv, h = self._nvml, self._h
        try:
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            smax = "[N/A]"
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                row = ["", str(self._index), str(sm), str(smax), f"{pw:.1f}", hex(r)] + \
                      ["Active" if r & b else "Not Active" for b in bits]
                self.samples.append((time.time(), row))
            except Exception:
                pass
            self._stop.wait(self.period_s)

    def wait_first(self, limit_s=5.0):
        """Wait (bounded) for the first sample: the sampler's start-up then lies
        outside the timed region."""
        t = time.time()
        while self.source is not None and not self.samples and time.time() - t < limit_s:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                self.samples.append((time.time(), parts))

    def stop(self):
        ev = getattr(self, "_stop", None)
        if ev is not None:
            ev.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [p for (t, p) in self.samples if t0 <= t <= t1]
        inside = len(rows)
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
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
               "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}
        if getattr(self, "source", None):
            out["source"] = f"{self.source}, every {self.period_s * 1e3:g} ms"
        if inside == 0:
            out["note"] = "no sample inside the timed region: the last samples before it"
        return out


def gpu_identity(dev, local):
    """(NVML index guess, NVML uuid) of the torch device `dev`."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    try:
        index = int(vis.split(",")[local]) if vis else local
    except ValueError:
        index = local
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    return index, uuid


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import rope_aware_key_b200 as tri
    from rope_aware_key_b200 import build as tri_build
    if tri_build.needs_build():
        # one process builds (the ranks of a torchrun launch take turns on a
        # lock; the later ones find the library current)
        import fcntl
        os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
        with open(os.path.join(ROOT, "_build", ".build.lock"), "w") as lock:
            fcntl.flock(lock, fcntl.LOCK_EX)
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
    if wl.layout == "paged":
        return run_paged(args, tri, dev, rank, ws)
    B = wl.budget

    t = time.time()
    if args.shard == "layers":
        # one cache split by whole layers (every KV head and sequence of a
        # layer on one rank): each rank draws only its own layers
        from rope_aware_key_b200.shard import layer_ranges
        whole = wl
        l0, l1 = layer_ranges(whole.num_layers, ws)[rank]
        if l1 == l0:
            raise SystemExit(f"--shard layers: {ws} ranks for {whole.num_layers} layers leaves rank {rank} empty")
        cache = gen.make_cache(whole, seed=args.seed, device=dev, layer_range=(l0, l1))
        wl = cache.wl
        job_keys = sum(cache.lens) * whole.num_layers * whole.num_kv_heads
        parallelism = f"one cache split by layers over {ws} ranks (layers {l0}..{l1 - 1} on rank {rank})"
    else:
        cache = gen.make_cache(wl, seed=rank_seed(args.seed, rank), device=dev)
        job_keys = None
        parallelism = f"independent caches x{ws}"
    torch.cuda.synchronize()
    log(f"[rank {rank}] generated {args.workload} in {time.time() - t:.1f}s")
    d = (tri.desc_contig(cache.k, cache.v) if wl.layout == "contig"
         else tri.desc_ragged(cache.k, cache.v, cache.cu_seqlens.cpu().tolist()))
    keys = sum(cache.lens) * wl.num_layers * wl.num_kv_heads
    if job_keys is None:
        job_keys = keys * ws                       # every rank its own cache of the same shape
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
        assert args.variant != "pos", "--path compress runs the folded score or the max over the offsets"
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
            # (the max over the offsets: its scorer, then the selection and the gather)
            if args.variant == "max":
                tri.compress_max(d, w, B, tri.COMPACT_OUT_OF_PLACE, kept, cnt, k_out, v_out, ws_buf, stream=st)
            else:
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

    sampler = ClockSampler(*gpu_identity(dev, local))
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
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
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
            flush_l2(flush_buf, flush_sink)
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
            flush_l2(flush_buf, flush_sink)
        step(evs[i])
    torch.cuda.synchronize()
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])   # ms: fold, score, select, compact
    st = tri.read_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the timed steps")

    ms_max = max_over_ranks(ms, ws, dev)
    ms_step = ms_max / args.steps
    value = job_keys * args.steps / (ms_max / 1e3)

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
    e2e = run_e2e(args, tri, cache, d, wl, qc, w, kept, cnt, k_out, v_out, stream, job_keys, ws, positions, qpos)

    result = None
    if rank == 0:
        cpu = cpu_baseline(wl, args) if ws == 1 and not args.no_cpu_baseline else None
        result = {
            "metric": METRICS[args.variant],
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if args.shard == "layers" else "weak", "vs_baseline": None,
            "dtype": "bf16 keys/values, fp32 scores (fp64 fold)", "data": "synthetic (seeded generator)",
            "config": {"workload": f"{args.workload}: {gen.WORKLOADS[args.workload].num_layers} layers x "
                                   f"{wl.num_kv_heads} KV heads x "
                                   f"{max(cache.lens)} keys, batch {wl.batch}, {wl.layout}, B={B}, "
                                   f"theta={wl.theta:g}, |D|={len(wl.offsets)}",
                       "keys_per_gpu": keys, "budget": B, "parallelism": parallelism,
                       "l2": ("K and V of %.3f GB each vs a 126 MB L2: L2 flushed before every timed step (a "
                              "512 MB buffer written then read back), each step timed alone" if flush else
                              "inputs larger than L2 (K and V of %.2f GB each vs 126 MB); no flush")
                             % (keys * KEY_BYTES / 1e9)},
            "step_breakdown_ms": ({"fold": float(per[:, 0].mean()), "score": score_ms,
                                   "select": float(per[:, 2].mean()), "compact": float(per[:, 3].mean())}
                                  if args.path == "calls" else
                                  {"fold": float(per[:, 0].mean()), "compress": score_ms}),
            "hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_gbs,
                    "frac_of_measured": step_gbs / peak, "frac_of_8tbps_spec": step_gbs / SPEC_HBM_GBS},
            "roofline": {"kernel": (SCORE_KERNELS[args.variant][0] if args.path == "calls" else
                                    f"{'tri_compress_max' if args.variant == 'max' else 'tri_compress'} "
                                    f"({launches_per_step - 1} kernel(s))"), "bound": "hbm", "achieved": achieved,
                         "peak": peak,
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


def run_paged(args, tri, dev, rank, ws):
    """The paged serving cache: an initial pruning event, then steady rounds
    (append PAGED_APPEND tokens per sequence, untimed; re-compress in place).
    The initial event is four calls (fold, score, select, in-place hole fill),
    a steady round two: the fold and tri_compress in place for the folded
    score, the per-offset fold and tri_compress_max for the max over the
    offsets.
    Every event is queued behind a GPU sleep so that the launches are all
    waiting when the first one runs, and timed with CUDA events on the
    launching stream; L2 is flushed (a 512 MB fill) before every event."""
    _, _, local = dist_env()
    if args.shard != "replicas":
        raise SystemExit("the paged workload runs as replicas (one cache per rank)")
    if args.variant == "pos":
        raise SystemExit("the paged workload runs the folded score (mean) or the max over the offsets (max)")
    use_max = args.variant == "max"
    wl = gen.WORKLOADS[args.workload]
    B = wl.budget
    L, H = wl.num_layers, wl.num_kv_heads
    seed = rank_seed(args.seed, rank)
    t = time.time()
    cache = gen.make_cache(wl, seed=seed, device=dev)
    torch.cuda.synchronize()
    log(f"[rank {rank}] generated {args.workload} in {time.time() - t:.1f}s "
        f"({sum(cache.lens) * L * H / 1e6:.1f} M keys)")
    units = wl.units
    qc = cache.query_center.reshape(-1, wl.head_dim).to(dev).contiguous()
    w = (torch.empty((qc.shape[0], len(wl.offsets), wl.head_dim), dtype=torch.float32, device=dev) if use_max
         else torch.empty_like(qc))
    kept = torch.empty((units, B), dtype=torch.int32, device=dev)
    cnt = torch.empty((units,), dtype=torch.int32, device=dev)
    flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)
    col = torch.arange(B, device=dev)[None, :]

    ws_buf = None                                  # tri_compress's workspace (the score matrix)

    def fold():
        if use_max:
            tri.fold_offset_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
        else:
            tri.fold_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)

    def score(d, scores):
        if use_max:
            tri.score_keys_max(d, w, scores, stream=stream)
        else:
            tri.score_keys(d, w, scores, stream=stream)

    def event(d, scores, evs=None):
        """The initial pruning event, one call per stage: fold, score, select,
        in-place hole fill.  evs: five events around the four calls."""
        def rec(i):
            if evs is not None:
                evs[i].record(stream)
        rec(0)
        fold()
        rec(1)
        score(d, scores)
        rec(2)
        tri.select_topk(d, scores, B, kept, cnt, stream=stream)
        rec(3)
        tri.compact_kv(d, kept, cnt, B, tri.COMPACT_IN_PLACE_HOLEFILL, None, None, stream=stream)
        rec(4)

    def steady(d, evs=None, score_alone=None):
        """A steady round: the fold, then tri_compress (tri_compress_max for
        the max over the offsets) in place: score, then a warp per row that
        selects and fills the row's holes.  score_alone: a score matrix; the
        scorer and then the selection (without the fill) run on their own
        first, each timed (the breakdown round; the compress call then redoes
        both).  evs: events around each call."""
        nonlocal ws_buf
        marks = iter(evs or [])

        def rec():
            if evs is not None:
                next(marks).record(stream)
        need = tri.workspace_size(d, B)
        if ws_buf is None or ws_buf.numel() < need:
            ws_buf = torch.empty(need, dtype=torch.uint8, device=dev)
        rec()
        fold()
        rec()
        if score_alone is not None:
            score(d, score_alone)
            rec()
            tri.select_topk(d, score_alone, B, kept, cnt, stream=stream)
            rec()
        if use_max:
            tri.compress_max(d, w, B, tri.COMPACT_IN_PLACE_HOLEFILL, kept, cnt, None, None, ws_buf, stream=stream)
        else:
            tri.compress(d, w, B, tri.COMPACT_IN_PLACE_HOLEFILL, kept, cnt, None, None, ws_buf, stream=stream)
        rec()

    def timed(fn, n_events):
        flush_l2(flush_buf, flush_sink)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
        torch.cuda.synchronize()
        torch.cuda._sleep(int(2e6))
        fn(evs)
        torch.cuda.synchronize()
        per = [evs[i].elapsed_time(evs[i + 1]) for i in range(n_events - 1)]
        moved = int(((kept >= B) & (col < cnt[:, None])).sum())     # rows the hole fill moved
        return per, moved

    # initial event: warm-up with the non-destructive stages, then the event once
    d0 = tri.desc_paged(cache.k, cache.v, cache.block_table, cache.lens)
    scores0 = torch.empty((units, tri.score_row_stride(d0)), dtype=torch.float32, device=dev)
    keys0 = sum(cache.lens) * L * H
    for _ in range(args.warmup):
        fold()
        score(d0, scores0)
        tri.select_topk(d0, scores0, B, kept, cnt, stream=stream)
    per0, moved0 = timed(lambda evs: event(d0, scores0, evs), 5)
    gen.release_tail_blocks(cache, [min(B, n) for n in cache.lens])
    del scores0
    torch.cuda.empty_cache()
    st = tri.read_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the initial event")

    # steady rounds
    sampler = ClockSampler(*gpu_identity(dev, local))
    sampler.wait_first()
    scores = None
    rounds = []
    launches0 = tri.kernel_launches()
    t0 = None
    for i in range(args.warmup + args.steps):
        gen.append_tokens(cache, PAGED_APPEND, step=1 + i)
        d = tri.desc_paged(cache.k, cache.v, cache.block_table, cache.lens)
        if scores is None:
            scores = torch.empty((units, tri.score_row_stride(d)), dtype=torch.float32, device=dev)
        if i == args.warmup:
            if ws > 1:
                torch.distributed.barrier()
            t0 = time.time()
            launches0 = tri.kernel_launches()
        per, moved = timed(lambda evs: steady(d, evs), 3)
        if i >= args.warmup:
            rounds.append((per, moved, sum(cache.lens) * L * H))
        gen.release_tail_blocks(cache, [min(B, n) for n in cache.lens])
    t1 = time.time()
    launches = tri.kernel_launches() - launches0
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    clocks["window"] = "the steady rounds, appends between them included"
    # breakdown rounds: the scorer alone, then the same round
    per1 = []
    for j in range(PAGED_BREAKDOWN_ROUNDS):
        gen.append_tokens(cache, PAGED_APPEND, step=1 + args.warmup + args.steps + j)
        d = tri.desc_paged(cache.k, cache.v, cache.block_table, cache.lens)
        per1.append(timed(lambda evs: steady(d, evs, score_alone=scores), 5)[0])
        gen.release_tail_blocks(cache, [min(B, n) for n in cache.lens])
    per1 = np.array(per1)                          # ms: fold, score alone, select alone, compress
    st = tri.read_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the steady rounds")

    per = np.array([r[0] for r in rounds])       # ms: fold, compress
    ms_rounds = float(per.sum())
    ms_max = max_over_ranks(ms_rounds, ws, dev)
    keys_round = rounds[0][2]
    moved = float(np.mean([r[1] for r in rounds]))
    value = keys_round * len(rounds) * ws / (ms_max / 1e3)
    ms_step = ms_max / len(rounds)
    peak, peak_kind = measured_hbm_peak()
    score_ms = float(per1[:, 1].mean())
    score_bytes = keys_round * KEY_BYTES
    achieved = score_bytes / (score_ms / 1e3) / 1e9
    step_bytes = keys_round * KEY_BYTES + moved * MOVE_BYTES
    step_gbs = step_bytes / (ms_step / 1e3) / 1e9
    init_ms = float(sum(per0))
    init_bytes = keys0 * KEY_BYTES + moved0 * MOVE_BYTES

    e2e = run_paged_e2e(args, tri, cache, wl, qc, kept, cnt, stream, ws, lambda dd: steady(dd))

    result = None
    if rank == 0:
        cpu = cpu_baseline(wl, args) if ws == 1 and not args.no_cpu_baseline else None
        result = {
            "metric": METRICS[args.variant] + ", paged cache, in place",
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": len(rounds), "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 keys/values, fp32 scores (fp64 fold)", "data": "synthetic (seeded generator)",
            "config": {"workload": f"{args.workload}: {L} layers x {H} KV heads, {wl.batch} sequences of "
                                   f"{wl.len_lo}..{wl.len_hi} tokens in {wl.block_size}-token pages, B={B}, "
                                   f"theta={wl.theta:g}, |D|={len(wl.offsets)}; a step is one steady round: "
                                   f"{PAGED_APPEND} tokens appended per sequence (untimed), every row of "
                                   f"{B + PAGED_APPEND} keys re-compressed to {B} in place",
                       "keys_per_gpu": keys_round, "budget": B, "parallelism": f"independent caches x{ws}",
                       "l2": "L2 flushed before every pruning event, outside the events: a 512 MB buffer "
                             "written then read back (the write's dirty lines drain before the event)"},
            "step_breakdown_ms": {("fold (per offset)" if use_max else "fold"): float(per[:, 0].mean()),
                                  ("compress_max" if use_max else "compress"): float(per[:, 1].mean()),
                                  "score (alone)": score_ms,
                                  "select alone (no fill, scores fresh in L2)": float(per1[:, 2].mean()),
                                  "select + hole fill (compress minus score alone)":
                                      float(per[:, 1].mean()) - score_ms,
                                  "breakdown": f"score alone, select alone: {PAGED_BREAKDOWN_ROUNDS} more "
                                               "rounds, each with the scorer and then the selection run on "
                                               "their own (after the flush) before the compress call; select + "
                                               "hole fill: the timed rounds' compress minus the scorer alone"},
            "rows_moved_per_step": moved,
            "hbm": {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_gbs,
                    "frac_of_measured": step_gbs / peak, "frac_of_8tbps_spec": step_gbs / SPEC_HBM_GBS},
            "initial_event": {"ms": init_ms, "keys": keys0, "rows_moved": moved0,
                              "breakdown_ms": dict(zip(("fold", "score", "select", "holefill"), per0)),
                              "keys_per_s": keys0 / (init_ms / 1e3),
                              "achieved_gbs": init_bytes / (init_ms / 1e3) / 1e9,
                              "frac_of_8tbps_spec": init_bytes / (init_ms / 1e3) / 1e9 / SPEC_HBM_GBS,
                              "timing": "one event (it compacts the cache in place), after warm-up passes of "
                                        "the fold, score and select"},
            "roofline": {"kernel": f"{SCORE_KERNELS[args.variant][0]} (paged)", "bound": "hbm",
                         "achieved": achieved, "peak": peak,
                         "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": ncu_traffic(args.workload, args.variant),
                         "algorithmic_bytes_per_launch": score_bytes},
            "clocks": clocks,
            "gpu_launches": int(launches),
            "timing": "each round: plain launches queued behind a GPU sleep, CUDA events around the fold and "
                      "the compress call",
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
    if ws > 1:
        torch.distributed.destroy_process_group()
    return result


def run_paged_e2e(args, tri, cache, wl, qc, kept, cnt, stream, ws, do_round):
    """A steady round end to end from host memory: the round's new tokens
    (K and V of PAGED_APPEND tokens per sequence, pinned) are copied to the
    device and written into fresh pages, the block table follows, the four
    calls run, and the kept indices and counts come back to the host.  The
    cache itself stays resident, as a serving cache does."""
    steps = max(1, min(args.steps, args.e2e_steps))
    B, L, H, bs, d = wl.budget, wl.num_layers, wl.num_kv_heads, wl.block_size, wl.head_dim
    per_seq = PAGED_APPEND // bs
    assert PAGED_APPEND % bs == 0 and all(n % bs == 0 for n in cache.lens)
    g = torch.Generator().manual_seed(gen.sub_seed(args.seed, "append_K", 1 << 20, 0))
    shape = (L, wl.batch * per_seq, bs * H * d)
    hk = torch.randn(shape, generator=g).to(torch.bfloat16).pin_memory()
    hv = torch.randn(shape, generator=g).to(torch.bfloat16).pin_memory()
    sk, sv = torch.empty(shape, dtype=torch.bfloat16, device=qc.device), \
        torch.empty(shape, dtype=torch.bfloat16, device=qc.device)
    hkept = torch.empty(kept.shape, dtype=kept.dtype, pin_memory=True)
    hcnt = torch.empty(cnt.shape, dtype=cnt.dtype, pin_memory=True)
    nb = cache.k.shape[1]
    kpool, vpool = cache.k.view(L, nb, -1), cache.v.view(L, nb, -1)
    table = cache.block_table.cpu()
    htable = torch.empty(table.shape, dtype=torch.int32, pin_memory=True)
    times = []
    for i in range(steps + 1):                     # the first round is a warm-up
        # host bookkeeping of the append: fresh pages for every sequence
        pages = []
        for b in range(wl.batch):
            n0 = cache.lens[b] // bs
            for j in range(per_seq):
                p = cache.free_blocks.pop()
                table[b, n0 + j] = p
                pages.append(p)
            cache.lens[b] += PAGED_APPEND
        htable.copy_(table)
        idx = torch.tensor(pages, dtype=torch.int64).pin_memory()
        dt = tri.desc_paged(cache.k, cache.v, cache.block_table, cache.lens)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(stream)
        cache.block_table.copy_(htable, non_blocking=True)
        di = idx.to(qc.device, non_blocking=True)
        sk.copy_(hk, non_blocking=True)
        sv.copy_(hv, non_blocking=True)
        kpool[:, di] = sk                          # the new tokens into their pages
        vpool[:, di] = sv
        do_round(dt)                               # fold, compress in place
        hkept.copy_(kept, non_blocking=True)
        hcnt.copy_(cnt, non_blocking=True)
        end.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            times.append(start.elapsed_time(end))
        # shrink every sequence back to B and free its tail pages (host)
        for b in range(wl.batch):
            keep = (B + bs - 1) // bs
            for j in range(keep, cache.lens[b] // bs):
                cache.free_blocks.append(int(table[b, j]))
                table[b, j] = 0
            cache.lens[b] = min(B, cache.lens[b])
        cache.block_table.copy_(table.to(qc.device))
    ms = max_over_ranks(float(np.sum(times)), ws, qc.device)
    keys = wl.units * (B + PAGED_APPEND)
    h2d = hk.numel() * 2 + hv.numel() * 2 + htable.numel() * 4 + len(pages) * 8
    d2h = hkept.numel() * 4 + hcnt.numel() * 4
    return {"value": keys * ws * steps / (ms / 1e3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps, "host_memory": "pinned",
            "what": "per round: the new tokens' K and V and the block table in, written into fresh pages, "
                    "fold + compress in place, kept indices and counts out; the cache stays resident"}


def run_e2e(args, tri, cache, d, wl, qc, w, kept, cnt, k_out, v_out, stream, job_keys, ws, positions=None,
            qpos=None):
    """Same step with the cache in pinned host memory: every step, H2D of K
    (all of it is scored) and of the centers, the four calls, D2H of the kept
    indices, counts and compacted K/V.  V is never copied: the descriptor
    points at the pinned host V, and the gather reads just the kept V rows
    over the bus (the library's out-of-place compaction takes V in mapped
    host memory).

    The results of step i go back on a second stream while step i+1's inputs
    come in (PCIe moves both directions at once): the outputs are double
    buffered, step i+1 overwrites K only after step i's compaction has read it
    (stream order), and a buffer is reused only after its copy-out has
    finished.  The timed region ends after the last copy-out."""
    steps = max(1, min(args.steps, args.e2e_steps))
    hk = torch.empty(cache.k.shape, dtype=cache.k.dtype, pin_memory=True)
    hv = torch.empty(cache.v.shape, dtype=cache.v.dtype, pin_memory=True)
    hk.copy_(cache.k)
    hv.copy_(cache.v)
    d = (tri.desc_contig(cache.k, hv) if wl.layout == "contig"
         else tri.desc_ragged(cache.k, hv, cache.cu_seqlens.cpu().tolist()))
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
        qc.copy_(hq, non_blocking=True)
        if hpos is not None:
            positions.copy_(hpos, non_blocking=True)
        stream.wait_event(copied[j])            # buffer j's previous copy-out is done
        if args.path == "compress" and args.variant == "max":
            tri.fold_offset_weights(qc, wl.theta, wl.offsets, wl.delta0, tri.PAIRING_HALF, out=w, stream=stream)
            tri.compress_max(d, w, B, tri.COMPACT_OUT_OF_PLACE, kp, cn, ko, vo, ws_e2e, stream=stream)
        elif args.path == "compress":
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
    v_rows = int(cnt.sum()) * cache.v.shape[-1] * 2        # the kept V rows the gather reads from the host
    h2d = hk.numel() * 2 + v_rows + hq.numel() * 4 + (hpos.numel() * 4 if hpos is not None else 0)
    d2h = hkept.numel() * 4 + hcnt.numel() * 4 + hko.numel() * 2 + hvo.numel() * 2
    return {"value": job_keys * steps / (ms / 1e3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "host_memory": "pinned",
            "values": "V stays in pinned host memory; the gather reads the kept V rows over the bus "
                      f"({v_rows / 1e6:.1f} MB of the {hv.numel() * 2 / 1e9:.2f} GB, counted in h2d_bytes_per_step)",
            "overlap": "results of step i copied back on a second stream while step i+1's inputs are copied in"}


# ---------------------------------------------------------------- the oracle as a CPU baseline

def oracle_unit_pipeline(orc, keys_bits, vals_bits, qc, wl, B, threads, variant="mean"):
    """The oracle's own path for one unit: literal per-offset average (or
    maximum), keep-highest, then a gather (or, for a paged cache, the
    in-place hole fill)."""
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
    if wl.layout == "paged":
        orc.holefill(keys_bits, kept, B)
        orc.holefill(vals_bits, kept, B)
    else:
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
    # a paged cache is timed in its steady rounds: rows of B + PAGED_APPEND keys
    n = wl.budget + PAGED_APPEND if wl.layout == "paged" else min(max(wl.seq_len, wl.len_hi, 4096), 32768)
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
                      f"select B={B}, {'hole fill' if wl.layout == 'paged' else 'gather'} K and V), fp64, "
                      f"{dt:.1f}s"}


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
    paged = wl.layout == "paged"
    if paged:
        # a paged cache is timed in its steady rounds: units of B + PAGED_APPEND
        # keys, as many per step as fill the step's time
        n = wl.budget + PAGED_APPEND
        units = int(min(64, max(1, rate * per_step_s / n)))
    else:
        n = int(min(32768, max(256, rate * per_step_s)))
        units = 1
    kb, vb, qc = cpu_sample(wl, n, args.seed)
    B = min(wl.budget, n)

    def step():
        for _ in range(units):
            oracle_unit_pipeline(orc, kb, vb, qc, wl, B, threads, args.variant)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = n * units * args.steps / dt
    kind = {"mean": "literal average", "max": "literal max", "pos": "literal average at per-key distances"}
    sample = (f"each step: {units} unit(s) of {n} keys of the {args.workload} workload ({kind[args.variant]} "
              f"over |D|={len(wl.offsets)} offsets, select B={B}, {'hole fill' if paged else 'gather'} K and V), "
              f"fp64")
    return {"impl": "reference", "metric": METRICS[args.variant],
            "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
            "config": {"workload": args.workload, "keys_per_step": n * units, "budget": B},
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
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 8 steady rounds for the paged workload)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen3_full", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time plain launches instead of a CUDA graph of the step")
    ap.add_argument("--path", default="calls", choices=["calls", "compress"],
                    help="calls: fold, score, select, compact as four calls (default); compress: fold + "
                         "tri_compress (tri_compress_max with --variant max)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "layers"],
                    help="N > 1: replicas (default): every rank compresses its own cache (weak scaling); "
                         "layers: one cache split by whole layers over the ranks (strong scaling)")
    ap.add_argument("--variant", default="mean", choices=["mean", "max", "pos"],
                    help="mean: the folded offset average (default); max: the max over the offsets; "
                         "pos: the offset average at per-key distances (pre-RoPE cache with positions)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = PAGED_ROUNDS if gen.WORKLOADS[args.workload].layout == "paged" else 1000
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

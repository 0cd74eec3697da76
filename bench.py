#!/usr/bin/env python
"""Benchmark of the streaming hot path of RTR-DiT's rerenderer on B200.

One step = one pass of the hot path for one DiT layer of the Wan-1.3B-shaped
workload: the current chunk (3 latent frames x 1560 tokens = 4680 queries,
12 heads, head_dim 128, bf16) attends under the frame-causal mask to
[1 anchored reference frame | 21 window frames | itself]
(``rtr_attn_frame_causal``), then its K/V are committed to the ring, evicting
the 3 oldest frames (``rtr_kvcache_append_frame``).

Prints one JSON line.  ``value`` is attention TFLOP/s of the whole job (the
algorithmic flops: visible query-key pairs x 4 x head_dim, summed over
heads, divided by the device time of the step); ``latent_frames_per_s_per_layer``
and the roofline fraction of the attention kernel come with it.  Usage:

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one independent replica stream per GPU.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
import argparse
import datetime
import hashlib
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

METRIC = "frame-causal attn TFLOP/s & latent frames/s per layer; % of BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
PROFILE = os.path.join(ROOT, "profiles", "fc_attn_fwd_tc__wan13_layer.md")
KERNEL_SOURCES = [os.path.join(ROOT, "causal_attention_rtr_b200", "csrc", f)
                  for f in ("attn_tc.cu", "ptx.cuh", "exp2_poly.h", "internal.h")]
APPEND_PROFILE = os.path.join(ROOT, "profiles", "kv_scatter__wan13_append.md")
APPEND_SOURCES = [os.path.join(ROOT, "causal_attention_rtr_b200", "csrc", f) for f in ("kv_copy.cu", "internal.h")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-extra-legs", action="store_true",
                    help="skip the prefill, backward and switching legs of the headline line")
    ap.add_argument("--workload", default="wan13_layer",
                    choices=["wan13_layer", "prefill_22", "prefill_22_bwd", "long_stream", "switch_14b", "tiny_f32",
                             "dit_block_13b", "append_13b"],
                    help="wan13_layer is the headline step; the others print one line each for reference")
    return ap.parse_args()


# ------------------------------------------------------------------ workload
def workload():
    from causal_attention_rtr_b200 import synth
    return synth.WAN13_LAYER


def visible_pairs_per_head(w):
    """Query-key pairs the mask leaves visible for one chunk: every chunk
    query sees all cached keys ((R + W) frames of k), and chunk frame c sees
    chunk frames 0..c."""
    cached = (w.ref_frames + w.window_frames) * w.k
    nq = w.chunk_frames * w.k
    chunk = sum(w.k * (c + 1) * w.k for c in range(w.chunk_frames))
    return nq * cached + chunk


def attn_flops(w):
    return 4.0 * w.head_dim * w.heads * visible_pairs_per_head(w)


def append_bytes(w):
    """Algorithmic bytes of committing one chunk: read K and V of the chunk,
    write them into their slots."""
    return 2 * 2 * w.chunk_frames * w.k * w.heads * w.head_dim * 2


def config_dict(w, world):
    return {"workload": w.name, "heads": w.heads, "head_dim": w.head_dim, "tokens_per_frame": w.k,
            "chunk_frames": w.chunk_frames, "ref_frames": w.ref_frames, "window_frames": w.window_frames,
            "queries": w.chunk_frames * w.k,
            "keys_per_head": (w.ref_frames + w.window_frames + w.chunk_frames) * w.k,
            "l2": "flushed between steps (256 MiB write outside the step events)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def profiled_traffic(profile=PROFILE, sources=KERNEL_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    if not os.path.exists(profile):
        return None
    h = hashlib.sha256()
    for p in sources:
        with open(p, "rb") as f:
            h.update(f.read())
    digest = h.hexdigest()
    vals = {}
    with open(profile) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip().strip("-* ")] = v.strip().strip("`")
    if vals.get("source_sha256") != digest:
        return None
    try:
        return int(float(vals["traffic_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def max_over_ranks(values, world, device):
    """Per-rank mean times -> the slowest rank's, identical on every rank
    (the job finishes when its slowest replica does)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(flops_per_step_per_rank, step_ms, world):
    """Whole-job TFLOP/s: every replica does the same work per step, timed
    by the slowest rank."""
    return world * flops_per_step_per_rank / (step_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        power = [num(r[3]) or 0.0 for r in rows]
        pmax = max(power)
        loaded = [r for r, p in zip(rows, power) if p >= 0.5 * pmax] or rows
        sm = [num(r[1]) for r in loaded if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in loaded for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(loaded[0][2]),
                "reasons": reasons, "samples": len(loaded), "power_w_max": pmax}


def device_bus_id(torch, dev_id):
    """PCI bus id of a device, for nvidia-smi -i."""
    props = torch.cuda.get_device_properties(dev_id)
    try:
        return f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except AttributeError:
        return os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0]


# ------------------------------------------------------------------ CPU oracle
def oracle_cache_for(w, x):
    import oracle
    o = oracle.ReferenceCache(w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, w.dtype)
    o.set_reference(x.ref_k, x.ref_v)
    for fk, fv in zip(x.window_k, x.window_v):
        o.append(fk, fv, 1)
    return o


def oracle_sample_flops(w, rows):
    cached = (w.ref_frames + w.window_frames) * w.k
    return sum(4.0 * w.head_dim * w.heads * (cached + (r // w.k + 1) * w.k) for r in rows)


def oracle_operands(w, x):
    """The oracle's decoded operands of the chunk's stream attention (queries,
    their logical positions, logical keys and values), assembled once so that
    the timed calls are the attention itself."""
    return oracle_cache_for(w, x).stream_operands(x.q, x.k_cur, x.v_cur, w.chunk_frames)


def oracle_rows(w, ops, rows, nthreads=0):
    import oracle
    Q, pos, K, V = ops
    return oracle.attention(Q[rows], pos[rows], K, V, w.k, True, None, nthreads)


def time_oracle(w, ops, seconds_target, nthreads=0, keep=None):
    """Time the oracle on sampled query rows (all heads) of the chunk,
    growing the sample until it takes about ``seconds_target``, on
    ``nthreads`` threads (0: all).  Returns (flops, seconds, rows); with a
    ``keep`` list, the last sample's outputs are appended to it."""
    import numpy as np
    nq = w.chunk_frames * w.k
    rng = np.random.default_rng(123)
    n = 2
    while True:
        rows = np.sort(rng.choice(nq, size=min(n, nq), replace=False))
        t0 = time.perf_counter()
        got = oracle_rows(w, ops, rows, nthreads)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * seconds_target or n >= nq:
            if keep is not None:
                keep.append(got)
            return oracle_sample_flops(w, rows), dt, rows
        n = min(nq, max(n * 2, int(n * seconds_target / max(dt, 1e-3) * 0.9)))


def output_accuracy(rtr, torch, w, x, dev, rows, want, dev_id):
    """The layer's attention on a fresh cache (the same history the oracle
    holds) through rtr_attn_frame_causal (bf16 output) and
    rtr_attn_frame_causal_f32out (fp32 output), against the oracle's rows."""
    import numpy as np
    c = rtr.rtr_kvcache_create(1, w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, "bf16", dev_id)
    try:
        rtr.rtr_kvcache_set_reference(c, 0, dev(x.ref_k), dev(x.ref_v))
        for fk, fv in zip(x.window_k, x.window_v):
            rtr.rtr_kvcache_append_frame(c, 0, dev(fk), dev(fv), 1)
        q, kc, vc = dev(x.q), dev(x.k_cur), dev(x.v_cur)
        o16 = torch.empty_like(q)
        o32 = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        rtr.rtr_attn_frame_causal(c, 0, q, kc, vc, w.chunk_frames, o16)
        rtr.rtr_attn_frame_causal_f32out(c, 0, q, kc, vc, w.chunk_frames, o32)
        torch.cuda.synchronize()
    finally:
        rtr.rtr_kvcache_destroy(c)
    idx = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
    res = {}
    for name, o in (("bf16_out", o16), ("f32_out", o32)):
        got = o.index_select(0, idx).double().cpu().numpy()
        diff = got - want
        res[name] = {"max_abs": float(np.max(np.abs(diff))),
                     "rel_l2": float(np.linalg.norm(diff.ravel()) / np.linalg.norm(want.ravel()))}
    res["rows"] = int(len(rows))
    res["bound"] = {"max_abs": 2e-2, "rel_l2": 5e-3}
    res["how"] = ("the cpu_baseline sample's query rows (all heads) against the fp64 oracle; f32_out is "
                  "rtr_attn_frame_causal_f32out, the same rows before the bf16 rounding")
    return res


def cpu_baseline_entry(flops, seconds, rows, w):
    import oracle
    return {"value": flops / seconds / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{len(rows)} query rows x {w.heads} heads of the chunk (of {w.chunk_frames * w.k}), "
                      f"fp64 C/OpenMP oracle, {flops / 1e9:.1f} GFLOP in {seconds:.2f} s",
            "cpu_model": cpu_model()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    if rank != 0:
        return
    from causal_attention_rtr_b200 import synth
    w = workload()
    x = synth.stream_layer_inputs(w)
    ops = oracle_operands(w, x)
    per_step = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    flops, dt, rows = time_oracle(w, ops, per_step)
    for _ in range(args.warmup):
        oracle_rows(w, ops, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_rows(w, ops, rows)
    total = time.perf_counter() - t0
    value = flops * args.steps / total / 1e12
    cb = cpu_baseline_entry(flops * args.steps, total, rows, w)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: N(0,1)*0.5 rounded to bf16, seed 1", "config": config_dict(w, world),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "note": "each step is the fp64 oracle on a bounded sample of the step's query rows"}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from causal_attention_rtr_b200 import rtr, synth

    torch.cuda.set_device(local_rank)
    dev_id = local_rank
    w = workload()
    x = synth.stream_layer_inputs(w, seed=w.seed + rank)

    def dev(a):
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()

    c = rtr.rtr_kvcache_create(1, w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, "bf16", dev_id)
    rtr.rtr_kvcache_set_reference(c, 0, dev(x.ref_k), dev(x.ref_v))
    for fk, fv in zip(x.window_k, x.window_v):
        rtr.rtr_kvcache_append_frame(c, 0, dev(fk), dev(fv), 1)
    q, kc, vc = dev(x.q), dev(x.k_cur), dev(x.v_cur)
    out = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    C = w.chunk_frames

    def step():
        rtr.rtr_attn_frame_causal(c, 0, q, kc, vc, C, out, 0.0, sh)
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, sh)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if rtr.rtr_get_device_status(dev_id, sh) != rtr.RTR_OK:
        raise RuntimeError("device status not OK after warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    bus = device_bus_id(torch, dev_id)
    sms = torch.cuda.get_device_properties(dev_id).multi_processor_count
    clocks = ClockSampler(bus)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches_before = rtr.rtr_kernel_launches()
    for s in range(K):
        flush.zero_()
        ev[s][0].record(stream)
        rtr.rtr_attn_frame_causal(c, 0, q, kc, vc, C, out, 0.0, sh)
        ev[s][1].record(stream)
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, sh)
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    launches_timed = rtr.rtr_kernel_launches() - launches_before
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    attn_ms = [e[0].elapsed_time(e[1]) for e in ev]
    app_ms = [e[1].elapsed_time(e[2]) for e in ev]
    step_ms = [a + b for a, b in zip(attn_ms, app_ms)]
    status = rtr.rtr_get_device_status(dev_id, sh)
    if status != rtr.RTR_OK:
        raise RuntimeError(f"device status {rtr.rtr_status_string(status)}")

    # ---- the append alone from a cold source: a 256 MiB read (twice L2)
    # evicts the chunk's K/V and leaves L2 holding clean lines, so the copy
    # reads its source from DRAM and pays for no one else's write-backs (a
    # flush by writing would leave L2 full of dirty lines for the copy's own
    # writes to evict)
    Kc = min(K, 50)
    evc = [_events(2) for _ in range(Kc)]
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    flush_sum = torch.empty((), dtype=torch.float32, device="cuda")
    for a, b in evc:
        torch.sum(flush_r, dim=0, out=flush_sum)
        a.record(stream)
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, sh)
        b.record(stream)
    torch.cuda.synchronize()
    cold_ms = [a.elapsed_time(b) for a, b in evc]
    del flush_r

    # ---- the same step with the chunk written by the attention launch
    # (rtr_attn_frame_causal_commit on a cache with commit room for the chunk),
    # alternated step by step with the separate attention + append so that
    # both see the same clocks (sustained load drifts the clock down).
    cf = rtr.rtr_kvcache_create_ex(1, w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, C, "bf16", dev_id)
    rtr.rtr_kvcache_set_reference(cf, 0, dev(x.ref_k), dev(x.ref_v))
    for fk, fv in zip(x.window_k, x.window_v):
        rtr.rtr_kvcache_append_frame(cf, 0, dev(fk), dev(fv), 1)
    for _ in range(max(3, args.warmup)):
        rtr.rtr_attn_frame_causal_commit(cf, 0, q, kc, vc, C, out, 0.0, sh)
    Kf = min(K, 50)
    evf = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(Kf)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(Kf):
        flush.zero_()
        evf[s][0].record(stream)
        rtr.rtr_attn_frame_causal_commit(cf, 0, q, kc, vc, C, out, 0.0, sh)
        evf[s][1].record(stream)
        flush.zero_()
        evf[s][2].record(stream)
        rtr.rtr_attn_frame_causal(c, 0, q, kc, vc, C, out, 0.0, sh)
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, sh)
        evf[s][3].record(stream)
    torch.cuda.synchronize()
    fused_ms = [e[0].elapsed_time(e[1]) for e in evf]
    sep_ms = [e[2].elapsed_time(e[3]) for e in evf]
    if rtr.rtr_get_device_status(dev_id, sh) != rtr.RTR_OK:
        raise RuntimeError("device status not OK after the fused-commit steps")
    rtr.rtr_kvcache_destroy(cf)

    # ---- end to end through the C ABI with host buffers (pinned), copies inside
    # the timed region: every step uploads its Q, K, V from pinned host memory
    # and reads its output back.  Two device buffer sets and one stream per copy
    # direction let step s+1's uploads and step s-1's download overlap step s's
    # kernels and each other (PCIe carries both directions at once).
    hq = torch.from_numpy(x.q.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(x.k_cur.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(x.v_cur.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Ke = min(K, 100)
    ho = [torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    bufs = [(torch.empty_like(q), torch.empty_like(kc), torch.empty_like(vc), torch.empty_like(out)) for _ in range(2)]
    up_stream, down_stream = torch.cuda.Stream(), torch.cuda.Stream()
    up_done = [torch.cuda.Event() for _ in range(Ke)]
    comp_done = [torch.cuda.Event() for _ in range(Ke)]
    down_done = [torch.cuda.Event() for _ in range(Ke)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def upload(s_):
        bq, bk, bv, _ = bufs[s_ % 2]
        with torch.cuda.stream(up_stream):
            if s_ >= 2:
                up_stream.wait_event(comp_done[s_ - 2])        # buffer set free again
            bq.copy_(hq, non_blocking=True)
            bk.copy_(hk, non_blocking=True)
            bv.copy_(hv, non_blocking=True)
            up_done[s_].record(up_stream)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    up_stream.wait_stream(stream)
    down_stream.wait_stream(stream)
    upload(0)
    for s in range(Ke):
        if s + 1 < Ke:
            upload(s + 1)
        bq, bk, bv, bo = bufs[s % 2]
        stream.wait_event(up_done[s])
        if s >= 2:
            stream.wait_event(down_done[s - 2])                 # output buffer read back
        rtr.rtr_attn_frame_causal(c, 0, bq, bk, bv, C, bo, 0.0, sh)
        rtr.rtr_kvcache_append_frame(c, 0, bk, bv, C, sh)
        comp_done[s].record(stream)
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(comp_done[s])
            ho[s % 2].copy_(bo, non_blocking=True)
            down_done[s].record(down_stream)
    stream.wait_event(down_done[Ke - 1])
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = [e_start.elapsed_time(e_end) / Ke]

    step_mean, attn_mean, app_mean, e2e_mean, fused_mean, sep_mean, cold_mean = max_over_ranks(
        [statistics.mean(step_ms), statistics.mean(attn_ms), statistics.mean(app_ms), statistics.mean(e2e_ms),
         statistics.mean(fused_ms), statistics.mean(sep_ms), statistics.mean(cold_ms)], world, "cuda")

    rtr.rtr_kvcache_destroy(c)
    if rank != 0:
        return

    flops = attn_flops(w)
    value = job_throughput(flops, step_mean, world)
    peaks = measured_peaks()
    peak_tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    attn_tflops = flops / (attn_mean * 1e-3) / 1e12
    app_gbs = append_bytes(w) / (app_mean * 1e-3) / 1e9
    traffic = profiled_traffic()
    app_traffic = profiled_traffic(APPEND_PROFILE, APPEND_SOURCES)
    per_clock = per_clock_peak_tflops(sms, clk.get("sm_mhz"))
    cold_gbs = append_bytes(w) / (cold_mean * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": step_mean, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: N(0,1)*0.5 rounded to bf16 (seed 1 + rank); stands in for projected Q/K/V of "
                "832x640 clips",
        "config": config_dict(w, world),
        "latent_frames_per_s_per_layer": world * w.chunk_frames / (step_mean * 1e-3),
        "pct_bf16_peak": 100.0 * attn_tflops / peak_tc,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak_tc, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak_tc, "traffic": traffic,
                     "kernel": "attn_fwd_tc<128> (rtr_attn_frame_causal)",
                     "peak_source": f"{peaks.get('source')} bf16_tflops (burst cuBLAS)",
                     "flops_per_launch": flops, "ms_per_launch": attn_mean,
                     "per_clock_peak": per_clock,
                     "frac_per_clock": attn_tflops / per_clock if per_clock else None,
                     "per_clock_how": "sms x 8192 flop/clk x median sampled SM clock"},
        "cache_update": {"kernel": "kv_scatter (rtr_kvcache_append_frame)", "bytes_per_launch": append_bytes(w),
                         "ms_per_launch": app_mean, "achieved_gbs": app_gbs, "peak_gbs": peak_hbm,
                         "frac": app_gbs / peak_hbm, "peak_source": f"{peaks.get('source')} hbm_gbs",
                         "traffic": app_traffic,
                         "source": "warm: in the step, right after the attention read the chunk's K/V",
                         "cold": {"ms_per_launch": cold_mean, "achieved_gbs": cold_gbs, "frac": cold_gbs / peak_hbm,
                                  "launches": Kc,
                                  "source": "cold: the append alone right after a 256 MiB read that evicts its "
                                            "source from L2 (L2 left clean)"}},
        "e2e": {"value": world * flops / (e2e_mean * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(3 * hq.numel() * 2), "d2h_bytes_per_step": int(ho[0].numel() * 2),
                "ms_per_step": e2e_mean,
                "how": "pinned host Q/K/V uploaded and output read back every step; copies of neighbouring "
                       "steps overlap the kernels (one stream per copy direction, two buffer sets)"},
        "fused_commit": {"entry": "rtr_attn_frame_causal_commit", "ms_per_step": fused_mean,
                         "separate_ms_per_step": sep_mean, "steps": Kf,
                         "value": job_throughput(flops, fused_mean, world), "unit": "TFLOP/s",
                         "how": "the same step (attention of the chunk + commit of its 3 frames) with the K/V "
                                "write done by the attention launch (cache with commit room 3), alternated step "
                                "by step with the separate attention + append (separate_ms_per_step)"},
        "gpu_launches": launches_timed,
        "clocks": clk,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(),
    }
    if world == 1 and not args.no_extra_legs:
        # the block-causal prefill, its backward and the 40-head switching
        # stream, each with its own clock record (single GPU only)
        cx = LegContext()
        line["prefill_22"] = clocked(cx, bus, leg_prefill_22, 100, False)
        line["prefill_22_bwd"] = clocked(cx, bus, leg_prefill_22_bwd, 40)
        line["switch_14b"] = clocked(cx, bus, leg_switch_14b, 8)
        # one Wan-1.3B-shaped DiT block around the attention (projections,
        # layer norms, cross attention); a failure here is reported in its
        # own entry and leaves the rest of the line intact
        try:
            line["dit_block_13b"] = clocked(cx, bus, leg_dit_block_13b, 20)
        except Exception as exc:                # noqa: BLE001 (reported, not hidden)
            line["dit_block_13b"] = {"error": f"{type(exc).__name__}: {exc}"}
        del cx
    if world == 1 and not args.no_cpu_baseline:
        ops = oracle_operands(w, x)
        kept = []
        fl, dt, rows = time_oracle(w, ops, 12.0, keep=kept)
        line["cpu_baseline"] = cpu_baseline_entry(fl, dt, rows, w)
        line["accuracy"] = output_accuracy(rtr, torch, w, x, dev, rows, kept[0], dev_id)
        fl1, dt1, rows1 = time_oracle(w, ops, 4.0, nthreads=1)
        line["cpu_baseline"]["single_core"] = {
            "value": fl1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
            "sample": f"{len(rows1)} query rows x {w.heads} heads, {fl1 / 1e9:.1f} GFLOP in {dt1:.2f} s"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ other workloads
def _events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


class LegContext:
    """What the timing legs of the non-headline workloads share (one GPU):
    the library, the stream, an L2 flush buffer, a seeded device generator
    (inputs drawn on the device as torch.randn * 0.5: values do not change
    the time) and the roofline denominators."""

    def __init__(self):
        import torch

        from causal_attention_rtr_b200 import rtr, synth
        self.torch, self.rtr, self.synth = torch, rtr, synth
        torch.cuda.set_device(0)
        self.sh = torch.cuda.current_stream().cuda_stream
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.gen = torch.Generator(device="cuda").manual_seed(0)
        peaks = measured_peaks()
        self.peak_tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        self.peak_hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        self.sms = torch.cuda.get_device_properties(0).multi_processor_count

    def rnd(self, shape, dtype=None, scale=0.5):
        torch = self.torch
        dtype = torch.bfloat16 if dtype is None else dtype
        return (torch.randn(shape, generator=self.gen, device="cuda", dtype=torch.float32) * scale).to(dtype)

    def check(self, what):
        if self.rtr.rtr_get_device_status(0, self.sh) != self.rtr.RTR_OK:
            raise RuntimeError(f"device status not OK after {what}")


def per_clock_peak_tflops(sms, sm_mhz):
    """Dense bf16 tensor peak at the sampled SM clock: 8192 flop per clock per
    SM (148 SMs x 8192 x 1.856 GHz = the nominal 2.25 PFLOP/s)."""
    return sms * 8192.0 * sm_mhz * 1e-6 if sm_mhz else None


def stream_flops(H, d, k, cached_frames, C):
    nq = C * k
    return 4.0 * d * H * (nq * cached_frames * k + sum(k * (c + 1) * k for c in range(C)))


def prefill_visible_pairs(n, k):
    return sum(min(n, (i // k + 1) * k) for i in range(n))


def leg_prefill_22(cx, calls, with_fill=True):
    """The 22-frame block-causal prefill (34,320 tokens, 12 heads), L2
    flushed before each call; optionally the prefill into a cache alternated
    call by call with the plain one."""
    rtr, w = cx.rtr, cx.synth.PREFILL_22
    n, H, d = w.chunk_frames * w.k, w.heads, w.head_dim
    q, k, v = (cx.rnd((n, H, d)) for _ in range(3))
    out = cx.torch.empty_like(q)
    flops = 4.0 * d * H * prefill_visible_pairs(n, w.k)
    for _ in range(3):
        rtr.rtr_attn_block_causal_prefill(q, k, v, n, H, d, w.k, "bf16", out, 0.0, 0, cx.sh)
    evs = [_events(2) for _ in range(calls)]
    for a, b in evs:
        cx.flush.zero_()
        a.record()
        rtr.rtr_attn_block_causal_prefill(q, k, v, n, H, d, w.k, "bf16", out, 0.0, 0, cx.sh)
        b.record()
    cx.torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    cx.check("the prefill")
    res = {"config": w.name, "ms_per_call": ms, "tflop_per_call": flops / 1e12, "tflops": flops / ms / 1e9,
           "frac_of_bf16_peak": flops / ms / 1e9 / cx.peak_tc, "calls": calls}
    if with_fill:
        F = w.chunk_frames
        c = rtr.rtr_kvcache_create(1, H, d, w.k, 1, F - 1, "bf16", 0)
        for _ in range(3):
            rtr.rtr_attn_block_causal_prefill_cache(c, 0, q, k, v, F, True, out, 0.0, cx.sh)
        tf, tp = [], []
        for _ in range(min(calls, 50)):
            for fill, acc in ((True, tf), (False, tp)):
                cx.flush.zero_()
                a, b = _events(2)
                a.record()
                if fill:
                    rtr.rtr_attn_block_causal_prefill_cache(c, 0, q, k, v, F, True, out, 0.0, cx.sh)
                else:
                    rtr.rtr_attn_block_causal_prefill(q, k, v, n, H, d, w.k, "bf16", out, 0.0, 0, cx.sh)
                b.record()
                acc.append((a, b))
        cx.torch.cuda.synchronize()
        cx.check("the prefill into the cache")
        rtr.rtr_kvcache_destroy(c)
        res["with_cache_fill"] = {
            "entry": "rtr_attn_block_causal_prefill_cache (reference + 21 window frames written by the attention "
                     "launch)",
            "ms_per_call": statistics.mean(a.elapsed_time(b) for a, b in tf),
            "plain_ms_per_call": statistics.mean(a.elapsed_time(b) for a, b in tp),
            "bytes_written": 2.0 * n * H * d * 2,
            "how": "alternated call by call with the plain prefill, L2 flushed before each"}
    return res


def leg_prefill_22_bwd(cx, calls):
    """Backward of the 22-frame prefill: algorithmic work 5 matmuls per
    visible (query, key) pair = 10 * d flops (2.5x the forward's 4 * d)."""
    rtr, w = cx.rtr, cx.synth.PREFILL_22
    n, H, d = w.chunk_frames * w.k, w.heads, w.head_dim
    q, k, v, do = (cx.rnd((n, H, d)) for _ in range(4))
    out = cx.torch.empty_like(q)
    lse = cx.torch.empty((H, n), dtype=cx.torch.float32, device="cuda")
    dq, dk, dv = (cx.torch.empty_like(q) for _ in range(3))
    flops = 10.0 * d * H * prefill_visible_pairs(n, w.k)
    rtr.rtr_attn_block_causal_prefill_lse(q, k, v, n, H, d, w.k, "bf16", out, lse, 0.0, 0, cx.sh)
    for _ in range(3):
        rtr.rtr_attn_block_causal_backward(q, k, v, out, do, lse, n, H, d, w.k, "bf16", dq, dk, dv, 0.0, 0, cx.sh)
    evs = [_events(2) for _ in range(calls)]
    for a, b in evs:
        cx.flush.zero_()
        a.record()
        rtr.rtr_attn_block_causal_backward(q, k, v, out, do, lse, n, H, d, w.k, "bf16", dq, dk, dv, 0.0, 0, cx.sh)
        b.record()
    cx.torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    cx.check("the backward")
    return {"config": w.name + ", backward (dQ, dK, dV)", "ms_per_call": ms, "tflop_per_call": flops / 1e12,
            "tflops": flops / ms / 1e9, "frac_of_bf16_peak": flops / ms / 1e9 / cx.peak_tc, "calls": calls,
            "kernels": "bwd_prep + bwd_dkdv (S^T, dP^T, dV, dK) + bwd_dq (S, dP, dQ): 7 tile MMAs per visible "
                       "tile pair for 5 of algorithmic work"}


def leg_switch_14b(cx, passes):
    """The 64-frame, 40-head stream with its three switches, frame by frame:
    self-attention (reference + window + frame), cross-attention to 512 text
    tokens, append; at frames 16/32/48 the text cache is reset and refilled,
    the window cut to its newest frame and the reference overwritten.  Each
    part is timed with its own events; ``passes`` passes on fresh caches
    after one untimed pass."""
    rtr, torch, w = cx.rtr, cx.torch, cx.synth.SWITCH_14B
    H, d, k, W, T = w.heads, w.head_dim, w.k, w.window_frames, w.text_tokens
    ref, kt, vt = cx.rnd((k, H, d)), cx.rnd((T, H, d)), cx.rnd((T, H, d))
    frames = [tuple(cx.rnd((k, H, d)) for _ in range(3)) for _ in range(2)]
    out = torch.empty_like(frames[0][0])
    xout = torch.empty_like(out)
    self_flops = cross_flops = 0.0
    count = 0
    for f in range(w.frames_total):
        if f > 0 and f % w.switch_every == 0:
            count = min(count, 1)
        self_flops += stream_flops(H, d, k, 1 + count, 1)
        cross_flops += 4.0 * d * H * k * T
        count = min(W, count + 1)

    def one_pass():
        c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
        x = rtr.rtr_crossattn_create(1, H, d, T, "bf16", 0)
        rtr.rtr_kvcache_set_reference(c, 0, ref, ref, cx.sh)
        rtr.rtr_crossattn_set_text(x, 0, kt, vt, T, cx.sh)
        torch.cuda.synchronize()
        ev = []
        a, b = _events(2)
        a.record()
        for f in range(w.frames_total):
            e = _events(5)
            e[0].record()
            if f > 0 and f % w.switch_every == 0:
                rtr.rtr_crossattn_reset(x)
                rtr.rtr_crossattn_set_text(x, 0, vt, kt, T, cx.sh)
                rtr.rtr_kvcache_retain_last(c, 0, 1)
                rtr.rtr_kvcache_set_reference(c, 0, ref, ref, cx.sh)
            e[1].record()
            q, kk, vv = frames[f % 2]
            rtr.rtr_attn_frame_causal(c, 0, q, kk, vv, 1, out, 0.0, cx.sh)
            e[2].record()
            rtr.rtr_attn_cross(x, 0, q, k, xout, 0.0, cx.sh)
            e[3].record()
            rtr.rtr_kvcache_append_frame(c, 0, kk, vv, 1, cx.sh)
            e[4].record()
            ev.append(e)
        b.record()
        torch.cuda.synchronize()
        parts = [sum(e[i].elapsed_time(e[i + 1]) for e in ev) for i in range(4)]
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)
        return a.elapsed_time(b), parts

    one_pass()
    runs = [one_pass() for _ in range(passes)]
    cx.check("the switching stream")
    ms = statistics.mean(r[0] for r in runs)
    sw, self_ms, cross_ms, app_ms = (statistics.mean(r[1][i] for r in runs) for i in range(4))
    flops = self_flops + cross_flops
    frame_bytes = 4.0 * k * H * d * 2
    return {"config": w.name, "total_ms": ms, "ms_per_frame": ms / w.frames_total,
            "attention_tflop": flops / 1e12, "tflops": flops / ms / 1e9,
            "frac_of_bf16_peak": flops / ms / 1e9 / cx.peak_tc,
            "latent_frames_per_s": w.frames_total / (ms / 1e3),
            "self_attention": {"ms": self_ms, "tflop": self_flops / 1e12, "tflops": self_flops / self_ms / 1e9,
                               "frac_of_bf16_peak": self_flops / self_ms / 1e9 / cx.peak_tc},
            "cross_attention": {"ms": cross_ms, "tflop": cross_flops / 1e12, "tflops": cross_flops / cross_ms / 1e9,
                                "frac_of_bf16_peak": cross_flops / cross_ms / 1e9 / cx.peak_tc},
            "append": {"ms": app_ms, "bytes": frame_bytes * w.frames_total,
                       "achieved_gbs": frame_bytes * w.frames_total / app_ms / 1e6},
            "switch_ms": sw, "passes": passes,
            "note": "parts timed with events around each call of every frame (sums over the 64 frames); "
                    "one untimed pass of the whole stream first"}


def leg_long_stream(cx):
    """The 30-layer, 120-frame stream (chunks of 3, 2 denoising steps), one
    stream; plus the 30 layers' appends of one chunk back to back after an L2
    flush (the append kernel's asymptote, labelled as such)."""
    rtr, torch, w = cx.rtr, cx.torch, cx.synth.LONG_STREAM
    L, H, d, k, C, W = w.layers, w.heads, w.head_dim, w.k, w.chunk_frames, w.window_frames
    c = rtr.rtr_kvcache_create(L, H, d, k, 1, W, "bf16", 0)
    ref = cx.rnd((k, H, d))
    for l in range(L):
        rtr.rtr_kvcache_set_reference(c, l, ref, ref, cx.sh)
    chunks = [tuple(cx.rnd((C * k, H, d)) for _ in range(3)) for _ in range(2)]  # reused inputs
    out = torch.empty_like(chunks[0][0])
    n_chunks = w.frames_total // C
    flops = 0.0
    for _ in range(3):                               # warm-up: attention leaves the cache unchanged
        rtr.rtr_attn_frame_causal(c, 0, chunks[0][0], chunks[0][1], chunks[0][2], C, out, 0.0, cx.sh)
    torch.cuda.synchronize()
    a, b = _events(2)
    a.record()
    for ch in range(n_chunks):
        cached = 1 + min(W, ch * C)
        for step_ in range(w.steps_per_chunk):
            q, kk, vv = chunks[(ch + step_) % 2]
            for l in range(L):
                rtr.rtr_attn_frame_causal(c, l, q, kk, vv, C, out, 0.0, cx.sh)
                flops += stream_flops(H, d, k, cached, C)
        for l in range(L):
            rtr.rtr_kvcache_append_frame(c, l, kk, vv, C, cx.sh)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    batch_bytes = L * 4.0 * C * k * H * d * 2
    srcs = [(cx.rnd((C * k, H, d)), cx.rnd((C * k, H, d))) for _ in range(L)]
    bts = []
    for _ in range(5):
        cx.flush.zero_()
        a2, b2 = _events(2)
        a2.record()
        for l in range(L):
            rtr.rtr_kvcache_append_frame(c, l, srcs[l][0], srcs[l][1], C, cx.sh)
        b2.record()
        torch.cuda.synchronize()
        bts.append(a2.elapsed_time(b2))
    bms = statistics.mean(bts[1:])
    st = rtr.rtr_get_device_status(0, cx.sh)
    rtr.rtr_kvcache_destroy(c)
    return {"config": w.name, "total_ms": ms, "attention_tflop": flops / 1e12,
            "tflops": flops / ms / 1e9, "frac_of_bf16_peak": flops / ms / 1e9 / cx.peak_tc,
            "latent_frames_per_s_per_layer": w.frames_total / (ms / 1e3 / L),
            "latent_frames_per_s_all_layers": w.frames_total / (ms / 1e3),
            "device_status": rtr.rtr_status_string(st),
            "append_batch_30_layers": {
                "what": "30 rtr_kvcache_append_frame calls (one per layer, 3 frames each, distinct sources) back "
                        "to back after an L2 flush: the append kernel's asymptote, not a step of the stream",
                "bytes": batch_bytes, "ms": bms, "achieved_gbs": batch_bytes / bms / 1e6, "peak_gbs": cx.peak_hbm,
                "frac": batch_bytes / bms / 1e6 / cx.peak_hbm},
            "note": "attention calls + appends of 30 layers x 40 chunks x 2 steps, one stream"}


def leg_dit_block_13b(cx, calls):
    """One Wan-1.3B-shaped DiT block on the 3-frame chunk (12 heads x 128,
    30 x 52 tokens per frame, 1 reference + 21 window frames, 512 text
    tokens, feed-forward 8960, random bf16 weights), alternated with the
    attention alone on the same cache, L2 flushed before each."""
    rtr, torch, w = cx.rtr, cx.torch, cx.synth.WAN13_LAYER
    H, d, k, W, C, F, T = w.heads, w.head_dim, w.k, w.window_frames, w.chunk_frames, 8960, 512
    D, n = H * d, C * k
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    x = rtr.rtr_crossattn_create(1, H, d, T, "bf16", 0)
    rtr.rtr_kvcache_set_reference(c, 0, cx.rnd((k, H, d)), cx.rnd((k, H, d)), cx.sh)
    for _ in range(W):
        rtr.rtr_kvcache_append_frame(c, 0, cx.rnd((k, H, d)), cx.rnd((k, H, d)), 1, cx.sh)
    rtr.rtr_crossattn_set_text(x, 0, cx.rnd((T, H, d)), cx.rnd((T, H, d)), T, cx.sh)
    shapes = {"wqkv": (D, 3 * D), "bqkv": (3 * D,), "wo": (D, D), "bo": (D,), "wq2": (D, D), "bq2": (D,),
              "wo2": (D, D), "bo2": (D,), "w1": (D, F), "b1": (F,), "w2": (F, D), "b2": (D,)}
    wts = {name: cx.rnd(shp, scale=(0.1 if name[0] == "b" else shp[0] ** -0.5)) for name, shp in shapes.items()}
    dw = rtr.dit_weights(wts, F)
    pw = rtr.rtr_dit_pack_weights(dw, D, 0, cx.sh)       # once, outside the timed calls
    mod = cx.rnd((6, D), scale=0.2)
    hid0 = cx.rnd((n, D), scale=1.0)
    hid = hid0.clone()
    q, kk, vv = cx.rnd((n, H, d)), cx.rnd((n, H, d)), cx.rnd((n, H, d))
    out = torch.empty_like(q)
    for _ in range(3):
        hid.copy_(hid0)
        rtr.rtr_dit_block_forward_packed(c, x, 0, pw, mod, hid, C, 30, 52, 22, False, cx.sh)
        hid.copy_(hid0)
        rtr.rtr_dit_block_forward(c, x, 0, dw, mod, hid, C, 30, 52, 22, False, cx.sh)
        rtr.rtr_attn_frame_causal(c, 0, q, kk, vv, C, out, 0.0, cx.sh)
    tb, tr, ta = [], [], []
    for _ in range(calls):
        hid.copy_(hid0)
        cx.flush.zero_()
        a, b = _events(2)
        a.record()
        rtr.rtr_dit_block_forward_packed(c, x, 0, pw, mod, hid, C, 30, 52, 22, False, cx.sh)
        b.record()
        hid.copy_(hid0)
        cx.flush.zero_()
        a3, b3 = _events(2)
        a3.record()
        rtr.rtr_dit_block_forward(c, x, 0, dw, mod, hid, C, 30, 52, 22, False, cx.sh)
        b3.record()
        cx.flush.zero_()
        a2, b2 = _events(2)
        a2.record()
        rtr.rtr_attn_frame_causal(c, 0, q, kk, vv, C, out, 0.0, cx.sh)
        b2.record()
        tb.append((a, b))
        tr.append((a3, b3))
        ta.append((a2, b2))
    torch.cuda.synchronize()
    cx.check("the DiT block")
    rtr.rtr_dit_packed_destroy(pw)
    rtr.rtr_kvcache_destroy(c)
    rtr.rtr_crossattn_destroy(x)
    ms = statistics.mean(a.elapsed_time(b) for a, b in tb)
    rms = statistics.mean(a.elapsed_time(b) for a, b in tr)
    ams = statistics.mean(a.elapsed_time(b) for a, b in ta)
    attn = stream_flops(H, d, k, 1 + W, C)
    cross = 4.0 * d * H * n * T
    mm = 2.0 * n * (6.0 * D * D + 2.0 * D * F)
    total = attn + cross + mm
    return {"config": "Wan-1.3B-shaped DiT block: H=12 d=128 k=1560 (30x52), chunk of 3 frames vs ref 1 + window "
                      "21, text 512, FFN 8960, random bf16 weights",
            "ms_per_block": ms, "latent_frames_per_s_per_block": C / (ms / 1e3),
            "tflop_per_block": total / 1e12, "tflops": total / ms / 1e9,
            "frac_of_bf16_peak": total / ms / 1e9 / cx.peak_tc,
            "self_attention_tflop": attn / 1e12, "projection_tflop": mm / 1e12,
            "attention_alone_ms": ams, "attention_share": ams / ms,
            "rest_ms": ms - ams, "rest_tflops": (total - attn) / (ms - ams) / 1e9,
            "row_major_weights_ms_per_block": rms,
            "how": "rtr_dit_block_forward_packed (weights packed once by rtr_dit_pack_weights, outside the timed "
                   "calls), alternated with rtr_dit_block_forward on the row-major weights and with the attention "
                   "alone on the same cache, L2 flushed before each"}


def leg_append_13b(cx, calls):
    """The headline step's cache update alone: rtr_kvcache_append_frame of a
    3-frame Wan-1.3B chunk (12 heads x 128, k = 1560) into a full 21-frame
    window (every call evicts 3 frames), each call right after a 256 MiB
    read that evicts its source from L2, so the source comes from DRAM."""
    rtr, torch, w = cx.rtr, cx.torch, cx.synth.WAN13_LAYER
    H, d, k, W, C = w.heads, w.head_dim, w.k, w.window_frames, w.chunk_frames
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    rtr.rtr_kvcache_set_reference(c, 0, cx.rnd((k, H, d)), cx.rnd((k, H, d)), cx.sh)
    for _ in range(W):
        rtr.rtr_kvcache_append_frame(c, 0, cx.rnd((k, H, d)), cx.rnd((k, H, d)), 1, cx.sh)
    kc, vc = cx.rnd((C * k, H, d)), cx.rnd((C * k, H, d))
    for _ in range(3):
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, cx.sh)
    # flush by reading 256 MiB: the source leaves L2, and L2 holds clean lines
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    flush_sum = torch.empty((), dtype=torch.float32, device="cuda")
    evs = [_events(2) for _ in range(calls)]
    for a, b in evs:
        torch.sum(flush_r, dim=0, out=flush_sum)
        a.record()
        rtr.rtr_kvcache_append_frame(c, 0, kc, vc, C, cx.sh)
        b.record()
    torch.cuda.synchronize()
    cx.check("the appends")
    rtr.rtr_kvcache_destroy(c)
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    nbytes = 4.0 * C * k * H * d * 2
    return {"config": w.name + ", append of the 3-frame chunk (cold source)", "ms_per_call": ms,
            "bytes_per_call": nbytes, "achieved_gbs": nbytes / ms / 1e6, "peak_gbs": cx.peak_hbm,
            "frac": nbytes / ms / 1e6 / cx.peak_hbm, "calls": calls}


def leg_tiny_f32(cx, warmup):
    """The fp32 correctness stream (10 frames, one at a time): launch-bound."""
    rtr, torch, w = cx.rtr, cx.torch, cx.synth.TINY_F32
    H, d, k, W = w.heads, w.head_dim, w.k, w.window_frames
    ref = cx.rnd((k, H, d), torch.float32, 1.0)
    fr = [tuple(cx.rnd((k, H, d), torch.float32, 1.0) for _ in range(3)) for _ in range(w.frames_total)]
    out = torch.empty_like(fr[0][0])
    for _ in range(max(3, warmup)):               # warm-up streams on throwaway caches
        cw = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "f32", 0)
        rtr.rtr_kvcache_set_reference(cw, 0, ref, ref, cx.sh)
        for q, kk, vv in fr:
            rtr.rtr_attn_frame_causal(cw, 0, q, kk, vv, 1, out, 0.0, cx.sh)
            rtr.rtr_kvcache_append_frame(cw, 0, kk, vv, 1, cx.sh)
        torch.cuda.synchronize()
        rtr.rtr_kvcache_destroy(cw)
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "f32", 0)
    rtr.rtr_kvcache_set_reference(c, 0, ref, ref, cx.sh)
    torch.cuda.synchronize()
    a, b = _events(2)
    a.record()
    for q, kk, vv in fr:
        rtr.rtr_attn_frame_causal(c, 0, q, kk, vv, 1, out, 0.0, cx.sh)
        rtr.rtr_kvcache_append_frame(c, 0, kk, vv, 1, cx.sh)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    rtr.rtr_kvcache_destroy(c)
    return {"config": w.name, "dtype": "f32", "total_ms": ms, "ms_per_frame": ms / w.frames_total,
            "note": "correctness workload; time is launch-bound"}


def clocked(cx, bus, fn, *args):
    """Run one leg with its own clock record; adds the fraction of the
    per-clock tensor peak where the leg reports TFLOP/s."""
    sampler = ClockSampler(bus)
    sampler.start()
    try:
        res = fn(cx, *args)
    finally:
        clk = sampler.stop()
    res["clocks"] = clk
    pc = per_clock_peak_tflops(cx.sms, res["clocks"].get("sm_mhz"))
    if pc and "tflops" in res:
        res["frac_per_clock"] = res["tflops"] / pc
    return res


def run_other(args):
    """One JSON line for a workload other than the headline one (single GPU)."""
    cx = LegContext()
    bus = device_bus_id(cx.torch, 0)
    legs = {"prefill_22": (leg_prefill_22, max(1, args.steps)),
            "prefill_22_bwd": (leg_prefill_22_bwd, max(1, args.steps)),
            "long_stream": (leg_long_stream,),
            "switch_14b": (leg_switch_14b, 3),
            "dit_block_13b": (leg_dit_block_13b, min(max(1, args.steps), 50)),
            "tiny_f32": (leg_tiny_f32, args.warmup),
            "append_13b": (leg_append_13b, max(1, args.steps))}
    fn, *rest = legs[args.workload]
    line = {"workload": args.workload, "n_gpus": 1, "dtype": "bf16",
            "data": "synthetic (torch.randn * 0.5 on device)"}
    line.update(clocked(cx, bus, fn, *rest))
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.workload != "wan13_layer":
        run_other(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

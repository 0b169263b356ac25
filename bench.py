"""Benchmark of the fused MoE decode step on B200.

Default workload: the large synthetic MoE decoder (16 layers, d_model 4096,
32/8 heads of 128, 128 experts top-8, expert and shared FFN 1536, vocab
64000, about 80 GB of bf16 weights) decoding greedily at batch 1 with a
4095-position prefilled cache.  Each step streams about 7.6 GB, far more than
the 126 MB L2, so no flush is needed between steps.

One JSON line on rank 0.  ``--impl reference`` times the CPU oracle instead.
Under torchrun each rank runs an independent replica (the path does not shard).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
NOMINAL_HBM_GBS = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---- distributed plumbing (replicas only) -----------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_init(ws, backend):
    import datetime

    import torch.distributed as dist

    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


# ---- clocks -----------------------------------------------------------------------
# Throttle-reason bits of NVML's clocks-event mask (read only; nothing is set).
_REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """Samples the SM clock and the throttle reasons every 10 ms during the
    timed region (NVML from a thread; nvidia-smi at its 200 ms floor if NVML is
    unavailable).  Only reads the GPU's state."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_s: float = 0.01):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.thread = None
        self.samples = []
        self.max_mhz = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self._start_smi()
            return
        self.stop_flag = threading.Event()

        def run():
            while not self.stop_flag.is_set():
                try:
                    self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(reasons_fn(h))))
                except Exception:
                    pass
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            reasons = sorted({name for _, mask in self.samples for bit, name in _REASON_BITS.items()
                              if mask & bit})
            return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml, 10 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows), "source": "nvidia-smi, 200 ms"}


# ---- bytes per step ---------------------------------------------------------------
def step_bytes(m, B, T, lengths_after, union_per_step):
    """Algorithmic bytes of one step: every weight read once (routed experts
    counted once per distinct expert per layer), plus the KV read of each
    sequence (its length after the append), the KV append, embedding rows and
    the logits write."""
    d, hd = m.d_model, m.head_dim
    qkv = (m.n_q_heads + 2 * m.n_kv_heads) * hd * d
    wo = d * m.n_q_heads * hd
    router = m.n_experts * d
    shared = 3 * m.shared_ffn * d
    per_layer = 2 * (qkv + wo + router + shared + 2 * d)
    expert = 3 * m.expert_ffn * d * 2
    kv_read = sum(2 * m.n_layers * m.n_kv_heads * hd * L * 2 for L in lengths_after)
    kv_write = 2 * m.n_layers * m.n_kv_heads * hd * B * T * 2
    lm = (m.vocab * d + d) * 2
    return (m.n_layers * per_layer + union_per_step * expert + lm + kv_read + kv_write
            + B * T * d * 2 + B * T * m.vocab * 4)


def profile_traffic(kernel_key: str):
    """DRAM traffic per launch recorded by ncu in profiles/, if the kernel source
    has not changed since the capture."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "megakernel_traffic.md")
    src = os.path.join(ROOT, "decode_megakernel_06_b200", "csrc", "mk_kernel.cu")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    m = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or m.group(1) != sha:
        return None
    t = re.search(rf"{kernel_key}:\s*([0-9.]+)", text)
    return float(t.group(1)) if t else None


# ---- our arm ----------------------------------------------------------------------
def build_workload(kind, B, device):
    import torch

    from synthetic import make_context_lengths, make_kv_cache, make_tokens, make_weights, workload

    if kind == "small":
        wl = workload("small") if B == 1 else workload("small_batch", B)
    else:
        wl = workload(kind, B) if kind in ("large", "profile", "dense") else workload(kind)
    m = wl.model
    t0 = time.perf_counter()
    w = make_weights(m, wl.seed, device)
    torch.cuda.synchronize()
    gen_s = time.perf_counter() - t0
    return wl, m, w, gen_s


def time_steps(dec, m, k, v, B, T, ctx, steps, warmup, device):
    """Greedy decode on the device: step s reads the argmax of step s-1."""
    import torch

    from synthetic import make_tokens

    n = warmup + steps
    pos = torch.tensor([[ctx[b] + s * T for b in range(B)] for s in range(n)], dtype=torch.int32,
                       device=device)
    bufs = [torch.tensor(make_tokens(m.vocab, B * T, 123), dtype=torch.int32, device=device),
            torch.empty(B * T, dtype=torch.int32, device=device)]
    logits = torch.empty((B * T, m.vocab), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    for s in range(warmup):
        rc = dec.step(bufs[s % 2], pos[s], B, T, k, v, logits, bufs[(s + 1) % 2])
        assert rc == 0, rc
    assert dec.status() == 0
    dec.stats(reset=True)
    barrier(device)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    torch.cuda.nvtx.range_push("timed_region")  # lets a profiler list exactly these launches
    ev[0].record(stream)
    for i in range(steps):
        s = warmup + i
        dec.step(bufs[s % 2], pos[s], B, T, k, v, logits, bufs[(s + 1) % 2])
        ev[i + 1].record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(device)
    st = dec.status()
    assert st == 0, st
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = ev[0].elapsed_time(ev[steps])
    stats = dec.stats(reset=True)
    return total, per, stats


def time_e2e(dec, m, k, v, B, T, ctx, steps, warmup):
    """Through the host-buffer entry point: H2D tokens/positions, the step, D2H
    argmax, every step."""
    import torch

    from synthetic import make_tokens

    th = torch.tensor(make_tokens(m.vocab, B * T, 321), dtype=torch.int32).pin_memory()
    ph = torch.empty(B, dtype=torch.int32).pin_memory()
    out = torch.empty(B * T, dtype=torch.int32).pin_memory()
    for s in range(warmup):
        ph.copy_(torch.tensor([ctx[b] + s * T for b in range(B)], dtype=torch.int32))
        assert dec.step_host(th, ph, B, T, k, v, out) == 0
        th.copy_(out)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(steps):
        s = warmup + i
        ph.copy_(torch.tensor([ctx[b] + s * T for b in range(B)], dtype=torch.int32))
        assert dec.step_host(th, ph, B, T, k, v, out) == 0
        th.copy_(out)
    dt = time.perf_counter() - t0
    return dt, (th.numel() + ph.numel()) * 4, out.numel() * 4


def oracle_sample(m, w, k_dev, v_dev, B, T, ctx, n_steps=1, min_compute_s=0.0, threads=0):
    """The CPU oracle as it stands on the same workload: whole decode steps
    (all layers), weights copied from the device on demand; the copy time is
    excluded from the compute time and reported beside it.  Runs ``n_steps``
    steps, or more until the compute time reaches ``min_compute_s`` (at most
    40 steps)."""
    import numpy as np

    import oracle
    from oracle import step as ostep
    from synthetic import bf16_bits, make_tokens

    threads = oracle.set_threads(threads)
    src = ostep.WeightSource(w, cache=False)
    # only the sequences' live layers of the cache are needed; copy it once
    kh = bf16_bits(k_dev[:, :B]).copy()
    vh = bf16_bits(v_dev[:, :B]).copy()
    toks = make_tokens(m.vocab, B * T, 555)
    pos = list(ctx)
    t_total = 0.0
    fetch_before = 0.0
    import time as _t

    orig = src._get

    def timed(key, fetch):
        t0 = _t.perf_counter()
        a = orig(key, fetch)
        timed.fetch += _t.perf_counter() - t0
        return a

    timed.fetch = 0.0
    src._get = timed
    done = 0
    while done < n_steps or (t_total - timed.fetch < min_compute_s and done < 40):
        t0 = _t.perf_counter()
        r = ostep.decode_step(m, src, kh, vh, toks, pos, B, T)
        t_total += _t.perf_counter() - t0
        toks = [int(x) for x in r.argmax]
        pos = [p + T for p in pos]
        done += 1
    compute = t_total - timed.fetch
    return {"compute_s": compute, "fetch_s": timed.fetch, "steps": done, "threads": threads,
            "tokens": done * B * T}


def trace_step(dec, m, k, v, B, T, ctx, device, out=sys.stderr, save=None):
    """One traced step: per op, when the first / last warp started it and when
    the last warp finished it (microseconds from the step's first op start)."""
    import torch

    import decode_megakernel_06_b200 as mk

    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    rc, info, ops = mk.mk_plan_describe(dec.desc, n_sm, B, T)
    nw = info.n_cta * info.warps_per_cta
    buf = torch.zeros((info.n_ops, nw, mk.MK_TRACE_WORDS), dtype=torch.int64, device=device)
    pos = torch.tensor([c for c in ctx], dtype=torch.int32, device=device)
    tok = torch.zeros(B * T, dtype=torch.int32, device=device)
    am = torch.empty(B * T, dtype=torch.int32, device=device)
    dec.set_trace(buf)
    assert dec.step(tok, pos, B, T, k, v, None, am) == 0
    assert dec.status() == 0
    dec.set_trace(None)
    t = buf.cpu().numpy()[:, :, [0, 3]].astype("float64")  # (inputs ready, arrived) per warp
    if save:
        import numpy as np

        np.save(save, buf.cpu().numpy())
    t0 = t[:, :, 0][t[:, :, 0] > 0].min()
    rows = []
    for i, (typ, layer, d0, d1) in enumerate(ops):
        s, e = t[i, :, 0] - t0, t[i, :, 1] - t0
        rows.append((i, mk.OP_NAMES[typ], layer, s.min() / 1e3, s.max() / 1e3, e.max() / 1e3))
    print(f"{'op':>4} {'name':>10} {'layer':>5} {'first_start':>12} {'last_start':>11} "
          f"{'last_end':>9} (us)", file=out)
    for r in rows:
        print(f"{r[0]:>4} {r[1]:>10} {r[2]:>5} {r[3]:>12.1f} {r[4]:>11.1f} {r[5]:>9.1f}", file=out)
    return rows


def measure_multi_step(dec, m, k, v, B, ctx, n_steps, device):
    """n_steps greedy steps in ONE persistent launch (mk_decode_steps), each
    step feeding its argmax to the next on the device; CUDA events around one
    launch after two warm-up launches.  The launch streams n_steps x the
    step's bytes, far more than L2."""
    import torch

    from synthetic import make_tokens

    tok = torch.tensor(make_tokens(m.vocab, B, 77), dtype=torch.int32, device=device)
    pos = torch.tensor(ctx[:B], dtype=torch.int32, device=device)
    out = torch.empty((n_steps, B), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        assert dec.steps(tok, pos, B, n_steps, k, v, None, out) == 0
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    assert dec.steps(tok, pos, B, n_steps, k, v, None, out) == 0
    e1.record(stream)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ms = e0.elapsed_time(e1)
    return {"steps_per_launch": n_steps, "batch": B, "ms_per_step": round(ms / n_steps, 4),
            "tok_s": round(n_steps * B / (ms / 1e3), 1), "launches": 1,
            "path": "mk_decode_steps: one persistent launch, argmax fed back on the device"}


def measure_sampled(dec, m, k, v, B, ctx, device, steps=20, warmup=3, temperature=1.0, top_p=0.9):
    """Sampled decode (mk_decode_step_sample: the step, then temperature / top-p
    sampling of its logits) with each step's token fed to the next on the
    device, and the sampler alone (mk_sample_top_p) on 1, 8 and 64 rows of
    this vocabulary: 50 launches queued behind a device-side sleep, so that the
    events time the device and not the host's launch rate.  CUDA events on the
    launching stream."""
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import make_logits, make_tokens, make_uniforms

    n = warmup + steps
    pos = torch.tensor([[ctx[b] + s for b in range(B)] for s in range(n)], dtype=torch.int32, device=device)
    u = torch.tensor(make_uniforms(n * B, 55), dtype=torch.float64, device=device).view(n, B)
    bufs = [torch.tensor(make_tokens(m.vocab, B, 56), dtype=torch.int32, device=device),
            torch.empty(B, dtype=torch.int32, device=device)]
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for s in range(n):
        if s == warmup:
            torch.cuda.synchronize()
            ev[0].record(stream)
        rc = dec.step_sample(bufs[s % 2], pos[s], B, 1, k, v, None, temperature, top_p, u[s], bufs[(s + 1) % 2])
        assert rc == 0, mk.mk_last_error()
    ev[1].record(stream)
    torch.cuda.synchronize()
    assert dec.status() == 0
    ms = ev[0].elapsed_time(ev[1]) / steps
    alone = {}
    for rows in (1, 8, 64):
        lg = make_logits(rows, m.vocab, 1.0, 57).to(device)
        uu = torch.tensor(make_uniforms(rows, 58), dtype=torch.float64, device=device)
        out = torch.empty(rows, dtype=torch.int32, device=device)
        for _ in range(3):
            assert mk.sample_top_p(lg, temperature, top_p, uu, out) == 0
        torch.cuda.synchronize()
        reps = 50
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(100_000_000)  # the host queues every launch before the device reaches them
        e0.record(stream)
        for _ in range(reps):
            mk.sample_top_p(lg, temperature, top_p, uu, out)
        e1.record(stream)
        torch.cuda.synchronize()
        alone[f"rows{rows}_us"] = round(e0.elapsed_time(e1) / reps * 1e3, 2)
    # where one row's sampler time goes: the device clock at each phase
    # boundary of row 0's first CTA (mk_sample_top_p_phases), median of 21 calls
    lg = make_logits(1, m.vocab, 1.0, 57).to(device)
    uu = torch.tensor(make_uniforms(1, 58), dtype=torch.float64, device=device)
    out = torch.empty(1, dtype=torch.int32, device=device)
    stamps = torch.zeros(mk.MK_SAMPLE_PHASES, dtype=torch.int64, device=device)
    names = ["load slice, largest key", "barrier 1 (share largest key)", "masses, first histogram",
             "radix pass 0", "radix pass 1", "radix pass 2", "radix pass 3", "nucleus, segment totals",
             "barrier 6 (share totals)", "draw", "barrier 7 (exit)"]
    deltas = []
    for _ in range(21):
        assert mk.sample_top_p_phases(lg, temperature, top_p, uu, out, stamps) == 0
        torch.cuda.synchronize()
        t = stamps.cpu().tolist()
        deltas.append([(t[i + 1] - t[i]) / 1e3 for i in range(len(names))])
    med = [sorted(col)[len(col) // 2] for col in zip(*deltas)]
    phases = {nm: round(v, 2) for nm, v in zip(names, med)}
    phases["total (first stamp to last)"] = round(sum(med), 2)
    phases["how"] = ("%globaltimer at each phase boundary of row 0's first CTA, median of 21 calls; the "
                     "device clock advances in steps of a few hundred ns")
    # the same sampled decode, 32 steps as one graph launch (mk_decode_steps_sample)
    nl = 32
    ul = torch.tensor(make_uniforms(nl * B, 59), dtype=torch.float64, device=device).view(nl, B)
    outl = torch.empty((nl, B), dtype=torch.int32, device=device)
    p0 = torch.tensor([ctx[b] for b in range(B)], dtype=torch.int32, device=device)
    for _ in range(2):
        assert dec.steps_sample(bufs[0], p0, B, nl, k, v, None, temperature, top_p, ul, outl) == 0, mk.mk_last_error()
    torch.cuda.synchronize()
    dec.stats(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    assert dec.steps_sample(bufs[0], p0, B, nl, k, v, None, temperature, top_p, ul, outl) == 0
    e1.record(stream)
    torch.cuda.synchronize()
    assert dec.status() == 0
    sts = dec.stats(reset=True)
    lms = e0.elapsed_time(e1) / nl
    loop = {"steps_per_call": nl, "ms_per_step": round(lms, 4), "tok_s": round(B / (lms / 1e3), 1),
            "graph_launches": int(sts.graph_launches), "kernels": int(sts.kernel_launches),
            "path": ("mk_decode_steps_sample: 32 x (megakernel step, sampler) as one CUDA graph launch"
                     if sts.graph_launches == 1 else
                     "mk_decode_steps_sample: 32 x (megakernel step, sampler) enqueued one by one")}
    return {"batch": B, "temperature": temperature, "top_p": top_p, "ms_per_step": round(ms, 4),
            "tok_s": round(B / (ms / 1e3), 1), "launches_per_step": 2,
            "sampler_alone": alone, "sampler_phases_rows1_us": phases, "vocab": m.vocab,
            "path": "mk_decode_step_sample: the megakernel step, then the cluster top-p sampler on its logits",
            "loop": loop}


def measure_dense(device, steps=20, warmup=3):
    """The dense-decoder variant at batch 1 (no router; a 14336-wide SwiGLU FFN
    per layer on the large model's attention): tokens/s and HBM bandwidth."""
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import make_kv_cache, make_weights, workload

    wl = workload("dense", 1)
    m, B, T = wl.model, wl.batch, wl.tokens_per_step
    w = make_weights(m, wl.seed, device)
    ctx = [wl.context] * B
    cap = (wl.context + (steps + warmup + 2) * T + 63) // 64 * 64
    k, v = make_kv_cache(m, B, cap, wl.seed, device)
    dec = mk.Decoder(m, w, max_rows=B * T, max_seqs=B, kv_capacity=cap)
    total, per, st = time_steps(dec, m, k, v, B, T, ctx, steps, warmup, device)
    lens = [c + (warmup + steps // 2) * T + T for c in ctx]
    by = step_bytes(m, B, T, lens, 0)
    ms = total / steps
    dec.close()
    del w, k, v
    torch.cuda.empty_cache()
    return {"workload": f"{wl.name} ({m.name} model: {m.n_layers} layers, d {m.d_model}, FFN {m.shared_ffn}, "
                        f"no router)", "ms_per_step": round(ms, 4), "tok_s": round(B * T / (ms / 1e3), 1),
            "hbm_gbs": round(by / (ms / 1e3) / 1e9, 1), "bytes_per_step": int(by),
            "launches_per_step": st.kernel_launches // steps}


def measure_verify_loop(device, n_steps=16, model=None, weights=None, seed=None, context=None, batch=1):
    """Speculative verify on the device (mk_verify_steps): `batch` sequences,
    blocks of 7 rows (the last accepted token + 6 drafts), n_steps blocks in
    one call, on the small model (default) or on the given model and weights.
    The synthetic drafter proposes the model's own greedy continuation (taken
    from a greedy multi-step launch first) with every 6th draft replaced, so
    that each block accepts 5 drafts plus one token: acceptance length 6 (a
    near tie read differently by the tensor-core path above 8 rows can end a
    block earlier).  Reports accepted tokens per second."""
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import make_kv_cache, make_tokens, make_weights, workload

    wl = workload("verify", 1)
    T, B = wl.tokens_per_step, batch
    if model is None:
        m, seed, p0 = wl.model, wl.seed, wl.context
        w = make_weights(m, seed, device)
    else:
        m, w, p0 = model, weights, context
    acc_len = T - 1
    cap = (p0 + (n_steps + 2) * T + 64 + 63) // 64 * 64
    k, v = make_kv_cache(m, B, cap, seed, device)
    dec = mk.Decoder(m, w, max_rows=B * T, max_seqs=B, kv_capacity=cap)
    firsts = make_tokens(m.vocab, B, 55)
    ng = n_steps * acc_len + T
    greedy = torch.empty((ng, B), dtype=torch.int32, device=device)
    assert dec.steps(torch.tensor(firsts, dtype=torch.int32, device=device),
                     torch.tensor([p0] * B, dtype=torch.int32, device=device), B, ng, k, v, None, greedy) == 0
    drafts = torch.empty((B, n_steps * T + T), dtype=torch.int32, device=device)
    drafts[:, 0] = torch.tensor(firsts, dtype=torch.int32, device=device)
    drafts[:, 1:ng + 1] = greedy.t()
    drafts[:, ng + 1:] = 0
    for s in range(1, n_steps + 2):
        j = s * acc_len
        if j < drafts.shape[1]:
            drafts[:, j] = (drafts[:, j] + 1) % m.vocab
    blk = drafts[:, :T].contiguous().view(-1).clone()
    pos = torch.tensor([p0] * B, dtype=torch.int32, device=device)
    out = torch.empty((n_steps, B * T), dtype=torch.int32, device=device)
    acc = torch.empty((n_steps, B), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        assert dec.verify_steps(blk, pos, B, T, n_steps, drafts, k, v, None, out, acc) == 0
    torch.cuda.synchronize()
    dec.stats(reset=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    assert dec.verify_steps(blk, pos, B, T, n_steps, drafts, k, v, None, out, acc) == 0
    e1.record(stream)
    torch.cuda.synchronize()
    assert dec.status() == 0
    kernels = dec.stats(reset=True).kernel_launches
    ms = e0.elapsed_time(e1)
    accepted = int(acc.sum().item())
    dec.close()
    del k, v
    if model is None:
        del w
    torch.cuda.empty_cache()
    path = ("one persistent megakernel launch" if B * T <= 8 else
            "tensor-core launch sequence with acceptance on the device, one CUDA graph launch")
    return {"workload": f"verify_b{B}_t{T} ({m.name} model, context {p0}), {n_steps} blocks in one call",
            "accepted_tok_s": round(accepted / (ms / 1e3), 1),
            "mean_acceptance": round(accepted / (n_steps * B), 2),
            "ms_per_block": round(ms / n_steps, 4), "launches": 1, "kernels": int(kernels), "path": path,
            "drafter": "the model's greedy continuation with every 6th draft replaced"}


def measure_verify_wide(device, steps=10, warmup=3, batch=8, model=None):
    """A speculative-verify block of 7 rows per sequence on the small model:
    8 sequences (56 rows, the wide-block tensor-core path) or 1 (7 rows, the
    megakernel).  `model` names another synthetic model for the same block
    (e.g. "small_profile", for profiler captures)."""
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import MODELS, make_kv_cache, make_weights, workload

    wl = workload("verify", batch)
    m, B, T = (MODELS[model] if model else wl.model), wl.batch, wl.tokens_per_step
    w = make_weights(m, wl.seed, device)
    ctx = [wl.context] * B
    cap = (wl.context + (steps + warmup + 2) * T + 63) // 64 * 64
    k, v = make_kv_cache(m, B, cap, wl.seed, device)
    dec = mk.Decoder(m, w, max_rows=B * T, max_seqs=B, kv_capacity=cap)
    total, per, st = time_steps(dec, m, k, v, B, T, ctx, steps, warmup, device)
    union = st.expert_union_total / steps / m.n_layers
    lens = [c + (warmup + steps // 2) * T + T for c in ctx]
    by = step_bytes(m, B, T, lens, st.expert_union_total / steps)
    ms = total / steps
    dec.close()
    del w, k, v
    torch.cuda.empty_cache()
    return {"workload": f"{wl.name} ({m.name} model, {B * T} rows per step)", "ms_per_step": round(ms, 4),
            "rows_per_s": round(B * T / (ms / 1e3), 1), "hbm_gbs": round(by / (ms / 1e3) / 1e9, 1),
            "expert_union_per_layer": round(union, 1), "launches_per_step": st.kernel_launches // steps,
            "path": ("tensor-core launch sequence (blocks above 8 rows), replayed as a CUDA graph"
                     if B * T > 8 else "megakernel")}


def measure_read_probe(device, gib=4):
    """The read-only HBM ceiling on this device (mk_hbm_read_probe over a
    buffer far larger than L2): the better of the vector-load and bulk-copy
    forms, 3 calls of 5 timed passes each."""
    import torch

    import decode_megakernel_06_b200 as mk

    buf = torch.empty(gib << 30, dtype=torch.uint8, device=device)
    buf.fill_(1)
    forms = {}
    for form, name in ((0, "vector_loads"), (1, "bulk_copies")):
        forms[name] = round(max(mk.hbm_read_probe(buf, form, 5) for _ in range(3)), 1)
    del buf
    torch.cuda.empty_cache()
    return {"gbs": max(forms.values()), "forms": forms, "bytes": gib << 30,
            "how": "mk_hbm_read_probe: each byte read once per pass, nothing written; best of 3 x 5 passes"}


# The synthetic workloads besides the large model (each also on both
# multi-kernel forms): latency of the tiny model, the small model at batch 1,
# the small model at batches 2/4/8 with per-sequence random contexts, and the
# 7-row speculative-verify block.
CONFIG_LINES = [("tiny_bs1", "tiny", 1), ("small_bs1", "small", 1), ("small_bs2", "small_batch", 2),
                ("small_bs4", "small_batch", 4), ("small_bs8", "small_batch", 8), ("verify_b1_t7", "verify", 1)]


def measure_config_lines(device, peak, probe_gbs, steps=20, warmup=3):
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import make_context_lengths, make_kv_cache, make_weights, workload

    out = {}
    for key, kind, B in CONFIG_LINES:
        wl = workload(kind, B)
        m, T = wl.model, wl.tokens_per_step
        w = make_weights(m, wl.seed, device)
        ctx = make_context_lengths(wl)
        cap = (max(ctx) + (steps + warmup + 2) * T + 63) // 64 * 64
        k, v = make_kv_cache(m, B, cap, wl.seed, device)
        dec = mk.Decoder(m, w, max_rows=B * T, max_seqs=B, kv_capacity=cap)
        row = {"workload": f"{wl.name}: {m.name} model ({m.n_layers} layers, d {m.d_model}, "
                           f"{m.n_experts} experts top-{m.top_k}), B {B}, T {T}, context "
                           + (str(wl.context) if wl.context else f"U{list(wl.context_range)} per sequence")}
        for var in ("megakernel", "multikernel", "multikernel_graph"):
            dec.set_variant(var)
            tot, per, st = time_steps(dec, m, k, v, B, T, ctx, steps, warmup, device)
            ms = tot / steps
            r = {"ms_per_step": round(ms, 4), "ms_per_step_p50": round(statistics.median(per), 4),
                 "tok_s": round(B * T / (ms / 1e3), 1), "launches_per_step": st.kernel_launches // steps}
            if kind != "tiny":  # the tiny model stays in L2: latency only
                lens = [c + (warmup + steps // 2) * T + T for c in ctx]
                by = step_bytes(m, B, T, lens, st.expert_union_total / steps)
                gbs = by / (ms / 1e3) / 1e9
                r.update({"hbm_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                          "frac_of_read_probe": round(gbs / probe_gbs, 4) if probe_gbs else None,
                          "bytes_per_step": int(by)})
            row[var] = r
        mkv = row["megakernel"]["tok_s"]
        row["megakernel_vs_multikernel"] = round(mkv / row["multikernel"]["tok_s"], 3)
        row["megakernel_vs_multikernel_graph"] = round(mkv / row["multikernel_graph"]["tok_s"], 3)
        out[key] = row
        dec.close()
        del w, k, v
        torch.cuda.empty_cache()
    return out


def run_mine(args):
    import torch

    import decode_megakernel_06_b200 as mk
    from synthetic import make_context_lengths, make_kv_cache

    ws, rank, local = dist_env()
    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)
    dist_init(ws, "nccl")
    peaks, peaks_kind = load_peaks()
    B = args.batch
    wl, m, w, gen_s = build_workload(args.workload, B, device)
    T = wl.tokens_per_step
    bmax = max([B] + ([1, 2, 4, 8] if args.sweep else []))
    steps_total = args.warmup + args.steps
    cap_need = max(make_context_lengths(wl)) + (max(steps_total, 30) + 8) * T + 64
    cap = (cap_need + 63) // 64 * 64
    k, v = make_kv_cache(m, bmax, cap, wl.seed, device)
    ctx = make_context_lengths(wl)
    dec = mk.Decoder(m, w, max_rows=bmax * T, max_seqs=bmax, kv_capacity=cap,
                     variant=args.variant)

    if args.trace:
        # warm, then one traced step (not part of the timed region)
        time_steps(dec, m, k, v, B, T, ctx, 1, 3, device)
        trace_step(dec, m, k, v, B, T, ctx, device, save=args.trace_out)

    clocks = ClockSampler(local)
    clocks.start()
    total_ms, per, stats = time_steps(dec, m, k, v, B, T, ctx, args.steps, args.warmup, device)
    clk = clocks.stop()

    union_per_step = stats.expert_union_total / max(1, args.steps)
    lens = [[ctx[b] + (args.warmup + i) * T + T for b in range(B)] for i in range(args.steps)]
    bytes_steps = [step_bytes(m, B, T, L, union_per_step) for L in lens]
    alg_bytes = sum(bytes_steps) / len(bytes_steps)
    ms_per_step = total_ms / args.steps
    max_total = max_over_ranks(total_ms, device)
    tokens_all = sum_over_ranks(args.steps * B * T, device)
    value = tokens_all / (max_total / 1e3)
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    launches = int(stats.kernel_launches)

    # end to end through the host-buffer entry point (fresh positions)
    e2e_steps = max(3, min(args.steps, 20))
    dt, bi, bo = time_e2e(dec, m, k, v, B, T, ctx, e2e_steps, 2)
    e2e = {"value": e2e_steps * B * T / dt, "unit": "tokens/s", "h2d_bytes_per_step": bi,
           "d2h_bytes_per_step": bo, "steps": e2e_steps}

    sweep = None
    if args.sweep and ws == 1:
        sweep = {}
        for bb in (1, 2, 4, 8):
            row = {}
            # MK_TENSORCORE: the tensor-core launch sequence for blocks of 2+ rows
            variants = ("megakernel", "multikernel", "multikernel_graph") + (
                ("tensorcore",) if bb >= 2 and m.n_experts > 0 else ())
            for var in variants:
                dec.set_variant(var)
                n = max(5, min(args.steps, 20))
                ctx_b = make_context_lengths(wl.__class__(wl.name, m, bb, T, wl.context,
                                                          wl.context_range, wl.steps, wl.seed))
                tot, _, st = time_steps(dec, m, k, v, bb, T, ctx_b, n, 3, device)
                u = st.expert_union_total / n
                Ls = [c + 3 * T + n * T // 2 + T for c in ctx_b]
                by = step_bytes(m, bb, T, Ls, u)
                row[var] = {"tok_s": round(n * bb * T / (tot / 1e3), 1),
                            "ms_per_step": round(tot / n, 4),
                            "hbm_gbs": round(by / (tot / n / 1e3) / 1e9, 1),
                            "launches_per_step": st.kernel_launches // n}
            sweep[f"bs{bb}"] = row
        dec.set_variant(args.variant)

    multi = None
    if args.sweep and T == 1:
        multi = measure_multi_step(dec, m, k, v, B, ctx, 32, device)

    sampled = None
    if args.sweep and T == 1:
        sampled = measure_sampled(dec, m, k, v, B, ctx, device)

    probe = measure_read_probe(device) if not args.no_probe else None
    probe_gbs = probe["gbs"] if probe else None

    verify56 = vloop = vloop_large = vloop56 = dense = configs = None
    if args.sweep and ws == 1 and args.workload == "large":
        verify56 = measure_verify_wide(device)
        vloop = measure_verify_loop(device)
        vloop_large = measure_verify_loop(device, model=m, weights=w, seed=wl.seed, context=wl.context)
        vloop56 = measure_verify_loop(device, batch=8)
        dense = measure_dense(device)
        configs = measure_config_lines(device, peak, probe_gbs)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # all host cores (the reported value), then one thread on a shorter sample
        o = oracle_sample(m, w, k, v, B, T, ctx, 1, min_compute_s=10.0)
        o1 = oracle_sample(m, w, k, v, B, T, ctx, 1, threads=1)
        cpu = {"value": round(o["tokens"] / o["compute_s"], 4), "unit": "tokens/s",
               "cores": o["threads"], "kind": "oracle",
               "sample": (f"{o['steps']} consecutive greedy decode steps of the same workload "
                          f"(all layers, from the same cache) on the host "
                          f"(compute {o['compute_s']:.2f} s; weight copy from the device "
                          f"{o['fetch_s']:.2f} s excluded)"),
               "one_thread": {"value": round(o1["tokens"] / o1["compute_s"], 4), "unit": "tokens/s",
                              "cores": 1, "sample": (f"{o1['steps']} decode step(s), compute "
                                                     f"{o1['compute_s']:.2f} s on one thread")}}

    traffic = profile_traffic(f"large_bs{B}_{args.variant}") if args.workload == "large" else None
    if rank == 0:
        line = {
            "metric": "decode tokens/s/GPU at bs 1-8; achieved HBM GB/s vs 8 TB/s peak",
            "value": round(value, 2), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "ms_per_step_p50": round(statistics.median(per), 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 weights / fp32 math", "data": "synthetic (seeded random weights, N(0,1) KV)",
            "config": {"workload": wl.name, "model": m.name, "layers": m.n_layers,
                       "d_model": m.d_model, "experts": f"{m.n_experts} top-{m.top_k}",
                       "global_batch": B * ws, "tokens_per_step": T,
                       "context": wl.context, "variant": args.variant, "parallelism": f"replicas x{ws}",
                       "l2": "inputs larger than L2 (about 7.6 GB streamed per step)"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": f"{peaks_kind} copy bandwidth",
                         "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "traffic": traffic,
                         "traffic_kind": ("ncu dram bytes of the profile model's launch (2 layers, same per-op "
                                          "shapes), scaled to this launch by its algorithmic bytes; null once the "
                                          "kernel source differs from the captured one") if args.workload == "large"
                                         else None,
                         "peak_read_probe": probe_gbs,
                         "frac_of_read_probe": round(achieved / probe_gbs, 4) if probe_gbs else None,
                         "algorithmic_bytes_per_step": int(alg_bytes),
                         "expert_union_per_step": round(union_per_step, 2)},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "weight_gen_s": round(gen_s, 2),
        }
        if sweep is not None:
            line["batch_sweep"] = sweep
        if multi is not None:
            line["multi_step"] = multi
        if sampled is not None:
            line["sampled"] = sampled
        if verify56 is not None:
            line["verify_56"] = verify56
        if probe is not None:
            line["read_probe"] = probe
        if configs is not None:
            line["configs"] = configs
        if vloop is not None:
            line["speculative"] = vloop
        if vloop_large is not None:
            line["speculative_large"] = vloop_large
        if vloop56 is not None:
            line["speculative_56"] = vloop56
        if dense is not None:
            line["dense"] = dense
        print(json.dumps(line), flush=True)
    dec.close()
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()


def run_reference(args):
    """The CPU oracle, as it stands, timed on the host cores (rank 0 only)."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import torch

    from synthetic import make_context_lengths, make_kv_cache

    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)
    B = args.batch
    wl, m, w, gen_s = build_workload(args.workload, B, device)
    T = wl.tokens_per_step
    ctx = make_context_lengths(wl)
    cap = (max(ctx) + (args.warmup + args.steps + 2) * T + 63) // 64 * 64
    k, v = make_kv_cache(m, B, cap, wl.seed, device)
    for _ in range(args.warmup):
        oracle_sample(m, w, k, v, B, T, ctx, 1)
    res = [oracle_sample(m, w, k, v, B, T, ctx, 1) for _ in range(args.steps)]
    comp = sum(r["compute_s"] for r in res)
    value = sum(r["tokens"] for r in res) / comp
    line = {
        "impl": "reference",
        "metric": "decode tokens/s/GPU at bs 1-8; achieved HBM GB/s vs 8 TB/s peak",
        "value": round(value, 4), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(comp / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp32 (bf16 weights)", "data": "synthetic (seeded random weights, N(0,1) KV)",
        "config": {"workload": wl.name, "model": m.name, "global_batch": B, "tokens_per_step": T,
                   "context": wl.context, "variant": "cpu oracle"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": res[0]["threads"],
                         "kind": "oracle",
                         "sample": "one full decode step per timed step; weight copies from the device excluded"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default="large",
                    choices=["large", "small", "tiny", "profile", "dense", "tiny_dense"])
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--variant", default="megakernel",
                    choices=["megakernel", "multikernel", "multikernel_graph", "tensorcore"])
    ap.add_argument("--sweep", action=argparse.BooleanOptionalAction, default=True)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-probe", action="store_true", help="skip the read-only HBM probe")
    ap.add_argument("--trace-out", default=None,
                    help="with --trace: save the raw per-op, per-warp [start, end] stamps (.npy)")
    ap.add_argument("--trace", action="store_true",
                    help="print a per-op timeline of one extra step to stderr")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mine(args)


if __name__ == "__main__":
    main()

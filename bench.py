"""Benchmark of the B200 split-RVQ hot path (Mimi tokenizer bottleneck).

A step is one pass of the whole hot path: the encode of 1 048 576 bf16 frames (bulk
tokenization: projection, semantic VQ, 7-level acoustic RVQ, codes) and the decode of
1 048 576 frames of codes (decode-heavy: gather-sum of the chosen codewords and the
projection back), each on its own seeded model. Other workloads (--workload) are the
240 000-frame fp32 offline batch (encode, then decode of its codes), either 1M-frame half
alone, the streaming step and the Moshi input (delay packing + embedding sum). --n-q uses
only the first n_q codebooks and --variant 1 runs the acoustic RVQ on y - S_s (encode and
decode workloads).

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize(), timed with CUDA events on the stream the kernels run
on; the max over ranks is reported. Inputs are larger than L2 (they are not
re-read from L2 between steps). One JSON line is printed by rank 0. Each call is
timed alone with its own events, so its roofline fraction is taken against the
burst peak (a kernel timed in isolation); the sustained peak applies only to a
region that runs for seconds.

--gpus N runs N replicas (one process per GPU, weak scaling). Under torchrun the
world size must equal N; without torchrun and N > 1 the script launches itself
under torch.distributed.run with N processes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--n-q Q] [--variant V]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

FRAME_HZ = 12.5


def enc_flop(n_q=8):
    """Scores of n_q codebooks plus the 512 -> 256 projection, per frame (8 650 752 at 8)."""
    return n_q * 2 * 2048 * 256 + 2 * 256 * 512


def dec_bytes(n_q=8):
    """n_q int16 codes in, 512 fp32 out, per frame (2 064 at 8)."""
    return n_q * 2 + 512 * 4


METRIC = "RVQ encode/decode frames/s (real-time streams @12.5 Hz) and % of roofline, 1xB200"

WORKLOADS = {
    "encode_decode_1m": "encode of 1048576 bf16 frames [1048576,512] to int16 codes "
                        "[1048576,8] (bulk tokenization) + decode of 1048576 frames of codes "
                        "(semantic uniform, acoustic Zipf(1.1)) to fp32 [1048576,512] "
                        "(decode-heavy); each half on its own seeded model",
    "offline_batch": "64 streams x 3750 frames = 240000 fp32 frames; encode to int16 codes "
                     "[240000,8] then decode to fp32 [240000,512]",
    "bulk_tokenization": "1048576 bf16 frames [1048576,512]; encode only, int16 codes out",
    "decode_heavy": "1048576 frames of codes (semantic uniform, acoustic Zipf(1.1)); decode "
                    "to fp32 [1048576,512]",
    "streaming": "B concurrent streams, one fp32 frame each per call; encode_step",
    "moshi_input": "65536 frames of Moshi + user codes (semantic uniform, acoustic Zipf(1.1)) "
                   "and text tokens (uniform over 32000); delay-pattern packing with tau = 1 "
                   "into 17 streams, then the sum of 17 bf16 embedding tables (text 32001 rows, "
                   "16 x 2049 audio rows, d = 4096) per step, bf16 out [65537,4096]",
}
MOSHI_DELAYS = [0, 1, 1, 1, 1, 1, 1, 1]   # acoustic delay 1 (the final model's)
# DRAM bytes (read + write) per unit from one ncu capture of the current kernel, with the
# summary that records it; the bench scales it by the units of a launch. None: not captured.
NCU_TRAFFIC_PER_UNIT = {
    "k_embed_sum": (48_927, "profiles/k_embed_sum_moshi_input.md"),        # per step
    "k_encode_tc/f32": (2_493, "profiles/k_encode_tc_offline_batch_fp32.md"),  # per fp32 frame
    "k_encode_tc/bf16": (1_159, "profiles/k_encode_tc_bulk_tokenization.md"),  # per bf16 frame
    "k_decode": (1_987, "profiles/k_decode_decode_heavy.md"),              # per frame
}


# Kernel launches of this library per encode call (k_encode_tc, then the float32 re-encode
# of the frames it could not certify) and per decode call (k_decode).
ENCODE_LAUNCHES = 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append(ln)
                self.started.set()

    def __enter__(self):
        import threading
        self.started = threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        self.started.wait(timeout=10)  # sampling is live before the timed region starts
        self.lines.clear()
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            import time as _t
            _t.sleep(0.06)  # one more sample interval covers the end of the region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=10)
        return False

    def summary(self):
        rows = []
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "util": float(parts[4]), "hw": parts[6], "hwt": parts[7],
                             "swt": parts[8], "pcap": parts[9]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        load = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in load:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in load), "reasons": sorted(reasons),
                "samples": len(load)}


# --------------------------------------------------------------------- ranks


def init_dist(world, backend="nccl"):
    """One process per GPU: the process group for world > 1 (None for one rank). A short
    timeout makes ranks that wait on one another end with an error."""
    if world <= 1:
        return None
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x, dist, device):
    """The largest value of x over all ranks (x itself with one rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Units per second of the whole job: every rank processes units_per_rank per step (weak
    scaling) and the step time is the slowest rank's."""
    return units_per_rank * world / (ms_per_step / 1e3)


def pipelined_e2e(torch, device, k, h2d, compute, d2h):
    """k end-to-end steps, each a host-to-device copy of its inputs (h2d(b)), its kernels
    (compute(b, stream)) and a device-to-host copy of its results (d2h(b)), with two sets of
    device buffers (b = step % 2) so that one step's copies overlap its neighbours' kernels on
    separate streams, as a serving pipeline would run. Returns device milliseconds per step,
    from the first copy's start to the last copy's end."""
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_c = torch.cuda.current_stream(device)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_in.wait_stream(s_c)
    start.record(s_in)
    s_c.wait_stream(s_in)
    s_out.wait_stream(s_in)
    for i in range(k):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])   # step i - 2 has finished reading buffer b
            h2d(b)
            in_done[b].record(s_in)
        s_c.wait_event(in_done[b])
        if i >= 2:
            s_c.wait_event(out_done[b])         # step i - 2's results have left buffer b
        compute(b, s_c)
        comp_done[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            d2h(b)
            out_done[b].record(s_out)
    s_out.wait_stream(s_c)
    s_out.wait_stream(s_in)
    stop.record(s_out)
    torch.cuda.synchronize(device)
    return start.elapsed_time(stop) / k


# --------------------------------------------------------------------- workloads


def make_workload(name, rank, frames=None):
    """Host-side inputs for one rank (weak scaling: every rank gets a full workload).

    Returns {"enc": {model, z, dtype} or None, "dec": {model, codes} or None, "frames": n,
    "decode_own_codes": bool}. The offline batch decodes the codes its own encode produced
    (one model); the 1M-frame target pairs the bulk encode and the decode-heavy decode, each
    with its own seeded model. ``frames`` shrinks the workload (profiling captures only; the
    bench line uses the full size)."""
    kw = {"n": frames} if frames else {}
    enc = dec = None
    if name == "offline_batch":
        w = synth.offline_batch(**kw, seed=1 + 100 * rank)
        enc = {"model": w.model, "z": w.z, "dtype": "f32"}
    if name in ("bulk_tokenization", "encode_decode_1m"):
        w = synth.bulk_tokenization(**kw, seed=3 + 100 * rank)
        enc = {"model": w.model, "z": w.z, "dtype": "bf16"}
    if name in ("decode_heavy", "encode_decode_1m"):
        model, codes = synth.decode_heavy(**kw, seed=4 + 100 * rank)
        dec = {"model": model, "codes": codes}
    if enc is None and dec is None:
        raise ValueError(name)
    n = len(enc["z"]) if enc is not None else len(dec["codes"])
    return {"enc": enc, "dec": dec, "frames": n, "decode_own_codes": name == "offline_batch"}


def to_device_latents(torch, z, dtype, device):
    if dtype == "bf16":
        return torch.from_numpy(z.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(z).to(device)


def oracle_step(work, nf, n_q=8, variant=0, nthreads=0):
    """The oracle's pass over the first nf frames of each half of the workload; returns the
    seconds spent on the encode half and on the decode half."""
    import oracle
    t_enc = t_dec = 0.0
    enc, dec = work["enc"], work["dec"]
    codes = None
    if enc is not None:
        m = enc["model"]
        t0 = time.perf_counter()
        codes, _, _ = oracle.encode(enc["z"][:nf], m.W_in, m.C, n_q=n_q, variant=variant,
                                    nthreads=nthreads)
        t_enc = time.perf_counter() - t0
    if work["decode_own_codes"]:
        m = enc["model"]
        t0 = time.perf_counter()
        oracle.decode(codes, m.C, m.W_out, nthreads=nthreads)
        t_dec = time.perf_counter() - t0
    elif dec is not None:
        m = dec["model"]
        t0 = time.perf_counter()
        oracle.decode(np.ascontiguousarray(dec["codes"][:nf, :n_q]), m.C, m.W_out,
                      nthreads=nthreads)
        t_dec = time.perf_counter() - t0
    return t_enc, t_dec


def _halves(work):
    parts = []
    if work["enc"] is not None:
        parts.append("encode")
    if work["decode_own_codes"] or work["dec"] is not None:
        parts.append("decode")
    return "+".join(parts)


def cpu_baseline(work, budget_s=12.0, n_q=8, variant=0):
    """The float64 oracle on this host's cores over a bounded sample of the workload, and the
    same on one thread over a small slice (with the run's n_q and variant). A frame counts
    once it has been through every half of the step, so the rate is 1 / (encode seconds per
    frame + decode seconds per frame)."""
    import oracle
    cores = oracle.threads(0)
    enc_only_cost = work["enc"] is not None
    n = 64 if enc_only_cost else 4096
    te, td = oracle_step(work, n, n_q, variant)
    n = int(max(n, min(work["frames"], n * budget_s / max(te + td, 1e-3))))
    te, td = oracle_step(work, n, n_q, variant)
    n1 = 32 if enc_only_cost else 4096
    te1, td1 = oracle_step(work, n1, n_q, variant, nthreads=1)
    return {"value": n / (te + td), "unit": "frames/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} frames of each half ({_halves(work)}), float64 oracle, "
                      f"{te:.1f} s encode + {td:.1f} s decode",
            "one_thread": {"value": n1 / (te1 + td1), "unit": "frames/s",
                           "sample": f"first {n1} frames"}}


# --------------------------------------------------------------------- our arm


def run_ours(args, rank, world, local_rank):
    import torch
    import split_residual_vector_b200 as pkg

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_dist(world)

    name = args.workload
    work = make_workload(name, rank, args.frames)
    enc, dec = work["enc"], work["dec"]
    n = work["frames"]
    n_q, variant = args.n_q, args.variant
    do_enc = enc is not None
    do_dec = work["decode_own_codes"] or dec is not None

    def handle(m):
        return pkg.Quantizer(torch.from_numpy(m.C).to(device), torch.from_numpy(m.W_in).to(device),
                             torch.from_numpy(m.W_out).to(device))

    q_enc = handle(enc["model"]) if do_enc else None
    q_dec = q_enc if work["decode_own_codes"] else (handle(dec["model"]) if do_dec else None)
    stream = torch.cuda.current_stream(device)
    z = codes = dcodes = x = None
    if do_enc:
        z = to_device_latents(torch, enc["z"], enc["dtype"], device)
        codes = torch.empty((n, n_q), dtype=torch.int16, device=device)
    if do_dec:
        dcodes = (codes if work["decode_own_codes"] else
                  torch.from_numpy(np.ascontiguousarray(dec["codes"][:, :n_q])).to(device))
        x = torch.empty((n, 512), dtype=torch.float32, device=device)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    enc_ms, dec_ms = [], []

    def step(timed):
        if do_enc:
            a, b = ev(), ev()
            a.record(stream)
            q_enc.encode(z, n_q=n_q, variant=variant, out=codes, stream=stream)
            b.record(stream)
            if timed:
                enc_ms.append((a, b))
        if do_dec:
            a, b = ev(), ev()
            a.record(stream)
            q_dec.decode(dcodes, out=x, stream=stream)
            b.record(stream)
            if timed:
                dec_ms.append((a, b))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(device)
    for q in {id(v): v for v in (q_enc, q_dec) if v is not None}.values():
        assert q.get_error(stream) == 0
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    start, stop = ev(), ev()
    with ClockSampler(local_rank) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step(True)
        stop.record(stream)
        torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), dist, device)
    status = 0
    for q in {id(v): v for v in (q_enc, q_dec) if v is not None}.values():
        status = status or q.get_error(stream)
    enc_avg = sum(a.elapsed_time(b) for a, b in enc_ms) / max(len(enc_ms), 1)
    dec_avg = sum(a.elapsed_time(b) for a, b in dec_ms) / max(len(dec_ms), 1)
    ms_per_step = elapsed_ms / args.steps
    value = whole_job_rate(n, world, ms_per_step)

    # ---- end to end through the public API, host buffers (pinned), copies inside
    e2e = None
    if not args.no_e2e:
        k = max(4, min(args.steps, 10))
        # two sets of device buffers; the host side holds one input set and two result sets
        h_z = None
        if do_enc:
            h_z = torch.empty(z.shape, dtype=z.dtype, pin_memory=True)
            h_z.copy_(z)
        h_dc = None
        if do_dec and not work["decode_own_codes"]:
            h_dc = torch.empty(dcodes.shape, dtype=dcodes.dtype, pin_memory=True)
            h_dc.copy_(dcodes)
        h_codes = ([torch.empty((n, n_q), dtype=torch.int16, pin_memory=True) for _ in range(2)]
                   if do_enc else None)
        h_x = ([torch.empty((n, 512), dtype=torch.float32, pin_memory=True) for _ in range(2)]
               if do_dec else None)
        z2 = [z, torch.empty_like(z)] if do_enc else None
        codes2 = [codes, torch.empty_like(codes)] if do_enc else None
        if do_dec:
            dcodes2 = codes2 if work["decode_own_codes"] else [dcodes, torch.empty_like(dcodes)]
            x2 = [x, torch.empty_like(x)]
        bi = ((h_z.numel() * h_z.element_size() if h_z is not None else 0)
              + (h_dc.numel() * 2 if h_dc is not None else 0))
        bo = (codes.numel() * 2 if do_enc else 0) + (x.numel() * 4 if do_dec else 0)

        def h2d(b):
            if h_z is not None:
                z2[b].copy_(h_z, non_blocking=True)
            if h_dc is not None:
                dcodes2[b].copy_(h_dc, non_blocking=True)

        def compute(b, s):
            if do_enc:
                q_enc.encode(z2[b], n_q=n_q, variant=variant, out=codes2[b], stream=s)
            if do_dec:
                q_dec.decode(dcodes2[b], out=x2[b], stream=s)

        def d2h(b):
            if do_enc:
                h_codes[b].copy_(codes2[b], non_blocking=True)
            if do_dec:
                h_x[b].copy_(x2[b], non_blocking=True)

        pipelined_e2e(torch, device, 2, h2d, compute, d2h)  # warm-up
        if dist:
            dist.barrier()
        e_ms = max_over_ranks(pipelined_e2e(torch, device, k, h2d, compute, d2h), dist, device)
        e2e = {"value": whole_job_rate(n, world, e_ms), "unit": "frames/s", "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": e_ms, "steps": k,
               "pipeline": "two buffer sets; each step's copies overlap its neighbours' kernels"}

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return None

    peaks = load_peaks()
    kernels = []
    lat_dtype = enc["dtype"] if do_enc else None
    lat_bytes = 2048 if lat_dtype == "f32" else 1024
    if do_enc:
        tf = enc_flop(n_q) * n / (enc_avg / 1e3) / 1e12
        f_enc, f_re = q_enc.stats()    # since create: warm-up, timed and e2e calls
        # the captured DRAM traffic is for the full 8-codebook, variant-0 encode
        tr = (NCU_TRAFFIC_PER_UNIT.get("k_encode_tc/" + lat_dtype)
              if (n_q, variant) == (8, 0) else None)
        kernels.append({
            "kernel": "encode call (k_encode_tc + float32 re-encode)", "bound": "tensor",
            "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tf / peaks["bf16_tflops"],
            "peak_source": f"{peaks['source']} bf16_tflops (burst: the call is timed alone)",
            "traffic": tr[0] * n if tr and tr[0] else None,
            "traffic_source": tr[1] if tr and tr[0] else None,
            "ms": enc_avg, "frames": n, "latent_dtype": lat_dtype,
            "reencoded_frames_per_call": f_re / f_enc * n if f_enc else None,
            "algorithmic": (f"{enc_flop(n_q)} FLOP/frame x {n} frames; "
                            f"HBM {lat_bytes + 2 * n_q} B/frame"),
            "hbm_gbs": (lat_bytes + 2 * n_q) * n / (enc_avg / 1e3) / 1e9})
    if do_dec:
        gbs = dec_bytes(n_q) * n / (dec_avg / 1e3) / 1e9
        tr = NCU_TRAFFIC_PER_UNIT["k_decode"] if n_q == 8 else None
        kernels.append({
            "kernel": "k_decode", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
            "peak_source": f"{peaks['source']} hbm_gbs",
            "traffic": tr[0] * n if tr and tr[0] else None,
            "traffic_source": tr[1] if tr and tr[0] else None, "ms": dec_avg, "frames": n,
            "codes": "from the encode" if work["decode_own_codes"] else
                     "semantic uniform, acoustic Zipf(1.1)",
            "algorithmic": f"{dec_bytes(n_q)} B/frame x {n} frames (codes in, fp32 latents out)"})
    dominant = max(kernels, key=lambda kk: kk["ms"])
    roofline = {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = dominant["kernel"]
    roofline["traffic_source"] = dominant.get("traffic_source")
    roofline["peak_source"] = dominant["peak_source"]
    if args.self_profile and do_enc and (n_q, variant) == (8, 0):
        _, cyc = q_enc.encode_profile(z, out=codes, stream=stream)
        total = max(cyc["cta_total"], 1)
        counts = set(q_enc.PROFILE_COUNTS)
        kernels[0]["self_profile_share"] = {k: round(v / total, 4) for k, v in cyc.items()
                                            if k not in counts}
        kernels[0]["self_profile_counts"] = {k: cyc[k] for k in q_enc.PROFILE_COUNTS}
    launches_per_step = (ENCODE_LAUNCHES if do_enc else 0) + (1 if do_dec else 0)
    line = {
        "metric": METRIC, "value": value, "unit": "frames/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 products, f32 accumulate/re-score", "data": "synthetic",
        "config": {"workload": f"{name}: {WORKLOADS[name]}" + (
                       f" (reduced to {n} frames)" if args.frames else ""), "frames_per_gpu": n,
                   "halves": _halves(work), "latent_dtype": lat_dtype, "n_q": n_q,
                   "variant": variant, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (not re-read from L2 between steps)"},
        "realtime_streams": value / FRAME_HZ,
        "roofline": roofline, "kernels": kernels,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(), "status": status, "e2e": e2e,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(work, n_q=n_q, variant=variant)
    if dist:
        dist.destroy_process_group()
    return line


def run_streaming(args):
    """Per-call device latency of encode_step for B in {1, 16, 128, 1024}, 1000 calls each.
    The calls cycle through a pool of distinct input batches larger than L2 (at least
    256 MiB), so every call reads its frames from HBM; the codebook tables, which every call
    reads, stay in L2 as they would in a streaming service."""
    import torch
    import split_residual_vector_b200 as pkg
    device = torch.device("cuda", 0)
    out = {}
    for B in args.batches:
        model, frames = synth.streaming_step(B, calls=args.calls)
        q = pkg.Quantizer(torch.from_numpy(model.C).to(device),
                          torch.from_numpy(model.W_in).to(device),
                          torch.from_numpy(model.W_out).to(device))
        pool_calls = max(args.calls, (256 << 20) // (B * 512 * 4))
        f = torch.from_numpy(frames).to(device)
        if pool_calls > args.calls:
            reps = (pool_calls + args.calls - 1) // args.calls
            f = f.repeat(reps, 1, 1)[:pool_calls].contiguous()
        stride = 7919  # a prime step through the pool: consecutive calls touch distant batches
        codes = torch.empty((B, 8), dtype=torch.int16, device=device)
        stream = torch.cuda.current_stream(device)
        for i in range(5):
            q.encode_step(f[i], out=codes, stream=stream)
        times = []
        for i in range(args.calls):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            q.encode_step(f[(i * stride) % f.shape[0]], out=codes, stream=stream)
            b.record(stream)
            times.append((a, b))
        torch.cuda.synchronize(device)
        ms = sorted(a.elapsed_time(b) for a, b in times)
        out[B] = {"median_us": 1e3 * ms[len(ms) // 2], "p99_us": 1e3 * ms[int(0.99 * len(ms))],
                  "frames_per_s": B / (ms[len(ms) // 2] / 1e3),
                  "input_pool_mib": f.numel() * 4 / 2**20}
        q.close()
    return {"metric": METRIC, "workload": f"streaming: {WORKLOADS['streaming']}",
            "calls": args.calls, "per_batch": out}


def run_moshi_input(args, rank, world, local_rank):
    """The language model's side of the codec: pack + embedding sum (one step = both calls
    over the whole workload)."""
    import torch
    import split_residual_vector_b200 as pkg

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_dist(world)
    T = args.frames or (1 << 16)
    text_h, audio_h = synth.moshi_streams(T, seed=5 + 100 * rank)
    rows = synth.moshi_rows()
    tables_h = synth.moshi_tables(seed=6 + 100 * rank)
    d = tables_h.shape[1]
    K = len(rows)
    S = T + max(MOSHI_DELAYS)
    text = torch.from_numpy(text_h).to(device)
    audio = torch.from_numpy(audio_h).to(device)
    tables = torch.from_numpy(tables_h.view(np.int16)).to(device).view(torch.bfloat16)
    packed = torch.empty((S, K), dtype=torch.int32, device=device)
    out = torch.empty((S, d), dtype=torch.bfloat16, device=device)
    n_bad = torch.zeros(1, dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    pack_ms, emb_ms = [], []

    def step(timed):
        a, b, c = ev(), ev(), ev()
        a.record(stream)
        pkg.delay_pack(text, audio, MOSHI_DELAYS, out=packed, stream=stream)
        b.record(stream)
        pkg.embed_sum(tables, rows, packed, out=out, n_bad=n_bad, stream=stream)
        c.record(stream)
        if timed:
            pack_ms.append((a, b))
            emb_ms.append((b, c))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    start, stop = ev(), ev()
    with ClockSampler(local_rank) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step(True)
        stop.record(stream)
        torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), dist, device)
    ms_per_step = elapsed_ms / args.steps
    value = whole_job_rate(T, world, ms_per_step)
    pack_avg = sum(a.elapsed_time(b) for a, b in pack_ms) / len(pack_ms)
    emb_avg = sum(a.elapsed_time(b) for a, b in emb_ms) / len(emb_ms)
    bad = int(n_bad.item())

    e2e = None
    if not args.no_e2e:
        k = max(4, min(args.steps, 8))
        h_text = torch.empty_like(text, device="cpu").pin_memory()
        h_audio = torch.empty_like(audio, device="cpu").pin_memory()
        h_text.copy_(text)
        h_audio.copy_(audio)
        h_out = [torch.empty((S, d), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        text2, audio2 = [text, torch.empty_like(text)], [audio, torch.empty_like(audio)]
        packed2, out2 = [packed, torch.empty_like(packed)], [out, torch.empty_like(out)]

        def h2d(b):
            text2[b].copy_(h_text, non_blocking=True)
            audio2[b].copy_(h_audio, non_blocking=True)

        def compute(b, st):
            pkg.delay_pack(text2[b], audio2[b], MOSHI_DELAYS, out=packed2[b], stream=st)
            pkg.embed_sum(tables, rows, packed2[b], out=out2[b], stream=st)

        def d2h(b):
            h_out[b].copy_(out2[b], non_blocking=True)

        pipelined_e2e(torch, device, 2, h2d, compute, d2h)  # warm-up
        if dist:
            dist.barrier()
        e_ms = max_over_ranks(pipelined_e2e(torch, device, k, h2d, compute, d2h), dist, device)
        e2e = {"value": whole_job_rate(T, world, e_ms), "unit": "frames/s",
               "h2d_bytes_per_step": text.numel() * 4 + audio.numel() * 2,
               "d2h_bytes_per_step": out.numel() * 2, "ms_per_step": e_ms, "steps": k,
               "pipeline": "two buffer sets; each step's copies overlap its neighbours' kernels"}
    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return None
    peaks = load_peaks()
    row_bytes = d * 2
    emb_bytes = K * row_bytes + K * 4 + row_bytes   # gathered rows + tokens + bf16 out, per step
    pack_bytes = 4 + 2 * 8 * 2 + K * 4              # text + codes in, packed row out, per step
    emb_gbs = emb_bytes * S / (emb_avg / 1e3) / 1e9
    pack_gbs = pack_bytes * S / (pack_avg / 1e3) / 1e9
    kernels = [
        {"kernel": "k_embed_sum", "bound": "hbm", "achieved": emb_gbs, "peak": peaks["hbm_gbs"],
         "unit": "GB/s", "frac": emb_gbs / peaks["hbm_gbs"],
         "traffic": NCU_TRAFFIC_PER_UNIT["k_embed_sum"][0] * S,
         "traffic_source": NCU_TRAFFIC_PER_UNIT["k_embed_sum"][1],
         "dram_gbs_from_traffic": NCU_TRAFFIC_PER_UNIT["k_embed_sum"][0] * S / (emb_avg / 1e3) / 1e9,
         "ms": emb_avg,
         "algorithmic": f"{emb_bytes} B/step ({K} gathered bf16 rows of {d}, tokens, bf16 out) "
                        f"x {S} steps; hot rows may come from L2"},
        {"kernel": "k_delay_pack", "bound": "hbm", "achieved": pack_gbs, "peak": peaks["hbm_gbs"],
         "unit": "GB/s", "frac": pack_gbs / peaks["hbm_gbs"], "traffic": None, "ms": pack_avg,
         "algorithmic": f"{pack_bytes} B/step x {S} steps"}]
    roofline = {k: kernels[0][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = "k_embed_sum"
    roofline["peak_source"] = f"{peaks['source']} hbm_gbs"
    line = {
        "metric": METRIC, "value": value, "unit": "frames/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 tables, f32 accumulate, bf16 out; int32 tokens", "data": "synthetic",
        "config": {"workload": f"moshi_input: {WORKLOADS['moshi_input']}"
                               + (f" (reduced to {T} frames)" if args.frames else ""),
                   "frames_per_gpu": T, "steps_per_frame_stream": S, "delays": MOSHI_DELAYS,
                   "parallelism": f"replicas x{world}",
                   "l2": "output (537 MB) larger than L2; tables 531 MB, hot rows stay in L2"},
        "realtime_streams": value / FRAME_HZ, "roofline": roofline, "kernels": kernels,
        "gpu_launches": 2 * args.steps, "clocks": clocks.summary(), "status": 0 if bad == 0 else -4,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline:
        import oracle
        cores = oracle.threads(0)
        n = 256
        for _ in range(2):
            t0 = time.perf_counter()
            V = oracle.delay_pack(text_h[:n], audio_h[:, :n], MOSHI_DELAYS)
            oracle.embed_sum(tables_h, rows, V)
            dt = time.perf_counter() - t0
            if dt > 3.0:
                break
            n = int(min(T, n * 12.0 / max(dt, 1e-3)))
        line["cpu_baseline"] = {"value": n / dt, "unit": "frames/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"first {n} frames: pack + embedding sum, float64 "
                                          f"oracle, {dt:.1f} s"}
    if dist:
        dist.destroy_process_group()
    return line


# --------------------------------------------------------------------- reference arm


def run_reference(args):
    """The float64 oracle on the host cores, each step a bounded sample of the workload."""
    import oracle
    name = args.workload
    if name == "moshi_input":
        text_h, audio_h = synth.moshi_streams(args.frames or (1 << 16), seed=5)
        tables_h, rows = synth.moshi_tables(seed=6), synth.moshi_rows()
        work = {"frames": len(text_h)}
    elif name == "streaming":
        model, frames = synth.streaming_step(1024, calls=1)
        work = {"enc": {"model": model, "z": frames[0], "dtype": "f32"}, "dec": None,
                "frames": frames.shape[1], "decode_own_codes": False}
    else:
        work = make_workload(name, 0)

    def one(nf):
        if name == "moshi_input":
            oracle.embed_sum(tables_h, rows,
                             oracle.delay_pack(text_h[:nf], audio_h[:, :nf], MOSHI_DELAYS))
            return
        oracle_step(work, nf, args.n_q, args.variant)

    t0 = time.perf_counter()
    one(32)
    per_frame = (time.perf_counter() - t0) / 32
    budget = 120.0 / (args.steps + args.warmup)  # whole run within ~2 minutes
    nf = int(max(8, min(work["frames"], budget / max(per_frame, 1e-9))))
    for _ in range(args.warmup):
        one(nf)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(nf)
    dt = (time.perf_counter() - t0) / args.steps
    value = nf / dt
    cores = oracle.threads(0)
    what = "pack + embedding sum" if name == "moshi_input" else _halves(work)
    sample = f"first {nf} frames of {name} per step ({what}), float64 oracle"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "frames/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{name}: {WORKLOADS[name]}", "sample_frames": nf,
                       **({"n_q": args.n_q, "variant": args.variant}
                          if name not in ("moshi_input", "streaming") else {})},
            "cpu_baseline": {"value": value, "unit": "frames/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------- launch


def check_world(gpus, env):
    """How this process runs --gpus N: "run" when it is one rank of a world of N processes
    (torchrun sets WORLD_SIZE) or N = 1 without torchrun; "launch" when N > 1 and no torchrun
    environment is present, so the script must start the N ranks itself. A world size that
    differs from N is an error (SystemExit), never a silent single replica."""
    if gpus < 1:
        raise SystemExit(f"bench.py: --gpus must be >= 1 (got {gpus})")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise SystemExit(f"bench.py: --gpus {gpus} but this world has WORLD_SIZE={world} "
                             f"processes; launch N processes for --gpus N")
        return "run"
    return "launch" if gpus > 1 else "run"


def torchrun_command(argv, gpus, port):
    """The command that runs this script as `gpus` ranks on one node (127.0.0.1 rendezvous)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__), *argv]


def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="encode_decode_1m", choices=list(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--calls", type=int, default=1000, help="streaming workload: calls per B")
    ap.add_argument("--batches", type=lambda v: [int(x) for x in v.split(",")],
                    default=[1, 16, 128, 1024], help="streaming workload: the B values")
    ap.add_argument("--frames", type=int, default=None,
                    help="shrink the workload (for profiler captures); default: full size")
    ap.add_argument("--self-profile", action="store_true",
                    help="add the encode kernel's per-role cycle shares (one extra untimed call)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--n-q", type=int, default=8, choices=range(1, 9),
                    help="codebooks used (encode/decode workloads): the semantic one and "
                         "n_q - 1 acoustic levels")
    ap.add_argument("--variant", type=int, default=0, choices=(0, 1),
                    help="encode workloads: 1 runs the acoustic RVQ on y - S_s")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if check_world(args.gpus, os.environ) == "launch":
        sys.exit(subprocess.call(torchrun_command(sys.argv[1:], args.gpus, free_port())))

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.workload == "streaming":
        if rank == 0:
            print(json.dumps(run_streaming(args)), flush=True)
        return
    if args.workload == "moshi_input":
        line = run_moshi_input(args, rank, world, local_rank)
    else:
        line = run_ours(args, rank, world, local_rank)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

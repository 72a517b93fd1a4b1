#!/usr/bin/env python
"""KDA benchmark: prefill Mtokens/s (H=64, d=128) and decode-step HBM GB/s on B200.

One step = one pass of the whole hot path:
  * kda_forward on the prefill workload  B=2, H=64, T=8192, d_k=d_v=128
    (bf16 q/k/v/alpha/beta, fp32 o and final state, zero initial state), and
  * kda_decode_step on the decode workload  256 sequences x 64 heads, d=128
    (bf16 inputs, fp32 128x128 state per head updated in place).
Each launch is bracketed by CUDA events on the launching stream.  ``value`` is
the prefill throughput in Mtokens/s (a token = one (sequence, position) across
all 64 heads) summed over ranks; the decode step is reported beside it in GB/s
of algorithmic HBM traffic.  Inputs (1.07 GB prefill, 2.2 GB decode state) are
far larger than the 126 MB L2, so no flush is needed between steps.

After the timed steps, a single-GPU run also times each further entry point once
on a workload of the same scale (``next_rows`` in the JSON line): the scalar-gate,
raw-input, packed-sequence and GDN-2 prefills, the multi-token decode with
per-token states, and the state copy, each with its algorithmic bytes and the
fraction of the measured copy bandwidth they reach.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run; every rank runs the same workload
on its own GPU (independent (sequence, head) shards, no collective on the data
path) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import itertools
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill Mtokens/s (H=64,d=128); decode-step HBM GB/s vs ~8 TB/s peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the prefill
# kernel on the prefill workload (1.0760 GB read + 0.5094 GB written) and on the long
# workload (4.3134 GB + 2.1216 GB), from the captures summarised under profiles/, with
# the hash of the kernel sources they were taken for: once the sources change, the
# line reports traffic as null until it is captured again.  (The long workload's kernel,
# the early-R form, was last changed before its capture; the prefill workload's was
# captured on these sources.)
PREFILL_TRAFFIC_BYTES = 1_076_045_824 + 509_351_936
LONG_TRAFFIC_BYTES = 4_313_396_736 + 2_121_649_920
PREFILL_TRAFFIC_SOURCES = "9afd6510a83d95c2"


def kernel_sources_hash() -> str:
    import hashlib
    csrc = os.path.join(ROOT, "gated_delta_rule_122_b200", "csrc")
    h = hashlib.sha256()
    for name in ("chunk_tc.cu", "tc_ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-entry-point measurements")
    ap.add_argument("--no-long", action="store_true", help="skip the long-prefill measurement")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run one kernel per step (for profiling); the JSON line is then partial")
    ap.add_argument("--prefill-workload", choices=["prefill", "long", "small"], default="prefill",
                    help="the prefill workload of each step (profiling the long or the small workload; the "
                         "JSON line then describes that workload)")
    ap.add_argument("--prefill-seqs", type=int, default=None,
                    help="sequences per rank of the prefill workload (profiling a smaller case; "
                         "the JSON line then describes that case, not the headline workload)")
    ap.add_argument("--prefill-len", type=int, default=None,
                    help="tokens per sequence of the prefill workload (profiling a smaller case)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_bytes(w, with_s0: bool) -> int:
    """Algorithmic bytes of one prefill launch: inputs read once, o and final state written once."""
    import torch
    qsz = torch.tensor([], dtype=w.qkv_dtype).element_size()
    gsz = torch.tensor([], dtype=w.gate_dtype).element_size()
    tokens = w.B * w.T * w.H
    per_token = 2 * w.dk * qsz + w.dv * qsz + w.dk * gsz + gsz + w.dv * 4
    state = w.B * w.H * w.dk * w.dv * 4
    return tokens * per_token + state * (2 if with_s0 else 1)


def decode_bytes(w) -> int:
    """Algorithmic bytes of one decode step: each state read once and written once, token vectors, o."""
    import torch
    qsz = torch.tensor([], dtype=w.qkv_dtype).element_size()
    gsz = torch.tensor([], dtype=w.gate_dtype).element_size()
    heads = w.B * w.H
    return heads * (2 * w.dk * w.dv * 4 + 2 * w.dk * qsz + w.dv * qsz + w.dk * gsz + gsz + w.dv * 4)


def time_call(torch, fn, reps=5, warmup=2):
    """Mean CUDA-event time of fn() in ms on the current stream, after warm-up calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_long(torch, kda, device, hbm):
    """The long prefill workload (B=1 H=64 T=65536 d=128, bf16 inputs, random initial
    state, 30% strong-forget channels), device-timed with CUDA events on its own, with its
    roofline against its algorithmic bytes (inputs, initial and final state, o)."""
    from gated_delta_rule_122_b200.inputs import make_inputs, workload
    w = workload("long")
    xl = make_inputs(w, device=device)
    ol = torch.empty((w.B, w.T, w.H, w.dv), device=device)
    Sl = torch.empty((w.B, w.H, w.dk, w.dv), device=device)
    fn = lambda: kda.forward(xl["q"], xl["k"], xl["v"], xl["alpha"], xl["beta"], initial_state=xl["s0"],
                             scale=xl["scale"], out=ol, final_state=Sl)
    ms = time_call(torch, fn, reps=5, warmup=2)
    nbytes = prefill_bytes(w, True)
    gbs = nbytes / (ms * 1e-3) / 1e9
    del xl, ol, Sl
    return {"workload": f"long prefill B={w.B} H={w.H} T={w.T} d_k=d_v={w.dk} bf16 q/k/v/alpha/beta, random "
                        "initial state, 30% strong-forget channels", "ms": ms,
            "mtokens_s": w.B * w.T / (ms * 1e-3) / 1e6,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": LONG_TRAFFIC_BYTES if kernel_sources_hash() == PREFILL_TRAFFIC_SOURCES else None,
                         "algorithmic_bytes": nbytes}}


def measure_rows(torch, kda, x, y, wp, hbm):
    """Each further entry point once, at the scale of the prefill and decode workloads.
    Returns {row: {workload, ms, throughput, algorithmic bytes, fraction of hbm}}."""
    dev = x["q"].device
    B, T, H, dk, dv = wp.B, wp.T, wp.H, wp.dk, wp.dv
    tok_heads = B * T * H
    state = B * H * dk * dv * 4
    rows = {}

    def row(name, workload, ms, nbytes, tokens=None):
        r = {"workload": workload, "ms": ms, "algorithmic_bytes": nbytes,
             "gbs": nbytes / (ms * 1e-3) / 1e9}
        r["frac_of_measured_hbm"] = r["gbs"] / hbm
        if tokens is not None:
            r["mtokens_s"] = tokens / (ms * 1e-3) / 1e6
        rows[name] = r

    # the small workload (B=1 H=4 T=2048 d=64, bf16 q/k/v, fp32 alpha/beta, random initial state)
    from gated_delta_rule_122_b200.inputs import make_inputs, workload
    ws_ = workload("small")
    xs = make_inputs(ws_, device=dev)
    small = f"B={ws_.B} T={ws_.T} H={ws_.H} d={ws_.dk}, bf16 q/k/v, fp32 alpha/beta, initial state"
    run_small = lambda: kda.forward(xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"],
                                    initial_state=xs["s0"], scale=xs["scale"])
    # the library's own choice for 4 (sequence, head) pairs: the column scan
    ms = time_call(torch, run_small)
    row("small_prefill", small + f", schedule {kda.get_schedule()} (column scan)", ms,
        prefill_bytes(ws_, True), ws_.B * ws_.T)
    with kda.schedule("chunked"):   # the CUDA-core chunk kernel on the same input
        ms = time_call(torch, run_small)
    row("small_prefill_chunked", small + ", chunkwise schedule (CUDA-core chunk kernel)", ms,
        prefill_bytes(ws_, True), ws_.B * ws_.T)
    del xs
    o = torch.empty((B, T, H, dv), device=dev)
    S = torch.empty((B, H, dk, dv), device=dev)
    # scalar gate: one retention factor per (token, head)
    ah = x["alpha"][..., 0].contiguous()
    ms = time_call(torch, lambda: kda.forward_scalar_gate(x["q"], x["k"], x["v"], ah, x["beta"], scale=x["scale"],
                                                          out=o, final_state=S))
    row("scalar_gate_prefill", f"B={B} T={T} H={H} d={dk} bf16, alpha [B,T,H]", ms,
        tok_heads * (3 * 256 + 2 + 2 + 512) + state, B * T)
    # raw inputs: the logits whose maps give the workload's alpha and beta (same bytes as the
    # plain prefill and the same recurrence; q and k go through the norm pass as they are)
    a = x["alpha"].float().clamp(1e-30, 1 - 1e-7)
    gl = torch.log((1 - a) / a).to(x["alpha"].dtype)
    del a
    bt = x["beta"].float().clamp(1e-7, 1 - 1e-7)
    bl = torch.log(bt / (1 - bt)).to(x["beta"].dtype)
    ms = time_call(torch, lambda: kda.forward_raw(x["q"], x["k"], x["v"], gl, bl, scale=x["scale"],
                                                  out=o, final_state=S))
    del gl, bl
    row("raw_inputs_prefill", f"B={B} T={T} H={H} d={dk} bf16 raw q/k, gate and beta logits", ms,
        tok_heads * 1538 + state, B * T)
    # packed sequences: the same tokens as 8 sequences of mixed lengths
    lengths = [4096, 1000, 3000, 200, 5000, 1084, 1500, 504]
    assert sum(lengths) == B * T
    cu = torch.tensor([0] + list(itertools.accumulate(lengths)), dtype=torch.int32, device=dev)
    flat = {n: x[n].reshape(B * T, *x[n].shape[2:]) for n in ("q", "k", "v", "alpha", "beta")}
    ov = o.view(B * T, H, dv)
    Sv = torch.empty((len(lengths), H, dk, dv), device=dev)
    ms = time_call(torch, lambda: kda.forward_varlen(flat["q"], flat["k"], flat["v"], flat["alpha"], flat["beta"], cu,
                                                     scale=x["scale"], out=ov, final_state=Sv))
    row("varlen_prefill", f"{B * T} tokens as sequences {lengths}, H={H} d={dk} bf16", ms,
        tok_heads * 1538 + len(lengths) * H * dk * dv * 4, B * T)
    # GDN-2 (tensor-core chunk kernel): erase [.., d_k] and write [.., d_v] gates in place of beta
    g = torch.Generator(device=dev).manual_seed(7)
    er = torch.sigmoid(torch.randn(x["k"].shape, generator=g, device=dev)).to(torch.bfloat16)
    wr = torch.sigmoid(torch.randn(x["v"].shape, generator=g, device=dev)).to(torch.bfloat16)
    ms = time_call(torch, lambda: kda.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], er, wr, scale=x["scale"],
                                                   out=o, final_state=S))
    row("gdn2_prefill", f"B={B} T={T} H={H} d={dk} bf16, erase/write gates (tensor-core kernel)", ms,
        tok_heads * (6 * 256 + 512) + state, B * T)
    del er, wr
    if y is not None:
        N, Hd, d = y["state"].shape[0], y["state"].shape[1], y["state"].shape[2]
        Td = 4
        gd = torch.Generator(device=dev).manual_seed(8)
        draft = {n: torch.cat([y[n].unsqueeze(1)] * Td, 1).contiguous() for n in ("q", "k", "v", "alpha", "beta")}
        ts = torch.empty((N, Td, Hd, d, d), device=dev)
        od = torch.empty((N, Td, Hd, d), device=dev)
        ms = time_call(torch, lambda: kda.decode_tokens(draft["q"], draft["k"], draft["v"], draft["alpha"],
                                                        draft["beta"], y["state"], commit=False, token_states=ts,
                                                        scale=y["scale"], out=od))
        heads = N * Hd
        row("decode_tokens_verify", f"N={N} H={Hd} d={d}, {Td} draft tokens, per-token states, no commit", ms,
            heads * (d * d * 4 * (1 + Td) + Td * (3 * 256 + 256 + 2 + 512)))
        del ts, od, draft
        pool = torch.empty_like(y["state"])
        perm = torch.randperm(N, generator=gd, device=dev).to(torch.int32)
        ms = time_call(torch, lambda: kda.state_copy(y["state"], pool, src_index=perm,
                                                     dst_index=torch.arange(N, dtype=torch.int32, device=dev)))
        row("state_copy", f"{N} states of H={Hd} d={d} gathered by a permutation", ms, 2 * N * Hd * d * d * 4)
        del pool
    return rows


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        super().__init__(daemon=True)
        self.samples = []
        self.period = period_s
        self.err = None
        self._halt = threading.Event()
        self.window = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            import torch
            handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # NVML missing: report it rather than guess
            self.err = repr(e)

    def run(self):
        if self.err:
            return
        while not self._halt.is_set():
            try:
                sm = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self._reasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception as e:
                self.err = repr(e)
                return
            time.sleep(self.period)

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)

    def summary(self):
        if self.err and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "error": self.err}
        sel = self.samples
        if self.window:
            inside = [s for s in self.samples if self.window[0] <= s[0] <= self.window[1]]
            if inside:
                sel = inside
        mhz = [s[1] for s in sel]
        mask = 0
        for s in sel:
            mask |= int(s[2])
        reasons = [name for bit, name in self.REASONS.items() if mask & bit]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel)}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        if world == 1 and n_gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return world, rank, local, pg


def reduce_max(pg, values, device):
    from gated_delta_rule_122_b200.shard import max_over_ranks
    return max_over_ranks(values, device=device)


def barrier(pg):
    if pg is not None:
        pg.barrier()


def cpu_baseline_prefill(x, w, max_heads=None):
    """Time the fp64 oracle on a bounded sample of the prefill workload (host cores)."""
    import oracle
    n_threads = oracle.threads_for(10 ** 6)
    n_heads = min(w.B * w.H, max(2 * n_threads, 4)) if max_heads is None else max_heads
    pairs = [(i // w.H, i % w.H) for i in range(n_heads)]
    sel = lambda t: t[[b for b, _ in pairs], :, [h for _, h in pairs]]   # [n, T, ...]
    q, k, v, a = (sel(x[n]).unsqueeze(0).transpose(1, 2).contiguous().cpu()
                  for n in ("q", "k", "v", "alpha"))                    # [1, T, n, d]
    beta = x["beta"][[b for b, _ in pairs], :, [h for _, h in pairs]].unsqueeze(0).transpose(1, 2).contiguous().cpu()
    q, k, v, a, beta = (oracle._f64(t) for t in (q, k, v, a, beta))
    t0 = time.perf_counter()
    oracle.forward(q, k, v, a, beta, s0=None, scale=x["scale"], n_threads=n_threads)
    dt = time.perf_counter() - t0
    used = oracle.threads_for(n_heads, n_threads)
    mtok = (n_heads / w.H) * w.T / dt / 1e6
    return {"value": mtok, "unit": "Mtokens/s", "cores": used, "kind": "oracle",
            "sample": f"{n_heads} of {w.B * w.H} (sequence, head) pairs x full T={w.T}, "
                      f"fp64 sequential loop, {dt:.2f} s wall; scaled by {n_heads}/{w.H} heads"}


def run_reference(args):
    """Reference arm: the fp64 oracle as it stands, on the host cores, bounded sample per step."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    import oracle
    from gated_delta_rule_122_b200.inputs import make_inputs, workload
    w = workload("prefill")
    n_threads = oracle.threads_for(10 ** 6)
    T_sample = 1024
    n_heads = min(w.H, max(n_threads, 4))
    ws = w.scaled(B=1, H=n_heads, T=T_sample)
    x = make_inputs(ws, device="cpu")
    f64 = [oracle._f64(x[n]) for n in ("q", "k", "v", "alpha", "beta")]
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.forward(*f64, s0=None, scale=x["scale"], n_threads=n_threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    value = (n_heads / w.H) * T_sample / step / 1e6
    used = oracle.threads_for(n_heads, n_threads)
    sample = (f"{n_heads} heads x T={T_sample} of the B=2 H=64 T=8192 d=128 prefill per step, "
              f"fp64 sequential loop; Mtokens/s scaled by {n_heads}/{w.H} heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Mtokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill B=2 H=64 T=8192 d_k=d_v=128 (bounded sample)",
                       "global_batch": 2, "seq_len": 8192, "parallelism": "host threads"},
            "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch

    import gated_delta_rule_122_b200 as kda
    from gated_delta_rule_122_b200.inputs import make_decode_inputs, make_inputs, workload

    world, rank, local, pg = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_kind = load_peaks()

    from gated_delta_rule_122_b200.shard import shard_bounds
    wp, wd = workload(args.prefill_workload), workload("decode")
    # the global batch is world x the workload's sequences; this rank's block of them
    p0, p1 = shard_bounds(world * wp.B, rank, world)
    d0, d1 = shard_bounds(world * wd.B, rank, world)
    wp, wd = wp.scaled(B=p1 - p0), wd.scaled(B=d1 - d0)
    if args.prefill_seqs is not None:
        wp = wp.scaled(B=args.prefill_seqs)
    if args.prefill_len is not None:
        wp = wp.scaled(T=args.prefill_len)
    x = make_inputs(wp, device=device, seed=wp.seed + p0)
    # the decode state (2.2 GB) is only allocated when the decode step runs
    y = make_decode_inputs(wd, device=device, seed=wd.seed + d0) if args.only != "prefill" else None
    o = torch.empty((wp.B, wp.T, wp.H, wp.dv), device=device, dtype=torch.float32)
    S = torch.empty((wp.B, wp.H, wp.dk, wp.dv), device=device, dtype=torch.float32)
    od = torch.empty((wd.B, wd.H, wd.dv), device=device, dtype=torch.float32)

    def prefill():
        if args.only == "decode":
            return
        kda.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=x["s0"],
                    scale=x["scale"], out=o, final_state=S)

    def decode():
        if args.only == "prefill":
            return
        kda.decode_step(y["q"], y["k"], y["v"], y["alpha"], y["beta"], y["state"],
                        scale=y["scale"], out=od)

    for _ in range(max(args.warmup, 0)):
        prefill()
        decode()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device.index)
    sampler.start()
    time.sleep(0.05)
    barrier(pg)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    start.record()
    for i in range(K):
        ev[i][0].record()
        prefill()
        ev[i][1].record()
        ev[i][2].record()
        decode()
        ev[i][3].record()
    end.record()
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    barrier(pg)
    sampler.mark(t_wall0, t_wall1)
    sampler.stop()

    step_ms = start.elapsed_time(end) / K
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / K
    step_ms, pre_ms, dec_ms = reduce_max(pg, [step_ms, pre_ms, dec_ms], device)
    pre_ms, dec_ms = max(pre_ms, 1e-9), max(dec_ms, 1e-9)

    tokens = wp.B * wp.T
    value = world * tokens / (pre_ms * 1e-3) / 1e6
    pb = prefill_bytes(wp, x["s0"] is not None)
    db = decode_bytes(wd)
    pre_gbs = pb / (pre_ms * 1e-3) / 1e9
    dec_gbs = db / (dec_ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])

    e2e = None
    if not args.no_e2e:
        # the whole step through the host-buffer C entry points: the prefill's inputs come
        # from pinned host memory and its o and final state go back (kda_forward_host), and
        # the decode step's token vectors come in and its o goes back with the state
        # resident on the device (kda_decode_step_host)
        hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta")}
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hS = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
        hy = {n: y[n].cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta")} if y is not None else None
        hod = torch.empty(od.shape, dtype=od.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in hx.values())
        d2h = ho.numel() * ho.element_size() + hS.numel() * hS.element_size()
        if hy is not None:
            h2d += sum(t.numel() * t.element_size() for t in hy.values())
            d2h += hod.numel() * hod.element_size()

        def host_step():
            kda.forward(hx["q"], hx["k"], hx["v"], hx["alpha"], hx["beta"], scale=x["scale"],
                        out=ho, final_state=hS)
            if hy is not None:
                kda.decode_step(hy["q"], hy["k"], hy["v"], hy["alpha"], hy["beta"], y["state"],
                                scale=y["scale"], out=hod)

        n_e2e = max(3, K // 4)
        host_step()   # warm-up of the host path
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(pg)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(n_e2e):
            host_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = reduce_max(pg, [e0.elapsed_time(e1) / n_e2e], device)[0]
        e2e = {"value": world * tokens / (e2e_ms * 1e-3) / 1e6, "unit": "Mtokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": n_e2e, "path": "kda_forward_host + kda_decode_step_host (C ABI, host buffers)"}

    long_leg = None
    if world == 1 and not args.no_long and args.only is None and args.prefill_seqs is None \
            and args.prefill_len is None and args.prefill_workload == "prefill":
        long_leg = measure_long(torch, kda, device, hbm)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_prefill(x, wp)
    rows = None
    if world == 1 and not args.no_rows and args.only is None and args.prefill_seqs is None \
            and args.prefill_len is None and args.prefill_workload == "prefill":
        rows = measure_rows(torch, kda, x, y, wp, float(peaks["hbm_gbs"]))

    clocks = sampler.summary()
    if rank != 0:
        return
    headline = args.prefill_seqs is None and args.prefill_len is None and args.prefill_workload == "prefill"
    traffic = PREFILL_TRAFFIC_BYTES if headline and kernel_sources_hash() == PREFILL_TRAFFIC_SOURCES else None
    dt = {torch.bfloat16: "bf16", torch.float32: "fp32"}
    workload_desc = (f"{wp.name} B={wp.B * world} H={wp.H} T={wp.T} d_k=d_v={wp.dk} {dt[wp.qkv_dtype]} q/k/v, "
                     f"{dt[wp.gate_dtype]} alpha/beta, fp32 o and state"
                     + (", random initial state" if wp.init_state else ""))
    if args.only != "prefill":
        workload_desc += f" (+ decode step N={wd.B * world} H={wd.H} d={wd.dk} in the same step)"
    line = {
        "metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload_desc,
                   "global_batch": wp.B * world, "seq_len": wp.T, "heads": wp.H, "d": wp.dk,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (126 MB), no flush",
                   "value_from": "prefill launches' CUDA-event time"},
        "prefill_ms": pre_ms,
        "roofline": {"bound": "hbm", "achieved": pre_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": pre_gbs / hbm, "traffic": traffic,
                     "algorithmic_bytes": pb, "peak_source": f"{peak_kind} hbm_gbs (copy)"},
        "decode": None if args.only == "prefill" else {
            "value": dec_gbs, "unit": "GB/s", "us_per_step": dec_ms * 1e3, "algorithmic_bytes": db,
            "frac_of_measured_hbm": dec_gbs / hbm, "frac_of_8TBs": dec_gbs / 8000.0},
        "long_prefill": long_leg,
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": (1 if args.only else 2) * K, "clocks": clocks,
        "next_rows": rows,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    try:
        main()
    finally:
        try:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                dist.destroy_process_group()
        except Exception:
            pass

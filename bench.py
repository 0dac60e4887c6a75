#!/usr/bin/env python
"""Benchmark of the gated-delta-rule QDQ-state hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on stdout (rank 0).  The headline `value` is GDN prefill
tokens/s on the GDN-prefill workload (B=4, H=16, T=4096, d_k=d_v=128, bf16
q/k/v, fp32 gates/state, FP8 E4M3 tile-64 state QDQ at every 64-token
chunk): one step = one gdn_prefill call over the whole batch with inputs
resident in HBM.  The serving-decode workload (256 sequences x 32 heads,
d=128, INT8 g32 state QDQ after every token, 512 single-token gdn_decode
calls) is measured in the same run and reported under "decode", the same
with the state stored packed under "decode_packed", one straight-through
backward call on the GDN-prefill workload under "backward", and the KDA and
packed-varlen prefill workloads under "prefill_other".  Beside each:
`roofline` (algorithmic bytes or flops per launch over the CUDA-event time,
against the measured peaks, with the DRAM traffic recorded by ncu for the
same sources), `cpu_baseline` (the oracle on the host cores) and, for the
headline, `e2e` (the same call with pinned host copies in the timed region).

With N > 1 (torchrun, one rank per GPU) every rank runs its own copy of the
workload (independent sequences; no collective on the data path), the step
time is the max over ranks, and `value` counts the tokens of all ranks.

`--impl reference` times the CPU oracle (fp64 token recurrence + fp32
codecs) on a bounded sample of the same workload on the host cores.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s + QDQ-state decode updates/s; % of TC / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


# The CUDA sources each recorded kernel is compiled from (its launch
# configuration in gdn_lib.cu is fixed per workload).
KERNEL_SOURCES = {
    "prefill_gdn": ["gdn_prefill_pair.cuh", "gdn_tc_util.cuh", "gdn_sm100.cuh", "gdn_common.cuh"],
    "decode": ["gdn_decode.cuh", "gdn_common.cuh"],
    "decode_packed": ["gdn_decode.cuh", "gdn_common.cuh"],
    "backward": ["gdn_backward.cuh", "gdn_common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of `kernel`'s CUDA sources; its recorded DRAM traffic is valid only for it."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "state_quantized_recurrence_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """Per-launch DRAM bytes (read + write) of `kernel` on the full workload,
    from profiles/traffic.json, or None if absent or taken on other sources."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
    except (OSError, ValueError, KeyError):
        return None
    ok = rec.get("source_hash") == kernel_source_hash(kernel)
    return rec.get("bytes_per_launch") if ok else None


# ------------------------------------------------------------ workload math
def prefill_bytes(tokens, n_states, H, dk, dv, in_bytes, state_in: bool, per_key: bool) -> int:
    """Algorithmic HBM bytes of one prefill call: q, k, v read and o written
    (in dtype), g and beta read (fp32), the states written (and read when an
    initial state is given)."""
    tok = tokens * H
    b = tok * (2 * dk + dv) * in_bytes + tok * dv * in_bytes
    b += tok * 4 * (dk if per_key else 1) + tok * 4
    b += n_states * H * dk * dv * 4 * (2 if state_in else 1)
    return b


def backward_bytes(tokens, n_states, H, dk, dv, in_bytes, state_in: bool, per_key: bool) -> int:
    """Algorithmic HBM bytes of one gdn_prefill_backward call: q, k, v and
    d_o read (in dtype), g and beta read, the initial state read; dq, dk, dv,
    dg, dbeta and dstate_in written in fp32 (the recomputation's re-reads and
    the workspace traffic are not algorithmic)."""
    tok = tokens * H
    g_el = dk if per_key else 1
    b = tok * (2 * dk + 2 * dv) * in_bytes + tok * 4 * (g_el + 1)
    b += tok * 4 * (2 * dk + dv + g_el + 1)
    b += n_states * H * dk * dv * 4 * (2 if state_in else 1)
    return b


def prefill_flops(tokens, H, dk, dv, C=64) -> int:
    """Dense algorithmic flops of the chunked WY form: per chunk of C tokens
    K K^T, Q K^T and W = T (bK): 3 * 2*C*C*d_k; U = T (bV) and Aqk Vn:
    2 * 2*C*C*d_v; W H0, Q H0 and K^T Vn: 3 * 2*C*d_k*d_v; counted per
    head-token (180,224 flop at d = 128)."""
    per_chunk = 3 * 2 * C * C * dk + 2 * 2 * C * C * dv + 3 * 2 * C * dk * dv
    return tokens * H * per_chunk // C


def decode_bytes_per_update(dk, dv, in_bytes, per_key: bool) -> int:
    """State read + write (fp32), q, k, v read and o written, g and beta."""
    return 2 * 4 * dk * dv + (2 * dk + dv) * in_bytes + dv * in_bytes + 4 * (dk if per_key else 1) + 4


def decode_bytes_per_update_packed(dk, dv, in_bytes, per_key: bool, qdq: str) -> int:
    """As decode_bytes_per_update with the state stored packed: one byte per
    code plus the fp32 scales (per INT8 group / FP8 tile), read and written."""
    n_scales = dv // 64 if qdq == "fp8_tile64" else dk * (dv // int(qdq.split("_g")[1]))
    return (2 * dk * dv + 2 * 4 * n_scales + (2 * dk + dv) * in_bytes + dv * in_bytes
            + 4 * (dk if per_key else 1) + 4)


# ------------------------------------------------------------ clock sampler
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, tagged with host time."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={period_ms}", f"-i={gpu_index}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        window = "timed region"
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = [p for (t, p) in self.samples if t0 - 0.5 <= t <= t1 + 0.5]
            window = "timed region +-0.5 s"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in inside if num(p[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in inside for i in range(4) if p[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(inside[0][2]), "reasons": reasons,
                "power_w_max": max((num(p[3]) or 0.0) for p in inside),
                "samples": len(inside), "window": window}


# ------------------------------------------------------------ distributed
class Dist:
    def __init__(self, n_gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={self.world}")

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        dev = "cuda" if self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------ our arm
def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_prefill(case, inp, min_seconds: float = 8.0, max_passes: int = 50) -> dict:
    """The oracle as it stands, on whole sequences of the workload (all
    heads), on this host's cores; tokens/s over passes through the
    workload's sequences until about `min_seconds` of CPU work (a whole
    sequence at a time).  One sequence is also run on a single thread."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    lengths = [int(x) for x in inp["lengths"]]
    packed = inp["cu_seqlens"] is not None
    done, tokens, t_total = 0, 0, 0.0
    for _ in range(max_passes):
        start = 0
        for s, n in enumerate(lengths):
            # one whole sequence (all heads): a batch row, or its packed token range
            sl = (slice(0, 1), slice(start, start + n)) if packed else (slice(s, s + 1),)
            st_in = inp["state_in"][s:s + 1] if inp["state_in"] is not None else None
            t0 = time.perf_counter()
            oracle.recurrence(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["g"][sl],
                              inp["beta"][sl], st_in, oracle.dense_cu_seqlens(1, n),
                              per_key_gate=case.gate == "per_key", qdq=case.qdq,
                              n_threads=threads)
            t_total += time.perf_counter() - t0
            start += n
            done += 1
            tokens += n
            if t_total >= min_seconds:
                break
        if t_total >= min_seconds:
            break
    # the first sequence again on one thread (its first 1024 tokens at most)
    n1 = min(1024, lengths[0])
    sl1 = (slice(0, 1), slice(0, n1))
    st1 = inp["state_in"][0:1] if inp["state_in"] is not None else None
    t0 = time.perf_counter()
    oracle.recurrence(inp["q"][sl1], inp["k"][sl1], inp["v"][sl1], inp["g"][sl1],
                      inp["beta"][sl1], st1, oracle.dense_cu_seqlens(1, n1),
                      per_key_gate=case.gate == "per_key", qdq=case.qdq, n_threads=1)
    t1 = time.perf_counter() - t0
    return {"value": tokens / t_total, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} whole sequences of the workload's {len(lengths)}, cycling "
                      f"({tokens} tokens x {case.H} heads), fp64 token recurrence + fp32 "
                      f"{case.qdq} codec, OpenMP over heads",
            "seconds": round(t_total, 3), "value_1_thread": round(n1 / t1, 1),
            "sample_1_thread": f"{n1} tokens x {case.H} heads of sequence 0",
            "cpu_model": cpu_model()}


def cpu_baseline_decode(case, inp, state, min_seconds: float = 6.0) -> dict:
    """The decode oracle on all sequences of the workload: one token first,
    then as many further tokens as about `min_seconds` of CPU work allow."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    n_seq = case.n_seq

    def run(t0_tok, n_tok, st):
        sl = (slice(t0_tok, t0_tok + n_tok), slice(0, n_seq))
        t0 = time.perf_counter()
        res = oracle.decode(inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl],
                            inp["dec_g"][sl], inp["dec_beta"][sl], st, per_key_gate=False,
                            qdq=case.qdq, n_threads=threads)
        return time.perf_counter() - t0, res[1]

    dt, st = run(0, 1, state[:n_seq])
    steps = int(inp["dec_q"].shape[0])
    more = max(0, min(steps - 1, int((min_seconds - dt) / max(dt, 1e-6))))
    n_tok = 1
    if more > 0:
        dt2, _ = run(1, more, st)
        dt += dt2
        n_tok += more
    return {"value": n_tok * n_seq * case.H / dt, "unit": "updates/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{n_tok} tokens of all {n_seq} sequences x {case.H} heads",
            "seconds": round(dt, 3)}


def cpu_baseline_backward(case, inp, d_o, max_tokens: int = 512) -> dict:
    """The backward oracle (fp64 numpy, one (sequence, head) at a time) on
    the first `max_tokens` tokens of the first sequence, all heads."""
    from oracle import backward as obw
    n = min(max_tokens, int(inp["lengths"][0]))
    sl = (slice(0, 1), slice(0, n))
    st_in = inp["state_in"][0:1] if inp["state_in"] is not None else None
    t0 = time.perf_counter()
    obw.backward(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["g"][sl], inp["beta"][sl], st_in,
                 [0, n], d_o[sl], None, per_key_gate=case.gate == "per_key", qdq=case.qdq)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of 1 of {case.n_seq} sequences x {case.H} heads, fp64 token "
                      f"reverse pass (numpy, one thread), {case.qdq} straight through",
            "seconds": round(dt, 3)}


def measure_backward(args, dist, dev, stream, sampler, peaks, case, steps, warmup) -> dict:
    """Time `steps` gdn_prefill_backward calls of `case` (inputs, upstream
    gradient and workspace resident in HBM)."""
    import torch

    import gdn_synth as gs
    import state_quantized_recurrence_b200 as sqr

    inp = gs.generate(case)
    gen = torch.Generator().manual_seed(case.seed + 500)
    d_o = torch.randn(inp["v"].shape, generator=gen).to(inp["q"].dtype)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    d_o_dev = d_o.to(dev)
    T_arg = int(sum(inp["lengths"])) if d["cu_seqlens"] is not None else case.T
    need = int(sqr.lib.gdn_prefill_backward_workspace_bytes(
        case.n_seq, T_arg, case.H, case.d_k, case.d_v, int(d["cu_seqlens"] is not None)))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def step():
        return sqr.gdn_prefill_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o_dev,
                                        d["state_in"], d["cu_seqlens"], None, qdq=case.qdq,
                                        workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    sqr.check_last_error(where=f"{case.name} backward warm-up")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    dist.barrier()
    ms = dist.max(ev0.elapsed_time(ev1) / steps)
    tokens = int(sum(inp["lengths"]))
    nbytes = backward_bytes(tokens, case.n_seq, case.H, case.d_k, case.d_v,
                            2 if case.dtype == "bf16" else 4, inp["state_in"] is not None,
                            case.gate == "per_key")
    gbs = nbytes / (ms / 1e3) / 1e9
    res = {
        "metric": "prefill backward tokens/s (straight-through state QDQ)",
        "workload": f"{case.name}: n_seq={case.n_seq} H={case.H} tokens={tokens} d={case.d_k}, "
                    f"{case.dtype}, {case.gate} gate, {case.qdq}, random d_o, no dstate_out",
        "value": round(dist.world * tokens / (ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms, 4), "steps": steps,
        "kernel": "bwd::prefill_backward_kernel (FFMA, token-reverse with chunk checkpoints)",
        "workspace_bytes": need,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 5),
                     "traffic": recorded_traffic("backward"),
                     "bytes_per_launch": nbytes, "peak_source": peaks["source"]},
        "gpu_launches": steps, "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if dist.rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_backward(case, inp, d_o)
    del d, d_o_dev, ws
    torch.cuda.empty_cache()
    return res


def measure_prefill(args, dist, dev, stream, sampler, peaks, case, steps, warmup,
                    traffic_key=None, keep=False, cpu=False):
    """Time `steps` gdn_prefill calls of `case` (inputs resident in HBM).
    Returns the result dict (and the device buffers when `keep`)."""
    import torch

    import gdn_synth as gs
    import state_quantized_recurrence_b200 as sqr

    inp = gs.generate(case)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    o = torch.empty(d["v"].shape, dtype=d["q"].dtype, device=dev)
    st = torch.empty((case.n_seq, case.H, case.d_k, case.d_v), dtype=torch.float32, device=dev)

    def step():
        sqr.gdn_prefill_into(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"],
                             d["cu_seqlens"], o, st, qdq=case.qdq)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    sqr.check_last_error(where=f"{case.name} warm-up")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    dist.barrier()
    ms = ev0.elapsed_time(ev1) / steps
    ms_max = dist.max(ms)
    tokens = int(sum(inp["lengths"]))
    in_bytes = 2 if case.dtype == "bf16" else 4
    nbytes = prefill_bytes(tokens, case.n_seq, case.H, case.d_k, case.d_v, in_bytes,
                           inp["state_in"] is not None, case.gate == "per_key")
    flops = prefill_flops(tokens, case.H, case.d_k, case.d_v)
    gbs = nbytes / (ms / 1e3) / 1e9
    tfs = flops / (ms / 1e3) / 1e12
    kernel = {"tc_wy_pair": "wy::prefill_wy_kernel (tcgen05, WY-form CTA pair per unit)",
              "tc_cta_pair": "pair::prefill_pair_kernel (tcgen05, CTA pair per unit)",
              "tc_one_cta": "tc::prefill_tc_kernel (tcgen05, one CTA per unit)",
              "cuda_cores": "simt::prefill_simt_kernel (FFMA)"}[
        sqr.gdn_prefill_schedule(case.n_seq, case.H, case.d_k, case.d_v, d["q"].dtype, case.gate,
                                 case.qdq)]
    res = {
        "workload": f"{case.name}: n_seq={case.n_seq} H={case.H} tokens={tokens} d={case.d_k}, "
                    f"{case.dtype}, {case.gate} gate, {case.qdq}, "
                    f"{'random' if inp['state_in'] is not None else 'zero'} initial state",
        "value": round(dist.world * tokens / (ms_max / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms_max, 5), "steps": steps,
        "kernel": kernel,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": (None if (args.small or traffic_key is None)
                                 else recorded_traffic(traffic_key)),
                     "bytes_per_launch": nbytes, "peak_source": peaks["source"],
                     "tensor": {"achieved": round(tfs, 2), "peak": peaks["bf16_tflops"],
                                "unit": "TFLOP/s", "frac": round(tfs / peaks["bf16_tflops"], 4),
                                "flops_per_launch": flops}},
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if cpu and dist.rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_prefill(case, inp, min_seconds=4.0)
    if keep:
        return res, (inp, d, o, st, step, tokens, nbytes)
    del d, o, st
    torch.cuda.empty_cache()
    return res


def run_ours(args, dist: Dist) -> dict:
    import torch

    import gdn_synth as gs
    import state_quantized_recurrence_b200 as sqr

    peaks = load_peaks()
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    dev = torch.device("cuda", dist.local)
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(dist.local)

    if args.only == "backward":  # profiler captures of the backward kernel
        bcase = gs.CONFIGS["gdn_prefill"]
        if args.small:  # the same 128 CTAs, 4 chunks each
            bcase = gs.small_case("gdn_prefill", T=256)
        bwd = measure_backward(args, dist, dev, stream, sampler, peaks, bcase, args.steps,
                               args.warmup)
        sampler.stop()
        dist.close()
        return {"metric": bwd["metric"], "value": bwd["value"], "unit": bwd["unit"],
                "n_gpus": dist.world, "impl": "ours", "backward": bwd}
    if args.only in ("decode", "decode_packed"):  # profiler captures of one decode kernel
        dec = run_decode(args, dist, dev, stream, sampler, peaks, packed=args.only == "decode_packed")
        sampler.stop()
        dist.close()
        return {"metric": dec["metric"], "value": dec["value"], "unit": dec["unit"],
                "n_gpus": dist.world, "impl": "ours", "decode": dec}
    if args.only == "kda":  # profiler captures of the CUDA-core prefill kernel
        kcase = gs.small_case("kda_prefill", decode_steps=0)
        if args.small:  # the same 128 CTAs, 8 chunks each
            kcase = gs.small_case("kda_prefill", T=512, decode_steps=0)
        kda = measure_prefill(args, dist, dev, stream, sampler, peaks, kcase, args.steps,
                              args.warmup)
        sampler.stop()
        dist.close()
        return {"metric": "prefill tokens/s", "value": kda["value"], "unit": kda["unit"],
                "n_gpus": dist.world, "impl": "ours", "kda_prefill": kda}

    # ---------------- prefill (headline) ----------------
    case = gs.CONFIGS["gdn_prefill"]
    if args.small:  # same CTA count (B*H = 64), 8 chunks: for profiler captures
        case = gs.small_case("gdn_prefill", T=512)
    head, (inp, d, o, st, step, tokens, nbytes) = measure_prefill(
        args, dist, dev, stream, sampler, peaks, case, args.steps, args.warmup,
        traffic_key="prefill_gdn", keep=True)
    ms_max = head["ms_per_step"]
    value = head["value"]
    clocks = head["clocks"]
    roofline = dict(head["roofline"], kernel="prefill (one launch per step)")
    B, T, H, dk, dv = case.n_seq, case.T, case.H, case.d_k, case.d_v

    # e2e through the C ABI from pinned host buffers (copies inside the timed region)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, dist, d, o, st, step, stream, tokens)
    cpu = None
    if dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_prefill(case, inp)
    del d, o, st
    torch.cuda.empty_cache()

    # ---------------- decode ----------------
    dec = dec_packed = None
    if not args.no_decode:
        dec = run_decode(args, dist, dev, stream, sampler, peaks)
        if not args.small:
            dec_packed = run_decode(args, dist, dev, stream, sampler, peaks, packed=True)

    # ---------------- the other prefill workloads (KDA, packed varlen) ----------------
    others = {}
    if not args.only and not args.small and not args.no_others:
        for name in ("kda_prefill", "varlen"):
            c = gs.small_case(name, decode_steps=0)
            others[name] = measure_prefill(args, dist, dev, stream, sampler, peaks, c,
                                           max(3, min(args.steps, 10)), args.warmup, cpu=True)

    # ---------------- backward (straight-through QDQ) on the prefill workload ----------------
    bwd = None
    if not args.only and not args.small and not args.no_others:
        bwd = measure_backward(args, dist, dev, stream, sampler, peaks, gs.CONFIGS["gdn_prefill"],
                               3, 3)

    sampler.stop()

    def pick(d, *path):
        for k in path:
            if not isinstance(d, dict) or d.get(k) is None:
                return None
            d = d[k]
        return d

    # the other targets, flat at the top level of the line
    flat = {
        "tensor_frac": pick(roofline, "tensor", "frac"),
        "decode_updates_per_s": pick(dec, "value"),
        "decode_ms_per_token_step": pick(dec, "ms_per_token_step"),
        "decode_hbm_frac": pick(dec, "roofline", "frac"),
        "decode_packed_updates_per_s": pick(dec_packed, "value"),
        "decode_packed_hbm_frac": pick(dec_packed, "roofline", "frac"),
        "kda_ms_per_step": pick(others, "kda_prefill", "ms_per_step"),
        "kda_hbm_frac": pick(others, "kda_prefill", "roofline", "frac"),
        "varlen_ms_per_step": pick(others, "varlen", "ms_per_step"),
        "varlen_hbm_frac": pick(others, "varlen", "roofline", "frac"),
        "backward_ms_per_step": pick(bwd, "ms_per_step"),
        "backward_hbm_frac": pick(bwd, "roofline", "frac"),
    }
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"gdn_prefill B={B} H={H} T={T} d_k={dk} d_v={dv}, bf16 q/k/v, "
                               f"fp32 g/beta/state, {case.qdq} state QDQ, zero initial state",
                   "global_batch": B * dist.world, "seq_len": T,
                   "l2": f"inputs {nbytes / 1e6:.0f} MB > 126 MB L2, no flush",
                   "parallelism": f"dp{dist.world} (independent sequences per rank)"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "clocks": clocks, "decode": dec, "decode_packed": dec_packed,
        "prefill_other": others or None, "backward": bwd, "impl": "ours",
        **flat,
    }
    dist.close()
    return res


def run_e2e(args, dist, d, o, st, step, stream, tokens) -> dict:
    """The headline metric through the C ABI with the step's inputs copied
    from pinned host memory and its outputs read back, inside the timed region."""
    import torch
    host = {k: d[k].cpu().pin_memory() for k in ("q", "k", "v", "g", "beta")}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    st_h = torch.empty(st.shape, dtype=st.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_step():
        for k in host:
            d[k].copy_(host[k], non_blocking=True)
        step()
        o_h.copy_(o, non_blocking=True)
        st_h.copy_(st, non_blocking=True)

    e2e_step()
    dev = o.device
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    ms_e2e = dist.max(ev0.elapsed_time(ev1) / e2e_steps)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + st_h.numel() * st_h.element_size()
    return {"value": dist.world * tokens / (ms_e2e / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms_e2e, 4), "steps": e2e_steps}


def run_decode(args, dist, dev, stream, sampler, peaks, packed: bool = False) -> dict:
    """The serving decode workload: 512 single-token calls in one CUDA graph,
    the state in fp32 storage, or (``packed``) as codes + scales."""
    import torch

    import gdn_synth as gs
    import state_quantized_recurrence_b200 as sqr

    case = gs.CONFIGS["serving_decode"]
    if args.small:  # 64 x 32 heads (134 MB of state > L2), 16 tokens: for profiler captures
        case = gs.small_case("serving_decode", n_seq=64, decode_steps=16)
    inp = gs.generate(case)
    S_steps = case.decode_steps
    dq, dk_, dv_ = inp["dec_q"].to(dev), inp["dec_k"].to(dev), inp["dec_v"].to(dev)
    dg, db = inp["dec_g"].to(dev), inp["dec_beta"].to(dev)
    state0 = inp["state_in"].to(dev)
    o = torch.empty((S_steps,) + tuple(dv_.shape[1:]), dtype=dq.dtype, device=dev)
    if packed:
        ps0 = sqr.gdn_state_pack(state0, case.qdq)
        ps = sqr.PackedState(ps0.codes.clone(), ps0.scales.clone(), case.qdq)

        def reset():
            ps.codes.copy_(ps0.codes)
            ps.scales.copy_(ps0.scales)

        def run_all():
            for t in range(S_steps):
                sqr.gdn_decode_packed_into(dq[t], dk_[t], dv_[t], dg[t], db[t], ps, o[t])
    else:
        state = state0.clone()

        def reset():
            state.copy_(state0)

        def run_all():
            for t in range(S_steps):
                sqr.gdn_decode_into(dq[t], dk_[t], dv_[t], dg[t], db[t], state, o[t], qdq=case.qdq)

    # warm-up, then capture the whole token loop in one CUDA graph
    for _ in range(max(1, args.warmup)):
        reset()
        run_all()
    torch.cuda.synchronize(dev)
    sqr.check_last_error(where="decode warm-up")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_all()
    reset()
    graph.replay()
    torch.cuda.synchronize(dev)
    reps = 3
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(reps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    dist.barrier()
    ms_loop = dist.max(ev0.elapsed_time(ev1) / reps)
    updates = case.n_seq * case.H * S_steps
    ups = dist.world * updates / (ms_loop / 1e3)
    bpu = (decode_bytes_per_update_packed(case.d_k, case.d_v, 2, False, case.qdq) if packed
           else decode_bytes_per_update(case.d_k, case.d_v, 2, False))
    ms_tok = ms_loop / S_steps
    gbs = case.n_seq * case.H * bpu / (ms_tok / 1e3) / 1e9
    cpu = None
    if dist.world == 1 and not args.no_cpu_baseline and not packed:
        cpu = cpu_baseline_decode(case, inp, inp["state_in"])
    del graph
    storage = ("packed state (1-byte codes + fp32 scales per group)" if packed
               else "fp32 state")
    return {"metric": "QDQ-state decode updates/s", "value": round(ups, 1), "unit": "updates/s",
            "sequence_tokens_per_s": round(ups / case.H, 1),
            "workload": f"serving_decode {case.n_seq} seq x H={case.H}, d=128, bf16, "
                        f"{case.qdq}, {S_steps} single-token calls in one CUDA graph, {storage}",
            "ms_per_token_step": round(ms_tok, 5), "reps": reps,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "traffic": None if args.small else recorded_traffic(
                             "decode_packed" if packed else "decode"),
                         "bytes_per_update": bpu, "bytes_per_launch": case.n_seq * case.H * bpu,
                         "peak_source": peaks["source"]},
            "gpu_launches": S_steps * reps, "clocks": sampler.summary(t_wall0, t_wall1),
            "cpu_baseline": cpu}


# ------------------------------------------------------------ reference arm
def run_reference(args, dist: Dist) -> dict | None:
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample (the first sequence, all heads, all 4096 tokens) of the workload."""
    if dist.rank != 0:
        return None
    import gdn_synth as gs
    import oracle

    case = gs.CONFIGS["gdn_prefill"]
    inp = gs.generate(case)
    threads = len(os.sched_getaffinity(0))
    Ts = 4096
    sl = (slice(0, 1), slice(0, Ts))

    def step():
        oracle.recurrence(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["g"][sl],
                          inp["beta"][sl], None, oracle.dense_cu_seqlens(1, Ts),
                          per_key_gate=False, qdq=case.qdq, n_threads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = Ts / dt
    sample = f"1 sequence x {case.H} heads x {Ts} tokens of the gdn_prefill workload per step"
    return {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"gdn_prefill B={case.n_seq} H={case.H} T={case.T} d=128, "
                                   f"{case.qdq} (sampled)", "global_batch": case.n_seq,
                       "seq_len": case.T, "parallelism": "host cores"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode", "decode_packed", "backward", "kda"],
                    default=None,
                    help="measure one kernel only (profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the KDA and packed-varlen prefill measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--small", action="store_true", help="small case (profiling captures)")
    args = ap.parse_args()
    if args.only == "prefill":
        args.no_decode = True
    if args.warmup < 3 and not args.small:
        raise SystemExit("--warmup must be >= 3")
    dist = Dist(args.gpus)
    if args.impl == "reference":
        res = run_reference(args, dist)
    else:
        res = run_ours(args, dist)
    if res is not None and dist.rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

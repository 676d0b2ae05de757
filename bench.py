"""Benchmark of the Gated Delta Rule-2 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|long|varlen] [--no-cpu-baseline]
                    [--no-e2e] [--no-backward] [--no-extra-workloads]

One step = one chunkwise forward (gdr2_chunk_fwd, bf16, H=16, d_k=d_v=128)
over the layer-shaped prefill batch B=4 x T=2048 (8,192 tokens). The line's
`value` is tokens/s over all ranks: K steps back to back, timed with CUDA
events on the launching stream between barriers (max over ranks), i.e. the
mean step time. Every per-launch figure also carries its median, p10 and p90.
In the same run:
  * roofline  -- the chunk forward's bound: the slower of its algorithmic HBM
                 bytes at the measured copy bandwidth and its algorithmic
                 FLOPs at the measured bf16 tensor-core rate (the bytes, for
                 this workload); achieved = bytes / median launch time;
  * l2_flushed -- the same launch timed alone after overwriting a 256 MiB
                 buffer (twice L2) before every launch;
  * long, varlen -- a few launches of the long-context (T=32768, H=16) and
                 packed variable-length (64 sequences) workloads, each with
                 its own roofline;
  * decode    -- 64 consecutive gdr2_recurrent_step calls on N=256 x H=16
                 heads (fp32 state 256 MiB), fresh token inputs every step,
                 achieved HBM GB/s per step;
  * e2e       -- the same tokens/s with pinned host inputs copied in and o and
                 the final states copied out inside every timed step;
  * backward  -- the gate-aware backward (gdr2_chunk_bwd) on the same batch:
                 time per call and its fp32 CUDA-core flops against the SIMT
                 fp32 peak (the kernels are ALU-bound);
  * cpu_baseline -- the fp64 oracle on the host cores (rank 0, N=1 only);
  * clocks    -- SM clock and throttle reasons sampled (NVML) while timing.
The prefill inputs (268 MB of token tensors) are larger than L2 (126 MB), so
the back-to-back steps of the headline number run without a flush.

Under torchrun every rank runs its own replica of the workload on its own GPU
(the (sequence, head) units are independent: no collective on the data path;
NCCL carries only the barrier and the max-over-ranks timing reduction).

--impl reference times the fp64 oracle (the only reference this operator
has) on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_recurrence_gdr2_b200 import inputs as gen  # noqa: E402

METRIC = "tokens/s of GDR-2 chunk fwd (bf16, H=16,d=128) + % roofline; decode HBM GB/s"
PEAK_FALLBACK_GBS = 6650.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return PEAK_FALLBACK_GBS, 1590.0, "fallback"


def workload(name: str):
    if name == "prefill":
        return gen.layer_prefill(), "layer prefill B=4 T=2048 H=16 d_k=d_v=128 bf16, zero initial state"
    if name == "long":
        return gen.long_context(), "long context B=1 T=32768 H=16 d=128 bf16, initial state 0.01*N(0,1)"
    if name == "varlen":
        return gen.varlen_packed(), "64 packed sequences, lengths U[128,8192], H=16 d=128 bf16"
    raise ValueError(name)


def measured_traffic():
    """DRAM bytes per chunk-forward launch from the committed ncu capture
    (profiles/traffic.json), or None once the kernel source has changed since
    the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
        with open(os.path.join(ROOT, t["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except (OSError, KeyError, ValueError):
        return None
    return int(t["bytes_per_launch"]) if sha == t["source_sha256_16"] else None


def chunk_bytes(inp) -> int:
    """Algorithmic HBM bytes of one chunk-forward launch: every input read
    once, o written once, initial states read once (if given), final states
    written once."""
    ntok = inp.q.shape[0] * inp.q.shape[1]
    H, dk = inp.q.shape[2], inp.q.shape[3]
    dv = inp.v.shape[3]
    el = 2 if inp.dtype == "bf16" else 4
    per_token_head = el * (3 * dk + 2 * dv) + 4 * dk + el * dv
    state = inp.num_seqs * H * dk * dv * 4
    return ntok * H * per_token_head + state * (2 if inp.init_state is not None else 1)


# fp32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flops (FMA) x 1.965 GHz
SIMT_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_flops(inp) -> int:
    """fp32 flops of one backward call per its three sweeps, per token-head and
    state element: forward sweep 5 (decay, read, write), reverse sweep 7
    (output term, du, decayed erase), per-chunk rows 14 (7 per pass)."""
    ntok = inp.q.shape[0] * inp.q.shape[1]
    H, dk = inp.q.shape[2], inp.q.shape[3]
    dv = inp.v.shape[3]
    return 26 * ntok * H * dk * dv


def decode_bytes(N, H, dk, dv, el=2) -> int:
    """Per decode step: state read + write, token inputs and o."""
    return N * H * (2 * dk * dv * 4 + el * (3 * dk + 2 * dv) + 4 * dk + el * dv)


def chunk_flops_per_chunk(d: int, C: int = 64) -> int:
    """Algorithmic FLOPs of the chunk form for one (chunk, head), triangular
    structure exploited: A = strict_tril(Ebar Kbar^T), P = tril(Qbar Kbar^T),
    (I + A)^{-1} (C^3 / 3), W = T Ebar and U0 = T Z (unit lower-triangular T),
    W S, Qbar S and (K e^{g_C - g})^T U (dense d x d), tril(P) U."""
    strict, incl = C * (C - 1) // 2, C * (C + 1) // 2
    return (strict * 2 * d + incl * 2 * d + C ** 3 // 3 + 2 * strict * 2 * d
            + 3 * C * d * d * 2 + incl * 2 * d)


def chunk_flops(inp) -> int:
    """Algorithmic FLOPs of one chunk-forward launch: every chunk of every
    sequence (a ragged last chunk counted whole, as the kernels run it)."""
    H, d = inp.q.shape[2], inp.q.shape[3]
    if inp.cu_seqlens is not None:
        lengths = np.diff(np.asarray(inp.cu_seqlens, dtype=np.int64))
        chunks = int(np.sum((lengths + 63) // 64))
    else:
        chunks = inp.q.shape[0] * ((inp.q.shape[1] + 63) // 64)
    return chunks * H * chunk_flops_per_chunk(d)


def stats_ms(per_ms):
    """Mean, median, p10 and p90 of per-launch times (ms -> us)."""
    xs = np.asarray(per_ms, dtype=np.float64) * 1e3
    return {"mean_us": float(xs.mean()), "median_us": float(np.median(xs)),
            "p10_us": float(np.percentile(xs, 10)), "p90_us": float(np.percentile(xs, 90))}


def chunk_roofline(inp, us, hbm_peak, tflops_peak, peak_src):
    """The chunk forward's roofline at a launch time of `us` microseconds: the
    bound is the slower of bytes / HBM bandwidth and FLOPs / tensor rate."""
    nbytes, flops = chunk_bytes(inp), chunk_flops(inp)
    t_hbm = nbytes / (hbm_peak * 1e9) * 1e6
    t_tc = flops / (tflops_peak * 1e12) * 1e6
    hbm = t_hbm >= t_tc
    achieved = nbytes / (us * 1e-6) / 1e9 if hbm else flops / (us * 1e-6) / 1e12
    peak = hbm_peak if hbm else tflops_peak
    return {"bound": "hbm" if hbm else "tensor", "achieved": achieved, "peak": peak,
            "unit": "GB/s" if hbm else "TFLOP/s", "frac": achieved / peak,
            "bytes_per_launch": nbytes, "flops_per_launch": flops,
            "t_hbm_us": t_hbm, "t_tensor_us": t_tc,
            "tensor_peak_tflops": tflops_peak, "peak_source": peak_src}


class ClockSampler:
    """Samples the SM clock and throttle reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no samples
            self.error = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.reasons |= int(r) & ~0x1
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b],
                "samples": len(self.samples)}


_T0 = time.time()


def log(msg: str) -> None:
    """Progress on stderr (the JSON line alone goes to stdout)."""
    sys.stderr.write(f"[bench {time.time() - _T0:7.1f}s] {msg}\n")
    sys.stderr.flush()


def reduce_max(x: float, device=None) -> float:
    """Max of a per-rank number over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own replica of the
    workload, so the job moves world x tokens_per_rank tokens in the slowest
    rank's time."""
    return world * tokens_per_rank / (max_ms * 1e-3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    """Reference arm: the fp64 oracle on the host cores, a bounded sample per step."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    import oracle
    inp, label = workload(args.workload)
    B, T, H, d = inp.q.shape
    sample_tokens = 128
    sl = lambda x: np.ascontiguousarray(x[:, :sample_tokens], dtype=np.float64)
    arrs = [sl(x) for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w)]
    s0 = (inp.init_state.astype(np.float64)
          if inp.init_state is not None and inp.cu_seqlens is None else None)
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle.forward(*arrs, s0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(*arrs, s0)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    tokens = arrs[0].shape[0] * arrs[0].shape[1]
    val = tokens / dt
    sample = (f"{arrs[0].shape[0]} sequences x first {arrs[0].shape[1]} tokens x {H} heads "
              f"of the {label} workload per step")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": label, "sample": sample},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(inp, label, wall_s=2.0):
    """Times the fp64 oracle on the host cores on a bounded sample of the
    workload: all sequences and heads, the first tokens, doubling the token
    count until one call takes about `wall_s` seconds (or covers everything)."""
    import oracle
    B, T, H, d = inp.q.shape
    cores = oracle.max_threads()
    tokens = min(T, 32)
    while True:
        sl = lambda x: np.ascontiguousarray(x[:, :tokens], dtype=np.float64)
        arrs = [sl(x) for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w)]
        t0 = time.perf_counter()
        oracle.forward(*arrs, None)
        dt = time.perf_counter() - t0
        if dt >= wall_s or tokens >= T:
            break
        tokens = min(T, tokens * 2)
    ntok = arrs[0].shape[0] * arrs[0].shape[1]
    return {"value": ntok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"all {B} sequences x first {tokens} tokens x {H} heads of the "
                      f"{label} workload ({dt:.2f} s wall of fp64 work on {cores} threads)"}


def cpu_backward_baseline(inp, d_o, label, tokens=512, heads=1):
    """Times the fp64 backward oracle (oracle.backward, plain numpy) on the
    host on a bounded sample: sequence 0, its first `tokens` tokens and
    `heads` heads, with the benchmark's output cotangents and no final-state
    cotangent. Reported in tokens/s of all H heads, like the GPU number."""
    import oracle
    B, T, H, d = inp.q.shape
    tokens = min(tokens, T)
    if inp.cu_seqlens is not None:   # stay inside the packed batch's first sequence
        tokens = min(tokens, int(inp.cu_seqlens[1] - inp.cu_seqlens[0]))
    sl = lambda x: np.ascontiguousarray(x[:1, :tokens, :heads], dtype=np.float64)
    arrs = [sl(x) for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.b, inp.w)]
    s0 = (np.ascontiguousarray(inp.init_state[:1, :heads], dtype=np.float64)
          if inp.init_state is not None else None)
    t0 = time.perf_counter()
    oracle.backward(*arrs, s0, sl(d_o), None)
    dt = time.perf_counter() - t0
    return {"value": tokens * heads / H / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"sequence 0, first {tokens} tokens, {heads} of {H} heads of the {label} "
                      f"workload ({dt:.2f} s wall of fp64 numpy on one thread)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "long", "varlen"], default="prefill")
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-qed", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the long-context and packed-batch objects")
    ap.add_argument("--extra-launches", type=int, default=4)
    ap.add_argument("--backward-calls", type=int, default=5)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)

    import torch
    import linear_attention_recurrence_gdr2_b200 as gdr2

    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dev)

    hbm_peak, tc_peak, peak_src = load_peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # twice the 126 MB L2

    def upload(inp):
        tdt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
        host = {k: torch.from_numpy(getattr(inp, k)).to(tdt if k != "log_alpha" else torch.float32)
                for k in ("q", "k", "v", "b", "w", "log_alpha")}
        t = {k: x.to(dev) for k, x in host.items()}
        t["s0"] = torch.from_numpy(inp.init_state).to(dev) if inp.init_state is not None else None
        t["cu"] = (torch.from_numpy(inp.cu_seqlens.astype(np.int32)).to(dev)
                   if inp.cu_seqlens is not None else None)
        B, T, H, d = inp.q.shape
        t["o"] = torch.empty((B, T, H, d), dtype=tdt, device=dev)
        t["sf"] = torch.empty((inp.num_seqs, H, d, d), dtype=torch.float32, device=dev)
        code = gdr2.GDR2_BF16 if inp.dtype == "bf16" else gdr2.GDR2_FP32
        wsb = gdr2.workspace_size(B, T, H, d, d, inp.num_seqs, code)
        t["ws"] = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
        t["ws_bytes"] = wsb
        return host, t

    def fwd(t):
        gdr2.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], t["s0"], t["cu"],
                       o=t["o"], final_state=t["sf"], workspace=t["ws"])

    def per_launch(fn, n, flush=False):
        """Per-launch CUDA-event times (ms) of n launches of fn, each bracketed
        by its own events; with flush, a 256 MiB write precedes every launch
        (outside the events)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for e0, e1 in ev:
            if flush:
                flush_buf.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    log(f"generating the {args.workload} workload")
    inp, label = workload(args.workload)
    host, t = upload(inp)
    log("timing the chunk forward")
    N = inp.num_seqs
    B, T, H, d = inp.q.shape
    step = lambda: fwd(t)
    # the chunk kernel; plus the order kernel of a packed batch, or the combine
    # and correction kernels of a segment split (few long sequences)
    launches_per_step = (1 + (1 if t["cu"] is not None and N > 1 else 0)
                         + (2 if t["cu"] is None and t["ws_bytes"] > 0 else 0))
    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    with clocks:
        for _ in range(args.warmup):
            step()
        barrier()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        barrier()
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
        total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]))
        flushed = per_launch(step, min(args.steps, 20), flush=True)
        barrier()
        log(f"chunk forward: {1e3 * statistics.median(per):.1f} us median")

        # The other chunk-forward workloads, a few launches each.
        extra = {}
        if not args.no_extra_workloads:
            for name in ("long", "varlen"):
                if name == args.workload:
                    continue
                log(f"generating the {name} workload")
                x_inp, x_label = workload(name)
                _, xt = upload(x_inp)
                log(f"timing {name}")
                xstep = lambda xt=xt: fwd(xt)
                xstep()
                barrier()
                xper = per_launch(xstep, args.extra_launches)
                st = stats_ms(xper)
                roof = chunk_roofline(x_inp, st["median_us"], hbm_peak, tc_peak, peak_src)
                extra[name] = {"workload": x_label, "tokens": x_inp.num_tokens, "launches": len(xper),
                               **st, "roofline": roof,
                               "segments": ("split" if xt["cu"] is None and xt["ws_bytes"] > 0 else "serial"),
                               "tokens_per_s": x_inp.num_tokens / (st["median_us"] * 1e-6)}
                del xt
                torch.cuda.empty_cache()
            barrier()

        # Decode: consecutive single-token steps on N=256 x H=16 heads, fresh
        # token inputs every step.
        log("decode")
        dec = gen.decode_batch(steps=args.decode_steps)
        Nd, Hd, dkd = dec.q.shape[1:]
        dvd = dec.v.shape[-1]
        dstate = torch.from_numpy(dec.state).to(dev)
        dtok = {k: torch.from_numpy(getattr(dec, k)).to(dev, torch.bfloat16 if k != "log_alpha" else torch.float32)
                for k in ("q", "k", "v", "b", "w", "log_alpha")}
        do = torch.empty((Nd, Hd, dvd), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            x = {k: v[i % args.decode_steps] for k, v in dtok.items()}
            gdr2.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], dstate, o=do)

        for i in range(3):
            dstep(i)
        barrier()
        dev_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.decode_steps + 1)]
        dev_ev[0].record(stream)
        for i in range(args.decode_steps):
            dstep(i)
            dev_ev[i + 1].record(stream)
        barrier()
        dper = [dev_ev[i].elapsed_time(dev_ev[i + 1]) for i in range(args.decode_steps)]
        # The same steps replayed from a CUDA graph (how a serving loop issues
        # them): back-to-back kernels without the host's per-launch gaps.
        dgraph = None
        try:
            graph = torch.cuda.CUDAGraph()
            gstream = torch.cuda.Stream(dev)
            gstream.wait_stream(stream)
            with torch.cuda.stream(gstream):
                dstep(0)  # (warm-up on the capture stream)
                with torch.cuda.graph(graph, stream=gstream):
                    for i in range(args.decode_steps):
                        dstep(i)
            stream.wait_stream(gstream)
            graph.replay()
            barrier()
            reps = []
            for _ in range(5):
                g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                g0.record(stream)
                graph.replay()
                g1.record(stream)
                barrier()
                reps.append(max_over_ranks(g0.elapsed_time(g1)) * 1e3 / args.decode_steps)
            dgraph = sorted(reps)[len(reps) // 2]
            del graph
        except RuntimeError as exc:  # capture unavailable: the eager per-step times stand
            log(f"decode graph replay skipped: {exc}")

        # End to end: pinned host inputs in, o and final states out, every step.
        e2e = None
        if not args.no_e2e:
            log("end to end")
            pinned = {k: x.pin_memory() for k, x in host.items()}
            o_h = torch.empty(t["o"].shape, dtype=t["o"].dtype).pin_memory()
            sf_h = torch.empty(t["sf"].shape, dtype=t["sf"].dtype).pin_memory()
            e2e_steps = max(3, min(args.steps, 20))

            # Two device buffer sets and three streams: step i+1's inputs go in
            # while step i computes and step i-1's outputs come out (PCIe is full
            # duplex), the way a data pipeline feeds the layer.
            def make_set():
                u = dict(t)
                for k in host:
                    u[k] = torch.empty_like(t[k])
                u["o"], u["sf"] = torch.empty_like(t["o"]), torch.empty_like(t["sf"])
                return u
            sets = [t, make_set()]
            outs_h = [(o_h, sf_h), (torch.empty_like(o_h).pin_memory(), torch.empty_like(sf_h).pin_memory())]
            s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
            used = [False, False]

            def e2e_step(i):
                x = i & 1
                u = sets[x]
                if used[x]:
                    s_in.wait_event(ev_comp[x])   # set x's inputs have been read
                with torch.cuda.stream(s_in):
                    for k in pinned:
                        u[k].copy_(pinned[k], non_blocking=True)
                ev_in[x].record(s_in)
                stream.wait_event(ev_in[x])
                if used[x]:
                    stream.wait_event(ev_out[x])  # set x's outputs have been copied out
                fwd(u)
                ev_comp[x].record(stream)
                s_out.wait_event(ev_comp[x])
                with torch.cuda.stream(s_out):
                    outs_h[x][0].copy_(u["o"], non_blocking=True)
                    outs_h[x][1].copy_(u["sf"], non_blocking=True)
                ev_out[x].record(s_out)
                used[x] = True

            for i in range(2):
                e2e_step(i)
            stream.wait_stream(s_out)
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(e2e_steps):
                e2e_step(i)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            e1.record(stream)
            barrier()
            e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
            h2d = sum(x.numel() * x.element_size() for x in pinned.values())
            d2h = t["o"].numel() * t["o"].element_size() + t["sf"].numel() * t["sf"].element_size()
            e2e = {"value": aggregate_throughput(inp.num_tokens, world, e2e_ms), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "ms_per_step": e2e_ms,
                   "pipeline": "pinned host buffers; two device buffer sets; inputs in, compute and "
                               "outputs out on three streams, overlapping across steps"}

        # Backward on the same batch (after everything above: it reuses o's dtype for d_o).
        bwd = None
        if not args.no_backward:
            log("backward")
            gen_do, gen_df = gen.cotangents(inp, seed=7)
            d_o = torch.from_numpy(gen_do).to(dev, t["o"].dtype)
            d_fin = torch.from_numpy(gen_df).to(dev)
            dcode = gdr2.GDR2_BF16 if inp.dtype == "bf16" else gdr2.GDR2_FP32
            bws = torch.empty(gdr2.bwd_workspace_size(B, T, H, d, d, N, dcode), dtype=torch.uint8,
                              device=dev)

            def bstep():
                return gdr2.chunk_bwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], d_o,
                                      t["s0"], d_fin, t["cu"], workspace=bws)

            for _ in range(3):
                bstep()
            barrier()
            bper = per_launch(bstep, args.backward_calls)
            bst = stats_ms(bper)
            bms = max_over_ranks(bst["mean_us"]) * 1e-3
            fl = bwd_flops(inp)
            bwd = {"kernels": "column sweeps + per-chunk rows (2 launches)", "calls": args.backward_calls,
                   **bst, "us_per_call": bms * 1e3, "tokens_per_s": inp.num_tokens / (bms * 1e-3),
                   "bound": "alu", "flops_per_call": fl, "achieved_tflops": fl / (bms * 1e-3) / 1e12,
                   "peak_tflops": SIMT_FP32_TFLOPS, "frac": fl / (bms * 1e-3) / 1e12 / SIMT_FP32_TFLOPS,
                   "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz"}

        # QED second erase direction on the same batch (a reading; token-serial CUDA-core path)
        qed = None
        if not args.no_qed:
            log("qed")
            lam = torch.full((H,), 0.1, dtype=torch.float32, device=dev)

            def qstep():
                return gdr2.qed_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["b"], t["w"], lam, None, 3,
                                    t["s0"], t["cu"], o=t["o"], final_state=t["sf"])

            qstep()
            barrier()
            qst = stats_ms(per_launch(qstep, 3))
            qms = max_over_ranks(qst["median_us"]) * 1e-3
            qed = {"kernel": "qed_fwd_kernel (token-serial, fp32 CUDA cores; strength 0.1, full arm)",
                   "calls": 3, **qst, "tokens_per_s": inp.num_tokens / (qms * 1e-3),
                   "note": "a reading of a page that does not print the update; parity unpinned"}

    ms_per_step = total_ms / args.steps
    value = aggregate_throughput(inp.num_tokens, world, ms_per_step)
    pst = stats_ms(per)
    fst = stats_ms(flushed)
    roof = chunk_roofline(inp, pst["median_us"], hbm_peak, tc_peak, peak_src)
    roof.update({"traffic": measured_traffic() if args.workload == "prefill" else None,
                 "kernel": "chunk forward (chunk_tc_kernel)", "us_per_launch": pst["median_us"], **pst,
                 "time_used": "median of the back-to-back launches"})
    dbytes = decode_bytes(Nd, Hd, dkd, dvd)
    dst = stats_ms(dper)
    d_us = dgraph if dgraph is not None else dst["median_us"]
    dgbs = dbytes / (d_us * 1e-6) / 1e9

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": label, "global_batch": world * B, "seq_len": T, "heads": H,
                   "d_k": d, "d_v": d, "tokens_per_rank": inp.num_tokens,
                   "parallelism": f"replicas x{world} (independent sequences per GPU)",
                   "l2": "inputs larger than L2 (no flush between the timed steps); "
                         "l2_flushed repeats the launch after a 256 MiB write"},
        "roofline": roof,
        "l2_flushed": {"launches": len(flushed), **fst,
                       "frac": chunk_roofline(inp, fst["median_us"], hbm_peak, tc_peak, peak_src)["frac"]},
        "decode": {"workload": "N=256 x H=16, d=128, fp32 state, bf16 tokens (fresh every step)",
                   "steps": args.decode_steps, "us_per_step": d_us, **dst,
                   "bytes_per_step": dbytes, "achieved_gbs": dgbs, "peak_gbs": hbm_peak,
                   "frac": dgbs / hbm_peak, "peak_source": peak_src,
                   "time_used": ("median over 5 replays of a CUDA graph of the steps, per step "
                                 "(mean_us .. p90_us: the same steps launched one by one)"
                                 if dgraph is not None else "median step, launched one by one")},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks.summary(),
    }
    line.update(extra)
    if e2e is not None:
        line["e2e"] = e2e
    if bwd is not None:
        line["backward"] = bwd
    if qed is not None:
        line["qed"] = qed
    if world == 1 and not args.no_cpu_baseline:
        log("cpu baseline")
        line["cpu_baseline"] = cpu_baseline(inp, label)
        if bwd is not None:
            bwd["cpu_baseline"] = cpu_backward_baseline(inp, gen_do, label)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

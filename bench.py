"""Benchmark of the Gated Delta Rule-2 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|long|varlen] [--no-cpu-baseline]

One step = one chunkwise forward (gdr2_chunk_fwd, bf16, H=16, d_k=d_v=128)
over the layer-shaped prefill batch B=4 x T=2048 (8,192 tokens). The line's
`value` is tokens/s over all ranks, timed with CUDA events on the launching
stream between barriers (max over ranks). In the same run:
  * roofline  -- algorithmic HBM bytes of one chunk-forward launch / its mean
                 CUDA-event duration, against the measured copy bandwidth;
  * decode    -- 64 consecutive gdr2_recurrent_step calls on N=256 x H=16
                 heads (fp32 state 256 MiB), achieved HBM GB/s per step;
  * e2e       -- the same tokens/s with pinned host inputs copied in and o and
                 the final states copied out inside every timed step;
  * backward  -- the gate-aware backward (gdr2_chunk_bwd) on the same batch:
                 time per call and its fp32 CUDA-core flops against the SIMT
                 fp32 peak (the kernels are ALU-bound);
  * cpu_baseline -- the fp64 oracle on the host cores (rank 0, N=1 only);
  * clocks    -- SM clock and throttle reasons sampled (NVML) while timing.
Inputs are larger than L2 (268 MB of token tensors vs 126 MB), so the steps
run back to back without an explicit flush.

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

    hbm_peak, _, peak_src = load_peaks()
    inp, label = workload(args.workload)
    tdt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(getattr(inp, k)).to(tdt if k != "log_alpha" else torch.float32)
            for k in ("q", "k", "v", "b", "w", "log_alpha")}
    dv_ = {k: x.to(dev) for k, x in host.items()}
    s0 = torch.from_numpy(inp.init_state).to(dev) if inp.init_state is not None else None
    cu = torch.from_numpy(inp.cu_seqlens.astype(np.int32)).to(dev) if inp.cu_seqlens is not None else None
    N = inp.num_seqs
    B, T, H, d = inp.q.shape
    o = torch.empty((B, T, H, d), dtype=tdt, device=dev)
    sf = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    dcode = gdr2.GDR2_BF16 if inp.dtype == "bf16" else gdr2.GDR2_FP32
    ws_bytes = gdr2.workspace_size(B, T, H, d, d, N, dcode)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    def step():
        gdr2.chunk_fwd(dv_["q"], dv_["k"], dv_["v"], dv_["log_alpha"], dv_["b"], dv_["w"], s0, cu,
                       o=o, final_state=sf, workspace=ws)

    # the chunk kernel; plus the order kernel of a packed batch, or the combine
    # and correction kernels of a segment split (few long sequences)
    launches_per_step = 1 + (1 if cu is not None and N > 1 else 0) + (2 if cu is None and ws_bytes > 0 else 0)
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
        total_ms = ev[0].elapsed_time(ev[-1])
        total_ms = max_over_ranks(total_ms)

        # Decode: 64 consecutive single-token steps on N=256 x H=16 heads.
        dec = gen.decode_batch(steps=4)
        Nd, Hd, dkd = dec.q.shape[1:]
        dvd = dec.v.shape[-1]
        dstate = torch.from_numpy(dec.state).to(dev)
        dtok = [{k: torch.from_numpy(getattr(dec, k)[i]).to(dev, torch.bfloat16 if k != "log_alpha"
                                                            else torch.float32)
                 for k in ("q", "k", "v", "b", "w", "log_alpha")} for i in range(4)]
        do = torch.empty((Nd, Hd, dvd), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            x = dtok[i % 4]
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

        # End to end: pinned host inputs in, o and final states out, every step.
        e2e = None
        if not args.no_e2e:
            pinned = {k: x.pin_memory() for k, x in host.items()}
            o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
            sf_h = torch.empty(sf.shape, dtype=sf.dtype).pin_memory()
            e2e_steps = max(3, min(args.steps, 20))

            def e2e_step():
                for k in pinned:
                    dv_[k].copy_(pinned[k], non_blocking=True)
                step()
                o_h.copy_(o, non_blocking=True)
                sf_h.copy_(sf, non_blocking=True)

            for _ in range(2):
                e2e_step()
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_step()
            e1.record(stream)
            barrier()
            e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
            h2d = sum(x.numel() * x.element_size() for x in pinned.values())
            d2h = o.numel() * o.element_size() + sf.numel() * sf.element_size()
            e2e = {"value": aggregate_throughput(inp.num_tokens, world, e2e_ms), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "ms_per_step": e2e_ms}

        # Backward on the same batch (after everything above: it reuses o's dtype for d_o).
        bwd = None
        if not args.no_backward:
            gen_do, gen_df = gen.cotangents(inp, seed=7)
            d_o = torch.from_numpy(gen_do).to(dev, tdt)
            d_fin = torch.from_numpy(gen_df).to(dev)
            bws = torch.empty(gdr2.bwd_workspace_size(B, T, H, d, d, N, dcode), dtype=torch.uint8,
                              device=dev)

            def bstep():
                return gdr2.chunk_bwd(dv_["q"], dv_["k"], dv_["v"], dv_["log_alpha"], dv_["b"],
                                      dv_["w"], d_o, s0, d_fin, cu, workspace=bws)

            for _ in range(3):
                bstep()
            barrier()
            bev = [torch.cuda.Event(enable_timing=True) for _ in range(args.backward_calls + 1)]
            bev[0].record(stream)
            for i in range(args.backward_calls):
                bstep()
                bev[i + 1].record(stream)
            barrier()
            bper = [bev[i].elapsed_time(bev[i + 1]) for i in range(args.backward_calls)]
            bms = max_over_ranks(statistics.mean(bper))
            fl = bwd_flops(inp)
            bwd = {"kernels": "column sweeps + per-chunk rows (2 launches)", "calls": args.backward_calls,
                   "us_per_call": bms * 1e3, "tokens_per_s": inp.num_tokens / (bms * 1e-3),
                   "bound": "alu", "flops_per_call": fl, "achieved_tflops": fl / (bms * 1e-3) / 1e12,
                   "peak_tflops": SIMT_FP32_TFLOPS, "frac": fl / (bms * 1e-3) / 1e12 / SIMT_FP32_TFLOPS,
                   "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz"}

    ms_per_step = total_ms / args.steps
    value = aggregate_throughput(inp.num_tokens, world, ms_per_step)
    kern_ms = statistics.mean(per)
    nbytes = chunk_bytes(inp)
    achieved = nbytes / (kern_ms * 1e-3) / 1e9
    dbytes = decode_bytes(Nd, Hd, dkd, dvd)
    dmean = statistics.mean(dper)
    dgbs = dbytes / (dmean * 1e-3) / 1e9

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
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": measured_traffic() if args.workload == "prefill" else None,
                     "kernel": "chunk forward", "bytes_per_launch": nbytes,
                     "us_per_launch": kern_ms * 1e3, "peak_source": peak_src},
        "decode": {"workload": "N=256 x H=16, d=128, fp32 state, bf16 tokens",
                   "steps": args.decode_steps, "us_per_step": dmean * 1e3,
                   "bytes_per_step": dbytes, "achieved_gbs": dgbs, "peak_gbs": hbm_peak,
                   "frac": dgbs / hbm_peak, "peak_source": peak_src},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if bwd is not None:
        line["backward"] = bwd
    if world == 1 and not args.no_cpu_baseline:
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

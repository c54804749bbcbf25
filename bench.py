#!/usr/bin/env python
"""Benchmark: zigzag-sharded causal attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl zsa|reference]

A step is one pass of the whole hot path over one batch of synthetic input: the
forward (zsa_attn_fwd: zigzag schedule + forward kernel) and the backward
(zsa_attn_bwd: Delta preprocess, backward main kernel, dQ conversion), all D logical
shards in one launch each.  Throughput is algorithmic causal FLOPs per second:
forward 4*B*Hq*d*S(S+1)/2, backward 2.5x that.

--gpus N > 1 (launched with torchrun, one rank per GPU) runs the D-GPU realisation of the
same problem: rank q owns D/N of the logical zigzag shards, all-gathers K/V (NCCL) in
the shard-major order the kernels read, runs the forward and backward over its own
shards, and reduce-scatters dK/dV back to the owners; value is the whole problem's
FLOPs over the slowest rank's time (strong scaling).
--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
Prints ONE JSON line on rank 0.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "causal attn fwd+bwd TFLOP/s at 1 B200 and % of BF16 tensor peak"
L2_BYTES = 126 * 2**20

CONFIGS = {
    "tiny": dict(B=1, S=256, Hq=2, Hkv=2, d=64, D=2, seed=0, stress=0.0,
                 desc="tiny: B=1 S=256 Hq=Hkv=2 d=64 D=2"),
    "7b_mha": dict(B=1, S=16384, Hq=32, Hkv=32, d=128, D=8, seed=1, stress=0.0,
                   desc="7B-dense MHA: B=1 S=16384 Hq=Hkv=32 d=128 D=8"),
    "8b_gqa": dict(B=1, S=32768, Hq=32, Hkv=8, d=128, D=8, seed=2, stress=0.0,
                   desc="Llama-3.1-8B-style GQA: B=1 S=32768 Hq=32 Hkv=8 d=128 D=8"),
    "wide_gqa": dict(B=1, S=65536, Hq=24, Hkv=4, d=256, D=4, seed=3, stress=0.0,
                     desc="wide-head GQA: B=1 S=65536 Hq=24 Hkv=4 d=256 D=4"),
    "long": dict(B=1, S=131072, Hq=32, Hkv=8, d=128, D=16, seed=4, stress=0.001,
                 desc="long context: B=1 S=131072 Hq=32 Hkv=8 d=128 D=16, 0.1% Q/K rows x8"),
}
# The largest configuration that fits one GPU, and the one at which the throughput
# targets (S >= 32K) apply.
DEFAULT_CONFIG = "long"
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture of
# the current kernel at the configuration's full size (dram__bytes_read.sum +
# dram__bytes_write.sum, a one-pass capture; profiles/dram_traffic_bwd_main.md);
# configurations without a capture report null.
MEASURED_TRAFFIC = {
    ("long", "zsa_bwd_wide_kernel"): 18.58e9 + 9.84e9,
    ("8b_gqa", "zsa_bwd_wide_kernel"): 1.812251e9 + 0.949273e9,
    ("wide_gqa", "zsa_bwd_pair_kernel"): 35.15e9 + 20.32e9,
}
# Oracle sample: full fwd+bwd at a reduced sequence length (same B, heads, d, D).
CPU_SAMPLE_S = {"tiny": 256, "7b_mha": 1024, "8b_gqa": 1024, "wide_gqa": 512, "long": 2048}


def fwd_flops(c, S=None):
    S = c["S"] if S is None else S
    return 4.0 * c["B"] * c["Hq"] * c["d"] * S * (S + 1) / 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk["bf16_tflops"], pk.get("bf16_tflops_sustained"), pk["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def max_over_ranks(x, dist=None, device=None):
    """The slowest rank's value (timing rule: max over ranks); x itself on one rank."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step, world, ms_max):
    """Whole-job throughput: every rank's work per step over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_max * 1e-3) / 1e12


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out = self.proc.communicate(timeout=10)[0]
        except Exception:
            self.proc.kill()
            return None
        sm, smax, power, reasons = [], [], [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(c, name):
    """One bounded oracle step: full fwd + bwd at a reduced S. Returns (seconds, flops, desc)."""
    import oracle
    from sequence_sharded_causal_b200 import inputs
    S = CPU_SAMPLE_S[name]
    q_nat, k, v, do_nat, _ = inputs.make_inputs(c["B"], S, c["Hq"], c["Hkv"], c["d"], c["seed"])
    perm, _ = oracle.partition(S, c["D"])
    q = inputs.to_shard_major(q_nat, perm, c["D"])
    do = inputs.to_shard_major(do_nat, perm, c["D"])
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, c["D"])
    oracle.attn_bwd(q, k, v, do, c["D"])
    dt = time.perf_counter() - t0
    flops = 3.5 * fwd_flops(c, S)
    desc = (f"oracle full fwd+bwd at S={S} (B={c['B']}, Hq={c['Hq']}, Hkv={c['Hkv']}, "
            f"d={c['d']}, D={c['D']}), fp64")
    return dt, flops, desc


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ------------------------------------------------------------------ reference arm
def run_reference(args, c, name):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    oracle._load()
    for _ in range(args.warmup):
        oracle_sample(c, name)
    total_t, total_f, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        dt, fl, desc = oracle_sample(c, name)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    cores = host_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": c["desc"], "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def run_zsa(args, c, name):
    import torch
    import sequence_sharded_causal_b200 as zsa
    from sequence_sharded_causal_b200 import inputs

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    B, S, Hq, Hkv, d, D = (c[k] for k in ("B", "S", "Hq", "Hkv", "d", "D"))
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D, causal=True)
    perm = zsa.zsa_partition(problem, want_schedule=False)["perm"]
    # every rank draws the same problem and keeps its own rows
    q_nat, k, v, do_nat, _ = inputs.make_inputs(B, S, Hq, Hkv, d, c["seed"], c["stress"],
                                                device=dev)
    q = inputs.to_shard_major(q_nat, perm, D)
    do = inputs.to_shard_major(do_nat, perm, D)
    del q_nat, do_nat
    stream = torch.cuda.current_stream(dev)
    if world == 1:
        # one launch over all D shards, natural-order K/V (the gathered buffer)
        ws_f = torch.empty(zsa.zsa_workspace_bytes(problem, 0), dtype=torch.uint8, device=dev)
        ws_b = torch.empty(zsa.zsa_workspace_bytes(problem, 1), dtype=torch.uint8, device=dev)

        def make_set(q, k, v, do):
            """A step over one set of device buffers: (inputs, outputs, step)."""
            o = torch.empty_like(q)
            lse = torch.empty(D, B, Hq, S // D, dtype=torch.float32, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

            def run():
                zsa.zsa_attn_fwd(problem, q, k, v, o, lse, ws_f, stream=stream)
                zsa.zsa_attn_bwd(problem, q, k, v, o, lse, do, dq, dk, dv, ws_b, stream=stream)
            return (q, k, v, do), (o, lse, dq, dk, dv), run

        inputs_t, outputs_t, step = make_set(q, k, v, do)
        o = outputs_t[0]

        def second_set():
            return make_set(*(torch.empty_like(x) for x in inputs_t))

        def device_status():
            return zsa.zsa_device_status(ws_f) or zsa.zsa_device_status(ws_b)
    else:
        from sequence_sharded_causal_b200 import dist as zdist
        core = zdist.ShardedAttention(B, S, Hq, Hkv, d, D, rank, world, device=dev)
        s0, ns = core.shard_begin, core.shard_count
        q = q[s0:s0 + ns].contiguous()
        do = do[s0:s0 + ns].contiguous()
        k = inputs.to_shard_major(k, perm, D)[s0:s0 + ns].contiguous()   # the rank's own K/V rows
        v = inputs.to_shard_major(v, perm, D)[s0:s0 + ns].contiguous()
        torch.cuda.empty_cache()
        o, dq = torch.empty_like(q), torch.empty_like(q)
        dk, dv = torch.empty_like(k), torch.empty_like(v)
        lse = core.lse

        def step():
            core.forward(q, k, v, o, stream=stream)
            core.backward(q, o, do, dq, dk, dv, stream=stream)

        def device_status():
            return core.status()
        inputs_t, outputs_t = (q, k, v, do), (o, lse, dq, dk, dv)
        second_set = None      # lse lives in the core: one buffer set, copies not overlapped

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = device_status()
    if status != zsa.ZSA_OK:
        raise RuntimeError(f"device status after warm-up: {zsa.status_string(status)}")

    # per-step kernel events (forward kernel, backward preprocess / main / dQ convert)
    K = args.steps
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(4)] for _ in range(K)]
    for row in kev:
        for b_, e_ in row:
            b_.record(stream)
            e_.record(stream)
    torch.cuda.synchronize(dev)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)   # let the sampler start before the timed region
    e0.record(stream)
    for i in range(K):
        for which in range(4):
            zsa.zsa_trace_events(which, kev[i][which][0], kev[i][which][1])
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier()
    for which in range(4):
        zsa.zsa_trace_events(which, None, None)
    status = device_status()
    if status != zsa.ZSA_OK:
        raise RuntimeError(f"device status after timing: {zsa.status_string(status)}")
    ms = e0.elapsed_time(e1) / K
    kms = [statistics.mean(kev[i][w][0].elapsed_time(kev[i][w][1]) for i in range(K))
           for w in range(4)]
    ms = max_over_ranks(ms, dist, dev)

    # ---- end to end through the API with host buffers (copies inside the timed region)
    pin = dict(pin_memory=True)
    h_in = [torch.empty(x.shape, dtype=x.dtype, **pin) for x in inputs_t]
    for hsrc, dsrc in zip(h_in, inputs_t):
        hsrc.copy_(dsrc)
    h_out = [torch.empty(x.shape, dtype=x.dtype, **pin) for x in outputs_t]
    bi = sum(x.numel() * x.element_size() for x in h_in)
    bo = sum(x.numel() * x.element_size() for x in h_out)
    K2 = max(1, min(K, 10))
    # One GPU: two sets of device buffers and two copy streams, so step i+1's inputs go
    # up and step i-1's results come down while step i's kernels run (a set is reused
    # only after its previous step's kernels and read-back are done).  Several ranks:
    # one set (the core owns lse), copies in line with the kernels.
    sets = [(inputs_t, outputs_t, step)]
    if second_set is not None:
        sets.append(second_set())
    e2e_mode = ("double-buffered device sets; H2D of step i+1 and D2H of step i-1 on two "
                "copy streams overlap step i" if len(sets) == 2 else "serial: H2D, step, D2H")
    h2d_s = torch.cuda.Stream(dev)
    d2h_s = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_done, ev_out = [ev() for _ in range(K2)], [ev() for _ in range(K2)], [ev() for _ in range(K2)]
    barrier()
    torch.cuda.synchronize(dev)
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for i in range(K2):
        ins, outs, run = sets[i % len(sets)]
        h2d_s.wait_event(x0)
        if i >= len(sets):
            h2d_s.wait_event(ev_done[i - len(sets)])     # the set's last step has read it
        with torch.cuda.stream(h2d_s):
            for dst, src in zip(ins, h_in):
                dst.copy_(src, non_blocking=True)
        ev_in[i].record(h2d_s)
        stream.wait_event(ev_in[i])
        if i >= len(sets):
            stream.wait_event(ev_out[i - len(sets)])     # its results have been read back
        run()
        ev_done[i].record(stream)
        d2h_s.wait_event(ev_done[i])
        with torch.cuda.stream(d2h_s):
            for dst, src in zip(h_out, outs):
                dst.copy_(src, non_blocking=True)
        ev_out[i].record(d2h_s)
    stream.wait_event(ev_out[K2 - 1])
    x1.record(stream)
    torch.cuda.synchronize(dev)
    del sets
    e2e_ms = x0.elapsed_time(x1) / K2
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_sus, hbm, peak_src = load_peaks()
    ff = fwd_flops(c)
    bf = 2.5 * ff
    # every rank's share of the problem, summed, over the slowest rank's time
    value = job_tflops((ff + bf) / world, world, ms)
    # kernel figures are this rank's: its kernels do 1/world of the problem
    fwd_tf = ff / world / (kms[0] * 1e-3) / 1e12
    bwd_ms = kms[1] + kms[2] + kms[3]
    bwd_tf = bf / world / (bwd_ms * 1e-3) / 1e12
    main_tf = bf / world / (kms[2] * 1e-3) / 1e12
    # dominant kernel by time: forward kernel or backward main kernel
    if kms[2] >= kms[0]:
        dom, dom_tf = ("zsa_bwd_wide_kernel" if d <= 128 else "zsa_bwd_pair_kernel"), main_tf
    else:
        dom, dom_tf = "zsa_fwd_kernel", fwd_tf
    traffic = MEASURED_TRAFFIC.get((name, dom))
    # the two HBM-bound kernels: algorithmic bytes per launch over their event time
    pairs = B * S * Hq // world
    # read O, dO, lse; write -Delta, -lse log2(e), the zeroed dQacc
    pre_bytes = pairs * (2 * d * 2 + 4 + 4 + 4 + 4 * d)
    dqc_bytes = pairs * d * (4 + 2)                # read fp32 dQacc; write bf16 dQ
    hbm_kernels = {
        "bwd_pre": {"bytes": pre_bytes, "gbs": pre_bytes / (kms[1] * 1e-3) / 1e9,
                    "frac": pre_bytes / (kms[1] * 1e-3) / 1e9 / hbm},
        "dq_convert": {"bytes": dqc_bytes, "gbs": dqc_bytes / (kms[3] * 1e-3) / 1e9,
                       "frac": dqc_bytes / (kms[3] * 1e-3) / 1e9 / hbm},
        "peak_gbs": hbm, "peak_source": f"{peak_src} copy bandwidth"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if world > 1 else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": c["desc"], "B": B, "S": S, "Hq": Hq, "Hkv": Hkv, "d": d, "D": D,
                   "causal": True,
                   "parallelism": f"sp{world}: {D // world} zigzag shards per rank, NCCL "
                                  "all-gather K/V + reduce-scatter dK/dV" if world > 1 else "single",
                   "l2": f"inputs larger than L2 ({(q.numel() + k.numel() + v.numel() + do.numel()) * 2 / 2**20:.0f} MiB vs 126 MiB), no flush"},
        "pct_of_peak": 100.0 * value / world / peak,
        "kv_layout": "natural" if world == 1 else "shard-major (all-gather order)",
        "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
        "fwd_frac": fwd_tf / peak, "bwd_frac": bwd_tf / peak, "bwd_main_tflops": main_tf,
        "kernel_ms": {"fwd": kms[0], "bwd_pre": kms[1], "bwd_main": kms[2], "dq_convert": kms[3]},
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": dom_tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": dom_tf / peak, "peak_source": f"{peak_src} bf16 burst",
                     "frac_of_sustained": (dom_tf / peak_sus) if peak_sus else None,
                     "traffic": traffic},
        "e2e": {"value": job_tflops((ff + bf) / world, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "mode": e2e_mode},
        "hbm_kernels": hbm_kernels,
        "gpu_launches": 4 * K,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle._load()
        dt, fl, desc = oracle_sample(c, name)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(),
                                "kind": "oracle", "sample": desc, "seconds": dt}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ NEXT-row components
MODEL_HIDDEN = {"tiny": 128, "7b_mha": 4096, "8b_gqa": 4096, "wide_gqa": 5120, "long": 4096}


def _time_events(fn, steps, warmup, dev):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / steps


def _component_ring(args, c, zsa, dev, g, peak, hbm, peak_src):
    import torch
    B, S, Hq, Hkv, d, D = (c[k] for k in ("B", "S", "Hq", "Hkv", "d", "D"))
    bf = torch.bfloat16
    C = S // (2 * D)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    if args.component == "permute":
        q = torch.randn((B, S, Hq, d), generator=g, device=dev).to(bf)
        k = torch.randn((B, S, Hkv, d), generator=g, device=dev).to(bf)
        v = torch.randn((B, S, Hkv, d), generator=g, device=dev).to(bf)
        qs = torch.empty((D, B, S // D, Hq, d), dtype=bf, device=dev)
        ks = torch.empty((D, B, S // D, Hkv, d), dtype=bf, device=dev)
        vs = torch.empty_like(ks)

        def step():
            zsa.to_shard_major(q, D, out=qs)
            zsa.to_shard_major(k, D, out=ks)
            zsa.to_shard_major(v, D, out=vs)
        zsa.zsa_trace_events(zsa.ZSA_TRACE_PERMUTE, ev[0], ev[1])
        ms = _time_events(step, args.steps, args.warmup, dev)
        zsa.zsa_trace_events(zsa.ZSA_TRACE_PERMUTE, None, None)
        kms = ev[0].elapsed_time(ev[1])                 # the last V copy alone
        nbytes = 2 * 2 * B * S * (Hq + 2 * Hkv) * d
        gbs = nbytes / (ms * 1e-3) / 1e9
        k_gbs = 2 * 2 * B * S * Hkv * d / (kms * 1e-3) / 1e9
        return {"metric": "K5 natural -> zigzag shard-major permute GB/s at 1 B200", "value": gbs,
                "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": c["desc"] + ", Q, K and V to shard-major order"},
                "roofline": {"kernel": "zsa_permute_kernel", "bound": "hbm", "achieved": gbs,
                             "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "peak_source": f"{peak_src} copy bandwidth", "traffic": None,
                             "last_launch_gbs": k_gbs},
                "gpu_launches": 3 * args.steps}
    q = torch.randn((D, B, S // D, Hq, d), generator=g, device=dev).to(bf)
    k = torch.randn((B, S, Hkv, d), generator=g, device=dev).to(bf)
    v = torch.randn((B, S, Hkv, d), generator=g, device=dev).to(bf)
    o, lse = torch.empty_like(q), torch.empty((D, B, Hq, S // D), device=dev)
    o_p, lse_p = torch.empty_like(q), torch.empty_like(lse)
    problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
    ws = torch.empty(zsa.zsa_workspace_bytes(problem, 0), dtype=torch.uint8, device=dev)
    # the ring order of rank 0: its own chunks first
    chunks = []
    for s_ in range(D):
        chunks += [s_, 2 * D - 1 - s_]

    def step():
        for i, ch in enumerate(chunks):
            dst = (o, lse) if i == 0 else (o_p, lse_p)
            zsa.attn_fwd_block(q, k, v, D, ch * C, (ch + 1) * C, rows_per_batch=S,
                               row_offset=ch * C, workspace=ws, out=dst)
            if i > 0:
                zsa.zsa_attn_merge(problem, [o, o_p], [lse, lse_p], o, lse)
    zsa.zsa_trace_events(zsa.ZSA_TRACE_MERGE, ev[0], ev[1])
    ms = _time_events(step, args.steps, args.warmup, dev)
    zsa.zsa_trace_events(zsa.ZSA_TRACE_MERGE, None, None)
    if zsa.zsa_device_status(ws) != zsa.ZSA_OK:
        raise RuntimeError("key-block forward reported a timeout")
    flops = fwd_flops(c)
    tf = flops / (ms * 1e-3) / 1e12
    return {"metric": "ring-attention forward (key blocks + running merge) TFLOP/s at 1 B200",
            "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{c['desc']}: {2 * D} key blocks of C={C} positions, "
                                   f"{2 * D - 1} in-place merges"},
            "roofline": {"kernel": "zsa_fwd_kernel (key-block)", "bound": "tensor",
                         "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_source": f"{peak_src} bf16 burst", "traffic": None,
                         "last_merge_ms": ev[0].elapsed_time(ev[1])},
            "gpu_launches": (4 * D - 1) * args.steps}


def run_component(args, c, name):
    """One JSON line for a NEXT-row kernel on one GPU, at the configuration's sizes.

    merge: one ring step's running merge, (O, lse) <- merge((O, lse), (O_s, lse_s)) in
      place over the whole Q layout (HBM-bound: reads 2 x (2d + 4) and writes 2d + 4 bytes
      per (row, head)); partials are seeded N(0, 1) values with lse ~ N(0, 1).
    tsp_projection: one rank's D projection steps of the TSP attention layer (QKV from
      the packed shards, then the output projection's fp32 partials), the rank's tokens
      T = B*S/D, hidden = the model's width; the broadcast is local on one GPU.
    permute: K5, natural -> zigzag shard-major copies of Q, K and V (HBM-bound: each
      byte read and written once).
    ring_forward: the forward as ring attention computes it, on one GPU: every shard's
      queries against one zigzag chunk of K/V at a time (2D key-block launches), each
      partial merged into the running (O, lse) in place; TFLOP/s of the causal FLOPs.
    """
    import torch
    import sequence_sharded_causal_b200 as zsa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, S, Hq, Hkv, d, D = (c[k] for k in ("B", "S", "Hq", "Hkv", "d", "D"))
    peak, peak_sus, hbm, peak_src = load_peaks()
    g = torch.Generator(device=dev).manual_seed(c["seed"])
    if args.component in ("permute", "ring_forward"):
        line = _component_ring(args, c, zsa, dev, g, peak, hbm, peak_src)
    elif args.component == "merge":
        problem = zsa.make_problem(B, S, Hq, Hkv, d, D)
        shp, lshp = (D, B, S // D, Hq, d), (D, B, Hq, S // D)
        o = torch.randn(shp, generator=g, device=dev).to(torch.bfloat16)
        o_s = torch.randn(shp, generator=g, device=dev).to(torch.bfloat16)
        lse = torch.randn(lshp, generator=g, device=dev)
        lse_s = torch.randn(lshp, generator=g, device=dev)
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

        def step():
            zsa.zsa_attn_merge(problem, [o, o_s], [lse, lse_s], o, lse)
        zsa.zsa_trace_events(zsa.ZSA_TRACE_MERGE, ev[0], ev[1])
        ms = _time_events(step, args.steps, args.warmup, dev)
        kms = ev[0].elapsed_time(ev[1])
        zsa.zsa_trace_events(zsa.ZSA_TRACE_MERGE, None, None)
        pairs = B * S * Hq
        nbytes = pairs * (3 * (2 * d + 4))
        gbs = nbytes / (ms * 1e-3) / 1e9
        line = {"metric": "ring-attention (O, lse) merge GB/s at 1 B200", "value": gbs,
                "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 O / fp32 lse", "data": "synthetic",
                "config": {"workload": c["desc"] + ", running merge of 2 partials in place"},
                "roofline": {"kernel": "zsa_merge_kernel", "bound": "hbm", "achieved": gbs,
                             "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "peak_source": f"{peak_src} copy bandwidth", "traffic": None,
                             "last_launch_ms": kms},
                "gpu_launches": args.steps}
    else:
        from sequence_sharded_causal_b200 import dist as zdist
        hidden = MODEL_HIDDEN[name]
        T = B * S // D
        nq, nk, nv = zdist.qkv_columns(Hq, Hkv, d, D)
        bf = torch.bfloat16
        x = (torch.randn(T, hidden, generator=g, device=dev)).to(bf)
        o = (torch.randn(T, Hq * d, generator=g, device=dev)).to(bf)
        shards = [(torch.randn(hidden, nq + nk + nv, generator=g, device=dev) * 0.02).to(bf)
                  for _ in range(D)]
        wo = [(torch.randn(nq, hidden, generator=g, device=dev) * 0.02).to(bf) for _ in range(D)]
        q = torch.empty(T, Hq * d, dtype=bf, device=dev)
        k = torch.empty(T, Hkv * d, dtype=bf, device=dev)
        v = torch.empty_like(k)
        y32 = torch.empty(T, hidden, dtype=torch.float32, device=dev)
        ws = torch.empty(256, dtype=torch.uint8, device=dev)

        def step():
            for s_ in range(D):
                zsa.zsa_tsp_project(x, shards[s_], [(q[:, s_ * nq:], Hq * d, nq, 0),
                                                    (k[:, s_ * nk:], Hkv * d, nk, 0),
                                                    (v[:, s_ * nv:], Hkv * d, nv, 0)], ws)
            y32.zero_()
            for s_ in range(D):
                zsa.zsa_tsp_project(o[:, s_ * nq:], wo[s_], [(y32, hidden, hidden, 1)], ws,
                                    T=T, K=nq, N=hidden, ldx=Hq * d)
        ms = _time_events(step, args.steps, args.warmup, dev)
        if zsa.zsa_device_status(ws) != zsa.ZSA_OK:
            raise RuntimeError("projection GEMM reported a timeout")
        flops = 2.0 * T * hidden * (nq + nk + nv) * D + 2.0 * T * (Hq * d) * hidden
        tf = flops / (ms * 1e-3) / 1e12
        line = {"metric": "TSP attention-layer projections (one rank, D steps) TFLOP/s at 1 B200",
                "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"{c['desc']}: T={T} tokens per rank, hidden={hidden}, "
                                       f"{D} QKV steps (N={nq + nk + nv}) + {D} output steps "
                                       f"(K={nq}, fp32 accumulate)"},
                "roofline": {"kernel": "zsa_proj_gemm_kernel", "bound": "tensor", "achieved": tf,
                             "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                             "peak_source": f"{peak_src} bf16 burst", "traffic": None},
                "gpu_launches": 2 * D * args.steps}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="zsa", choices=("zsa", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--component", default="attention",
                    choices=("attention", "merge", "tsp_projection", "permute", "ring_forward"),
                    help="attention: the hot path (default); merge / tsp_projection / "
                         "permute / ring_forward: the ring-attention merge, the TSP "
                         "projection schedule, the K5 permute or a ring-attention forward "
                         "on one GPU")
    ap.add_argument("--seq", type=int, default=0,
                    help="run the configuration's heads, d and D at this sequence length "
                         "(profiling captures of a smaller case); 0 = the configuration's S")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    c = dict(CONFIGS[args.config])
    if args.seq:
        if args.seq % (2 * c["D"] * 128):
            ap.error(f"--seq must be a multiple of 2*D*128 = {2 * c['D'] * 128}")
        c["desc"] = c["desc"].replace(f"S={c['S']}", f"S={args.seq}") + " (reduced S)"
        c["S"] = args.seq
    _, world, _ = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, c, args.config)
    elif args.component != "attention":
        run_component(args, c, args.config)
    else:
        run_zsa(args, c, args.config)


if __name__ == "__main__":
    main()

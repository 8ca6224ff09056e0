"""Benchmark of the GDN token mixer on B200: prefill T=4096 and decode B=64.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdn|reference]

One step = one gdn_prefill over a Qwen3.8-shaped layer (B=1, T=4096, 16 key /
48 value heads x 128, chunk 64, bf16 inputs, zero initial state), which runs
every prefill stage of the mixer.  The decode entry point (64 sequences, one
token each, fresh bf16 inputs per step, states ~N(0, 0.02)) is timed over
1000 consecutive steps in the same run and reported under "decode"; K=2
draft-and-verify rounds (a verify pass, then a commit of a seeded accepted
prefix) on the same sequences are reported under "draft_verify".  The
layer's input and output projections (bf16 tensor-core GEMMs around the
mixer, synthetic weights) are timed at T=4096 and at 64 tokens and reported
under "projections", with cuBLAS on the same operands for context.  One
65536-token sequence on a GPU holding 6 of the 48 value heads is prefilled
with and without the sequence-parallel carry ("seq_parallel").

Inputs are synthetic (seeded numpy draws) and resident in HBM before timing.
Between timed prefill steps the inputs rotate over 3 sets (~540 MB, > 4x L2)
so no step reads its inputs from L2; the decode state alone is 201 MB.
Times are CUDA events on the launching stream; the dominant kernel's average
launch time comes from the library's own per-launch events.  Under torchrun
every rank runs its own replica (no data-path collective) and the slowest
rank's time is reported.  ``--impl reference`` times the float64 CPU oracle
on a bounded sample of the same workload on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_recurrence_deltanet_b200 import inputs as gi  # noqa: E402

METRIC = "GDN tokens/s (prefill T=4096, decode B=64) and % of HBM/tensor roofline"
PREFILL_WORKLOAD = "prefill_t4096"
DECODE_WORKLOAD = "decode_b64"
DECODE_STEPS = 1000
ROTATE = 3
DRAFT_ROUNDS = 200
# arithmetic of the prefill path: bf16 inputs; fp16 hi + lo tensor-core operands; fp32 accumulation and state
DTYPE = "bf16 in, fp16x2 MMA, fp32 acc/state"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ algorithmic traffic


def prefill_bytes(geo, lengths, zero_state: bool) -> int:
    """Bytes the prefill must move at minimum: every token's qkv, z, a, b in
    and o out (io dtype), each sequence's fp32 state written (and read unless
    it starts at zero), its conv history read and written, and the
    parameters read once."""
    io = geo.io_bytes
    T = int(sum(lengths))
    per_tok = (geo.conv_dim + geo.value_dim + 2 * geo.num_v_heads + geo.value_dim) * io
    state = geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4
    hist = (geo.conv_width - 1) * geo.conv_dim * io
    params = (geo.conv_dim * geo.conv_width + 2 * geo.num_v_heads + geo.head_v_dim) * 4
    n = len(lengths)
    return T * per_tok + n * state * (1 if zero_state else 2) + n * 2 * hist + params


def decode_bytes(geo, num_seqs: int) -> int:
    io = geo.io_bytes
    per_seq = (geo.conv_dim + geo.value_dim + 2 * geo.num_v_heads + geo.value_dim) * io \
        + 2 * geo.num_v_heads * geo.head_v_dim * geo.head_k_dim * 4 + 2 * (geo.conv_width - 1) * geo.conv_dim * io
    params = (geo.conv_dim * geo.conv_width + 2 * geo.num_v_heads + geo.head_v_dim) * 4
    return num_seqs * per_seq + params


def source_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "linear_attention_recurrence_deltanet_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, src_hash: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("source_hash") != src_hash:
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while
    active (reading only; no setting is changed)."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
             0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, torch_device: int):
        self.ok = False
        self.samples = []
        self.active = False
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            h = None
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                try:
                    pci = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus, getattr(props, "pci_device_id", 0))
                    h = nv.nvmlDeviceGetHandleByPciBusId(pci.encode())
                except Exception:
                    h = None
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(torch_device)
            self.nv, self.h = nv, h
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks
            self.err = str(e)
        self._stop = threading.Event()
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return f(self.h)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            if self.active:
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), self._reasons(),
                                         nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
                except Exception:
                    pass
            time.sleep(0.005)

    def summary(self):
        if not self.ok:
            return None
        self._stop.set()
        s = self.samples
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for _, r, _ in s:
            mask |= r
        reasons = sorted(n for b, n in self.NAMES.items() if mask & b and b != 0x1)
        return {"sm_mhz": statistics.median(x[0] for x in s), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(s), "power_w_max": round(max(x[2] for x in s), 1), "source": "nvml"}


# ------------------------------------------------------------------ ranks


def rank_ops(dist, device):
    """(barrier, max_over_ranks) for one process per GPU; with dist None, a
    single process.  The barrier also synchronises the local device."""
    import torch

    def barrier():
        if dist is not None:
            dist.barrier()
        if device.type == "cuda":
            torch.cuda.synchronize(device)

    def max_over_ranks(x: float) -> float:
        if dist is None:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank processes the same units
    per step (weak scaling) and the slowest rank's time counts."""
    return world * units_per_rank_step * steps / (max_ms / 1000.0)


# ------------------------------------------------------------------ oracle timing


def time_oracle(inp, tokens: int):
    """Wall time of the float64 oracle over the first `tokens` tokens of a
    single-sequence problem (all heads, all host cores)."""
    import oracle
    sl = slice(0, tokens)
    params = (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w)
    t0 = time.perf_counter()
    oracle.prefill(inp.geo, params, inp.f32("qkv")[sl], inp.f32("z")[sl], inp.f32("a")[sl], inp.f32("b")[sl],
                   [0, tokens], inp.f32("conv_state"), inp.state)
    return time.perf_counter() - t0


def cpu_baseline(inp, budget_s=8.0):
    import oracle
    cores = oracle.default_threads()
    probe = 128
    dt = time_oracle(inp, probe)
    tokens = int(min(inp.total_tokens, max(probe, budget_s / max(dt, 1e-6) * probe)))
    dt = time_oracle(inp, tokens)
    return {"value": round(tokens / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"float64 oracle, first {tokens} of the 4096 prefill tokens, all 48 value heads, "
                      f"{cores} threads, {dt:.2f} s wall"}


def run_reference(args, rank):
    if rank != 0:
        return 0
    w = gi.WORKLOADS[PREFILL_WORKLOAD]
    inp = gi.workload_inputs(PREFILL_WORKLOAD)
    import oracle
    cores = oracle.default_threads()
    # every step is the whole 4096-token prefill (all heads) unless the requested steps would take more than
    # about three minutes on the host cores; then each step is the leading part of it that fits
    per_token = time_oracle(inp, 256) / 256
    steps, warm = args.steps, args.warmup
    tokens = int(max(256, min(inp.total_tokens, 180.0 / max(1, steps + warm) / max(per_token, 1e-9))))
    for _ in range(warm):
        time_oracle(inp, tokens)
    t = 0.0
    for _ in range(steps):
        t += time_oracle(inp, tokens)
    value = tokens * steps / t
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": round(1000 * t / steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "GDN prefill, B=1, T=4096, 16 key / 48 value heads x 128, chunk 64, bf16 inputs",
                       "global_batch": 1, "seq_len": 4096, "chunk": w["chunks"][0], "parallelism": "none (CPU)"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": (f"the whole {tokens}-token prefill per step" if tokens == inp.total_tokens
                                        else f"the first {tokens} of the 4096 prefill tokens per step")
                                       + ", all 48 value heads"},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm


def run_gdn(args, rank, world, local_rank):
    import torch
    import linear_attention_recurrence_deltanet_b200 as gdn
    from linear_attention_recurrence_deltanet_b200.device import io_tensor

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    stream = torch.cuda.current_stream()
    pk = peaks()
    barrier, max_over_ranks = rank_ops(dist, torch.device("cuda", local_rank))

    # ---------------- prefill workload (B=1, T=4096)
    w = gi.WORKLOADS[PREFILL_WORKLOAD]
    inp = gi.workload_inputs(PREFILL_WORKLOAD)
    geo, C = inp.geo, (args.chunk or w["chunks"][0])
    cfg = gdn.make_config(geo)
    T = inp.total_tokens
    params = tuple(torch.from_numpy(np.ascontiguousarray(p)).cuda() for p in (inp.conv_w, inp.A_log, inp.dt_bias,
                                                                               inp.norm_w))
    cu_h = np.ascontiguousarray(inp.cu_seqlens, np.int32)
    cu_d = torch.from_numpy(cu_h).cuda()
    sets = []
    base = [io_tensor(x) for x in (inp.qkv, inp.z, inp.a, inp.b)]
    for r in range(ROTATE):
        sets.append(dict(qkv=base[0].clone(), z=base[1].clone(), a=base[2].clone(), b=base[3].clone(),
                         o=torch.empty((T, geo.value_dim), dtype=torch.bfloat16, device="cuda"),
                         conv=io_tensor(inp.conv_state), state=torch.zeros((1, geo.num_v_heads, 128, 128),
                                                                           dtype=torch.float32, device="cuda")))
    del base
    ws = torch.empty(gdn.prefill_workspace_size(cfg, T, 1, C) + 256, dtype=torch.uint8, device="cuda")
    flags = gdn.ZERO_INIT_STATE | (gdn.PREFILL_RECURRENT if args.recurrent else 0) | \
        (gdn.PREFILL_FUSED if args.fused else 0) | (gdn.PREFILL_AFFINE if args.affine else 0)

    def prefill(i):
        s = sets[i % ROTATE]
        gdn.prefill(cfg, params, s["qkv"], s["z"], s["a"], s["b"], cu_d, cu_h, C, flags, s["conv"], s["state"],
                    s["o"], ws, stream=stream)

    clocks = ClockSampler(local_rank)
    for i in range(args.warmup):
        prefill(i)
    barrier()
    gdn.profiler_reset()
    gdn.profiler_enable(True)
    gdn.launch_count_reset()
    clocks.active = True
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        prefill(i)
    ev1.record(stream)
    barrier()
    clocks.active = False
    launches = gdn.launch_count()
    gdn.profiler_enable(False)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1))
    per_kernel = {gdn.kernel_name(k): gdn.profiler_read(k) for k in range(gdn.K.COUNT)}
    # The mixer kernel(s) that ran.  The three-kernel chunked path is one
    # logical kernel: its roofline takes the prefill's algorithmic bytes over
    # the summed average launch times of its three stages.
    split_ids = (gdn.K.SPLIT_CONV, gdn.K.SPLIT_PREP, gdn.K.SPLIT_CHAIN)
    wy_ids = (gdn.K.WY_CONV, gdn.K.WY_PREP, gdn.K.WY_CHAIN)
    if per_kernel[gdn.kernel_name(gdn.K.WY_CHAIN)][0]:
        kids, kname, src = wy_ids, "wy_conv+wy_prep+wy_chain", source_hash("prefill_wy.cu")
    elif per_kernel[gdn.kernel_name(gdn.K.SPLIT_CHAIN)][0]:
        kids, kname, src = split_ids, "split_conv+split_prep+split_chain", source_hash("prefill_split.cu")
    elif args.recurrent:
        kids, kname, src = (gdn.K.PREFILL_RECURRENT,), "prefill_recurrent", source_hash("prefill_recurrent.cu")
    else:
        kids, kname, src = (gdn.K.PREFILL_CHUNKED,), "prefill_chunked", source_hash("prefill_chunked.cu")
    k_avg_ms = 0.0
    for k in kids:
        n_launch, k_ms = per_kernel[gdn.kernel_name(k)]
        k_avg_ms += k_ms / max(1, n_launch)
    k_avg_ms = max_over_ranks(k_avg_ms)
    ms_per_step = ms_total / args.steps
    value = whole_job_rate(world, T, args.steps, ms_total)
    pbytes = prefill_bytes(geo, [T], zero_state=True)
    roof_p = {"bound": "hbm", "achieved": round(pbytes / (k_avg_ms / 1000.0) / 1e9, 1), "peak": pk["hbm"],
              "unit": "GB/s", "frac": round(pbytes / (k_avg_ms / 1000.0) / 1e9 / pk["hbm"], 4),
              "traffic": measured_traffic(kname + ":" + PREFILL_WORKLOAD, src), "kernel": kname,
              "kernel_ms": round(k_avg_ms, 5), "algorithmic_bytes": pbytes, "peak_source": pk["src"]}
    kernel_share = {k: {"launches": v[0], "ms": round(v[1], 3)} for k, v in per_kernel.items() if v[0]}

    # ---------------- end to end: pinned host inputs -> device -> prefill -> host output
    # Every step copies its inputs from pinned host memory and reads its output back.  Three streams pipeline
    # the steps (upload of step i+1 and download of step i-1 beside the prefill of step i) over two device
    # buffer sets; events order each buffer's reuse.
    e2e_steps = max(3, min(args.steps, 20))
    pin = {k: sets[0][k].cpu().pin_memory() for k in ("qkv", "z", "a", "b")}
    o_host = [torch.empty_like(sets[0]["o"], device="cpu").pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = o_host[0].numel() * o_host[0].element_size()
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    up_done = [torch.cuda.Event() for _ in range(2)]
    run_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        s = sets[b]
        with torch.cuda.stream(s_up):
            if used[b]:
                s_up.wait_event(run_done[b])  # the prefill of step i-2 has read this set
            for k in ("qkv", "z", "a", "b"):
                s[k].copy_(pin[k], non_blocking=True)
            up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        if used[b]:
            stream.wait_event(down_done[b])  # step i-2's output has left
        gdn.prefill(cfg, params, s["qkv"], s["z"], s["a"], s["b"], cu_d, cu_h, C, flags, s["conv"], s["state"],
                    s["o"], ws, stream=stream)
        run_done[b].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(run_done[b])
            o_host[b].copy_(s["o"], non_blocking=True)
            down_done[b].record(s_down)
        used[b] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    ev_a = torch.cuda.Event(enable_timing=True)
    ev_b = torch.cuda.Event(enable_timing=True)
    ev_a.record(s_up)
    for i in range(e2e_steps):
        e2e_step(i)
    s_down.wait_event(run_done[(e2e_steps - 1) % 2])
    ev_b.record(s_down)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(ev_a.elapsed_time(ev_b)) / e2e_steps
    e2e = {"value": round(whole_job_rate(world, T, 1, e2e_ms), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
           "overlap": "upload, prefill and download of consecutive steps on three streams (two buffer sets)"}
    del sets, pin
    torch.cuda.empty_cache()

    # ---------------- decode workload (64 sequences, 1000 steps)
    wd = gi.WORKLOADS[DECODE_WORKLOAD]
    gd, seed, N = wd["geo"], wd["seed"], 64
    dparams = tuple(torch.from_numpy(np.ascontiguousarray(p)).cuda() for p in gi.make_params(gd, seed))
    conv0, st0 = gi.make_initial_state(gd, N, seed, zero=False)
    conv = io_tensor(conv0)
    st = torch.from_numpy(st0).cuda()
    dsteps = args.decode_steps
    toks = [gi.make_decode_step_tokens(gd, N, seed, s) for s in range(dsteps)]
    dq = torch.stack([io_tensor(t[0]) for t in toks])
    dz = torch.stack([io_tensor(t[1]) for t in toks])
    da = torch.stack([io_tensor(t[2]) for t in toks])
    db = torch.stack([io_tensor(t[3]) for t in toks])
    del toks
    do = torch.empty((N, gd.value_dim), dtype=torch.bfloat16, device="cuda")
    for s in range(min(20, dsteps)):  # warm-up on the first steps' inputs, then restart from the initial state
        gdn.decode_step(cfg, dparams, dq[s], dz[s], da[s], db[s], N, conv, st, do, stream=stream)
    conv.copy_(io_tensor(conv0))
    st.copy_(torch.from_numpy(st0))
    barrier()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(dsteps + 1)]
    gdn.profiler_reset()
    gdn.profiler_enable(True)
    clocks.active = True
    evs[0].record(stream)
    for s in range(dsteps):
        gdn.decode_step(cfg, dparams, dq[s], dz[s], da[s], db[s], N, conv, st, do, stream=stream)
        evs[s + 1].record(stream)
    barrier()
    clocks.active = False
    gdn.profiler_enable(False)
    step_ms = [evs[s].elapsed_time(evs[s + 1]) for s in range(dsteps)]
    dn, dms = gdn.profiler_read(gdn.K.DECODE)
    d_kernel_ms = max_over_ranks(dms / max(1, dn))
    d_mean = max_over_ranks(sum(step_ms) / dsteps)
    dbytes = decode_bytes(gd, N)
    roof_d = {"bound": "hbm", "achieved": round(dbytes / (d_kernel_ms / 1000.0) / 1e9, 1), "peak": pk["hbm"],
              "unit": "GB/s", "frac": round(dbytes / (d_kernel_ms / 1000.0) / 1e9 / pk["hbm"], 4),
              "traffic": measured_traffic("decode:" + DECODE_WORKLOAD, source_hash("decode.cu")), "kernel": "decode",
              "kernel_ms": round(d_kernel_ms, 5), "algorithmic_bytes": dbytes, "peak_source": pk["src"]}
    decode = {"value": round(whole_job_rate(world, N, 1, d_mean), 1), "unit": "tokens/s", "ms_per_step": round(d_mean, 5),
              "median_ms": round(statistics.median(step_ms), 5), "steps": dsteps, "num_seqs": N, "roofline": roof_d,
              "workload": "GDN decode, 64 sequences x 1 token, 16 key / 48 value heads x 128, bf16 inputs, "
                          "fp32 states ~N(0,0.02), fresh inputs every step",
              "cpu_baseline": (oracle_decode_sample(gd, seed, N, conv0, st0)
                               if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None)}

    # ---------------- K=2 draft-and-verify rounds on the same sequences: a verify pass over both tokens, then a
    # commit of each sequence's accepted prefix (1 or 2 tokens, seeded); accepted tokens/s is the rate
    K = 2
    rounds = max(1, min(DRAFT_ROUNDS, dsteps // K))
    mq, mz, ma, mb = (x[:rounds * K].view(rounds, K, *x.shape[1:]).transpose(1, 2).contiguous()
                      for x in (dq, dz, da, db))
    del dq, dz, da, db
    acc_h = np.random.default_rng([seed, 7]).integers(1, K + 1, size=(rounds, N)).astype(np.int32)
    acc = torch.from_numpy(acc_h).cuda()
    mo = torch.empty((N, K, gd.value_dim), dtype=torch.bfloat16, device="cuda")

    def draft_round(r):
        gdn.decode_multi(cfg, dparams, mq[r], mz[r], ma[r], mb[r], N, K, False, None, conv, st, mo, stream=stream)
        vev[r].record(stream)
        gdn.decode_multi(cfg, dparams, mq[r], mz[r], ma[r], mb[r], N, K, True, acc[r], conv, st, mo, stream=stream)
        cev[r + 1].record(stream)

    vev = [torch.cuda.Event(enable_timing=True) for _ in range(rounds)]
    cev = [torch.cuda.Event(enable_timing=True) for _ in range(rounds + 1)]
    for r in range(min(3, rounds)):
        draft_round(r)
    conv.copy_(io_tensor(conv0))
    st.copy_(torch.from_numpy(st0))
    barrier()
    clocks.active = True
    cev[0].record(stream)
    for r in range(rounds):
        draft_round(r)
    barrier()
    clocks.active = False
    v_ms = max_over_ranks(sum(cev[r].elapsed_time(vev[r]) for r in range(rounds)) / rounds)
    c_ms = max_over_ranks(sum(vev[r].elapsed_time(cev[r + 1]) for r in range(rounds)) / rounds)
    r_ms = max_over_ranks(cev[0].elapsed_time(cev[rounds]) / rounds)
    state_b = N * gd.num_v_heads * gd.head_v_dim * gd.head_k_dim * 4
    tok_in = N * K * (gd.conv_dim + gd.value_dim + 2 * gd.num_v_heads) * gd.io_bytes
    hist_b = N * (gd.conv_width - 1) * gd.conv_dim * gd.io_bytes
    prm_b = (gd.conv_dim * gd.conv_width + 2 * gd.num_v_heads + gd.head_v_dim) * 4
    v_bytes = state_b + tok_in + hist_b + prm_b + N * K * gd.value_dim * gd.io_bytes
    c_bytes = 2 * state_b + tok_in + 2 * hist_b + prm_b + int(acc_h.mean() * N) * gd.value_dim * gd.io_bytes

    def roof(b, ms, name):
        return {"bound": "hbm", "achieved": round(b / (ms / 1000.0) / 1e9, 1), "peak": pk["hbm"], "unit": "GB/s",
                "frac": round(b / (ms / 1000.0) / 1e9 / pk["hbm"], 4), "traffic": None, "kernel": name,
                "kernel_ms": round(ms, 5), "algorithmic_bytes": int(b), "peak_source": pk["src"]}

    draft = {"value": round(whole_job_rate(world, float(acc_h.sum()) / rounds, 1, r_ms), 1),
             "unit": "accepted tokens/s", "ms_per_round": round(r_ms, 5), "rounds": rounds, "draft_tokens": K,
             "mean_accepted": round(float(acc_h.mean()), 4), "verify": roof(v_bytes, v_ms, "decode (verify, K=2)"),
             "commit": roof(c_bytes, c_ms, "decode (commit)"),
             "workload": "64 sequences, K=2 draft tokens per round, verify then commit of a seeded accepted "
                         "prefix (1 or 2 tokens), same geometry and states as the decode workload; "
                         "time between events on the launching stream"}
    del mq, mz, ma, mb

    proj = run_projections(gdn, torch, pk, stream, barrier, max_over_ranks, world, args.projection_reps)
    seqpar = run_seqpar(gdn, torch, pk, stream, barrier, max_over_ranks, world)
    slots = run_slots(gdn, torch, pk, stream, barrier, max_over_ranks, world)
    extra = {} if args.no_workloads else run_workloads(gdn, torch, pk, stream, barrier, max_over_ranks, world, rank,
                                                       clocks)

    clk = clocks.summary()
    cpu = cpu_baseline(inp) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if rank == 0:
        # the long blocks first, so that a tail of the line keeps the per-workload summaries
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
            "config": {"workload": f"GDN prefill, B=1, T=4096, 16 key / 48 value heads x 128, chunk {C}, bf16 inputs, "
                                   "fp32 state from zero", "global_batch": world, "seq_len": T, "chunk": C,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs rotate over {ROTATE} sets (> 4x L2) between steps"},
            "projections": proj, "seq_parallel": seqpar, "slots": slots, "kernels": kernel_share,
            "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu, "e2e": e2e,
            "roofline": roof_p,
            **extra,
            "draft_verify": draft, "decode": decode,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def oracle_decode_sample(geo, seed, N, conv0, st0, steps=5):
    """The float64 oracle, as it stands, on the first `steps` decode steps of
    the decode workload (all sequences and value heads, all host cores): the
    per-step time beside the GPU's."""
    import oracle
    params = gi.make_params(geo, seed)
    hist, state = conv0, st0
    times = []
    for s in range(steps):
        q, z, a, b = (gi.f32_from_bf16_bits(t) for t in gi.make_decode_step_tokens(geo, N, seed, s))
        t0 = time.perf_counter()
        _, state, hist = oracle.decode_step(geo, params, q, z, a, b, hist, state)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    cores = oracle.default_threads()
    return {"value": round(N / med, 2), "unit": "tokens/s", "ms_per_step": round(1000 * med, 2), "cores": cores,
            "kind": "oracle", "sample": f"float64 oracle, the first {steps} of the decode workload's steps ({N} "
                                       f"sequences, all {geo.num_v_heads} value heads), median step, {cores} threads"}


def oracle_sample(inp, budget_s=5.0):
    """The float64 oracle, as it stands, on a bounded sample of a workload:
    the leading tokens of the packed stream with their true sequence
    boundaries and starting states, all value heads, all host cores."""
    import oracle
    cu = np.asarray(inp.cu_seqlens, np.int64)
    params = (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w)

    def run(tokens):
        n_used = int(np.searchsorted(cu, tokens, side="left"))  # sequences that start before `tokens`
        cu_s = np.minimum(cu[:n_used + 1], tokens).astype(np.int32)
        cu_s[-1] = tokens
        sl = slice(0, tokens)
        t0 = time.perf_counter()
        oracle.prefill(inp.geo, params, inp.f32("qkv")[sl], inp.f32("z")[sl], inp.f32("a")[sl], inp.f32("b")[sl],
                       cu_s, inp.f32("conv_state")[:n_used], inp.state[:n_used])
        return time.perf_counter() - t0, n_used

    probe = 128
    dt, _ = run(probe)
    tokens = int(min(inp.total_tokens, max(probe, budget_s / max(dt, 1e-6) * probe)))
    dt, n_used = run(tokens)
    cores = oracle.default_threads()
    return {"value": round(tokens / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"float64 oracle, first {tokens} of {inp.total_tokens} packed tokens ({n_used} sequence(s) "
                      f"started), all {inp.geo.num_v_heads} value heads, {cores} threads, {dt:.2f} s wall"}


def run_workloads(gdn, torch, pk, stream, barrier, max_over_ranks, world, rank, clocks, reps=3):
    """The long-context one-pass prefill (B=1, T=65536) and the packed varlen
    batch (16 sequences, lengths uniform in 1..8192) at chunk 16, 64 and 128,
    at the full 16 key / 48 value head geometry, each prefill timed alone with
    events on the launching stream (inputs > L2), with the oracle timed on a
    bounded sample of the same workload beside it (rank 0, one GPU)."""
    from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_tensor
    out = {}
    for name, tag in (("prefill_t65536", "long_context"), ("varlen_16", "varlen_16")):
        w = gi.WORKLOADS[name]
        inp = gi.workload_inputs(name)
        zero = w["zero_init"]
        flags0 = (gdn.ZERO_INIT_STATE | gdn.ZERO_INIT_CONV) if zero else 0
        res = {}
        for C in w["chunks"]:
            dp = DeviceProblem(inp, C)
            conv0, st0 = dp.conv_state.clone(), dp.state.clone()
            ms_all, per = [], {}
            for i in range(reps + 1):
                if not zero:
                    dp.conv_state.copy_(conv0)
                    dp.state.copy_(st0)
                barrier()
                gdn.profiler_reset()
                gdn.profiler_enable(True)
                clocks.active = i > 0
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                dp.prefill(flags0, stream=stream)
                b.record(stream)
                b.synchronize()
                clocks.active = False
                gdn.profiler_enable(False)
                if i > 0:  # the first run is a warm-up
                    ms_all.append(a.elapsed_time(b))
                    for k in range(gdn.K.COUNT):
                        nl, kms = gdn.profiler_read(k)
                        if nl:
                            per[gdn.kernel_name(k)] = per.get(gdn.kernel_name(k), 0.0) + kms / reps
            ms = max_over_ranks(sum(ms_all) / len(ms_all))
            nbytes = prefill_bytes(inp.geo, list(np.diff(inp.cu_seqlens)), zero_state=zero)
            gbs = nbytes / (ms / 1000.0) / 1e9
            res[f"chunk_{C}"] = {
                "ms": round(ms, 4), "value": round(world * inp.total_tokens / (ms / 1000.0), 1), "unit": "tokens/s",
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm"], "unit": "GB/s",
                             "frac": round(gbs / pk["hbm"], 4), "traffic": None, "algorithmic_bytes": nbytes,
                             "kernel": "whole prefill (every launch)", "peak_source": pk["src"]},
                "kernels_ms": {k: round(v, 4) for k, v in per.items()}}
            del dp, conv0, st0
            torch.cuda.empty_cache()
        lengths = [int(x) for x in np.diff(inp.cu_seqlens)]
        res["workload"] = (f"{len(lengths)} sequence(s), {inp.total_tokens} tokens"
                           + (f" (lengths {lengths})" if len(lengths) > 1 else "")
                           + ", 16 key / 48 value heads x 128, bf16 inputs, "
                           + ("zero initial states" if zero else "initial states ~N(0,0.02) and histories ~N(0,1)")
                           + "; time per whole prefill (every launch), inputs > L2")
        res["cpu_baseline"] = oracle_sample(inp) if (rank == 0 and world == 1) else None
        out[tag] = res
        del inp
    return out


def run_projections(gdn, torch, pk, stream, barrier, max_over_ranks, world, reps):
    """The layer's input and output projections (bf16 GEMMs on the tensor
    cores) at the prefill (T=4096) and decode (64 tokens) sizes, with
    synthetic weights.  Each launch is timed alone with events on the
    launching stream, after a write of 256 MB (> L2) that evicts its operands;
    torch.matmul (cuBLAS) on the same operands is timed the same way for
    context.  The prefill sizes are bound by the tensor cores (roofline against
    the measured bf16 peak), the decode sizes by streaming the weights from
    HBM (roofline against the measured copy bandwidth)."""
    geo = gi.QWEN_GEO
    hidden = gi.QWEN_HIDDEN
    cfg = gdn.make_config(geo)
    w_in_h, w_out_h = gi.make_projection_weights(geo, hidden, 5)
    bf = torch.bfloat16

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits)).view(bf).cuda()

    w_in, w_out = dev(w_in_h), dev(w_out_h)
    del w_in_h, w_out_h
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def timed(fn):
        for _ in range(3):
            fn()
        total = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            total += a.elapsed_time(b)
        return max_over_ranks(total / reps)

    out = {}
    for T, tag in ((4096, "prefill_t4096"), (64, "decode_b64")):
        x = dev(gi.make_hidden_states(T, hidden, 6))
        qkv = torch.empty((T, geo.conv_dim), dtype=bf, device="cuda")
        z = torch.empty((T, geo.value_dim), dtype=bf, device="cuda")
        a = torch.empty((T, geo.num_v_heads), dtype=bf, device="cuda")
        b = torch.empty((T, geo.num_v_heads), dtype=bf, device="cuda")
        o = dev(gi.make_hidden_states(T, geo.value_dim, 7))
        y = torch.empty((T, hidden), dtype=bf, device="cuda")
        y_in = torch.empty((T, w_in.shape[0]), dtype=bf, device="cuda")
        barrier()
        for name, fn, ref, (M, K, N) in (
                ("project_in", lambda: gdn.project_in(cfg, x, w_in, qkv, z, a, b, stream=stream),
                 lambda: torch.matmul(x, w_in.t(), out=y_in), (T, hidden, w_in.shape[0])),
                ("project_out", lambda: gdn.project_out(cfg, o, w_out, y, stream=stream),
                 lambda: torch.matmul(o, w_out.t(), out=y), (T, geo.value_dim, hidden))):
            ms = timed(fn)
            ms_ref = timed(ref)
            flops = 2.0 * M * N * K
            nbytes = 2.0 * (M * K + N * K + M * N)
            if T >= 256:
                achieved, peak, unit, bound = flops / (ms / 1000.0) / 1e12, pk["bf16"], "TFLOP/s", "tensor"
            else:
                achieved, peak, unit, bound = nbytes / (ms / 1000.0) / 1e9, pk["hbm"], "GB/s", "hbm"
            out[f"{name}:{tag}"] = {
                "shape": {"M": M, "K": K, "N": N}, "ms": round(ms, 5),
                "value": round(world * M / (ms / 1000.0), 1), "unit": "tokens/s",
                "roofline": {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
                             "frac": round(achieved / peak, 4),
                             "traffic": measured_traffic({("project_in", 4096): "gemm:project_in_t4096",
                                                          ("project_out", 64): "gemm:project_out_b64"}
                                                         .get((name, T), ""), source_hash("gemm.cu")),
                             "kernel": "gemm", "peak_source": pk["src"]},
                "tflops": round(flops / (ms / 1000.0) / 1e12, 1), "cublas_ms": round(ms_ref, 5),
                "vs_cublas": round(ms_ref / ms, 3)}
        del x, qkv, z, a, b, o, y, y_in
    del w_in, w_out, flush
    torch.cuda.empty_cache()
    out["workload"] = ("hidden 5120 -> qkv/z/a/b (16480 columns) and 6144 -> 5120, synthetic bf16 weights "
                       "~N(0, 1/fan_in); each launch timed alone after a 256 MB L2-evicting write; "
                       "cublas_ms: torch.matmul on the same operands, for context")
    return out


def run_seqpar(gdn, torch, pk, stream, barrier, max_over_ranks, world, reps=5):
    """One long sequence on a GPU that holds few heads: B=1, T=65536, 2 key /
    6 value heads x 128 (one eighth of the layer's heads, as on each of 8 GPUs
    sharding them), chunk 64, bf16, zero start.  gdn_prefill (the state carry
    along the sequence on 2 SMs per value head) against gdn_prefill_seqpar
    (the carry as a scan over segments; segment count from the SM count).
    Inputs (~270 MB) exceed L2; CUDA events on the launching stream."""
    from linear_attention_recurrence_deltanet_b200.device import DeviceProblem
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6)
    T = 65536
    inp = gi.make_prefill_inputs(geo, [T], seed=3, zero_init=True)
    dp = DeviceProblem(inp, 64)
    ws = torch.empty(gdn.prefill_seqpar_workspace_size(dp.cfg, T, 0), dtype=torch.uint8, device="cuda")
    used = [0]

    def plain():
        dp.prefill(gdn.ZERO_INIT_STATE, stream=stream)

    def segmented():
        used[0] = gdn.prefill_seqpar(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, T, 0, gdn.ZERO_INIT_STATE,
                                     dp.conv_state, dp.state, dp.o, ws, stream=stream)

    def timed(fn):
        for _ in range(3):
            fn()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        b.synchronize()
        return max_over_ranks(a.elapsed_time(b) / reps)

    nbytes = prefill_bytes(geo, [T], zero_state=True)
    out = {}
    for name, fn in (("prefill", plain), ("seqpar", segmented)):
        ms = timed(fn)
        gbs = nbytes / (ms / 1000.0) / 1e9
        out[name] = {"ms": round(ms, 4), "value": round(world * T / (ms / 1000.0), 1), "unit": "tokens/s",
                     "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm"], "unit": "GB/s",
                                  "frac": round(gbs / pk["hbm"], 4), "traffic": None, "algorithmic_bytes": nbytes,
                                  "peak_source": pk["src"]}}
    out["seqpar"]["segments"] = used[0]
    out["speedup"] = round(out["prefill"]["ms"] / out["seqpar"]["ms"], 3)
    out["workload"] = ("B=1, T=65536, 2 key / 6 value heads x 128 (an eighth of the layer's heads), chunk 64, "
                       "bf16 inputs, fp32 state from zero; time per whole prefill (all kernels)")
    del dp, ws
    torch.cuda.empty_cache()
    return out


def run_slots(gdn, torch, pk, stream, barrier, max_over_ranks, world, steps=50, reps=10):
    """Slot-indexed state pools (continuous batching): the states and conv
    histories of a 256-slot pool, 16 key / 48 value heads x 128, bf16 inputs.
    (1) Decode of 64 sequences whose states sit at seeded slots of the pool
    (gdn_decode_step_indexed), fresh inputs every step; (2) one mixed step,
    4 prefill sequences of 1024 tokens and 60 one-token decode rows packed in
    one gdn_prefill_indexed call at chunk 64.  The pool (805 MB of state)
    exceeds L2; CUDA events on the launching stream, and the library profiler
    for the decode kernel's own time."""
    from linear_attention_recurrence_deltanet_b200.device import io_tensor
    geo = gi.QWEN_GEO
    seed, N, P = 2, 64, 256
    cfg = gdn.make_config(geo)
    params = tuple(torch.from_numpy(np.ascontiguousarray(p)).cuda() for p in gi.make_params(geo, seed))
    conv0, st0 = gi.make_initial_state(geo, P, seed, zero=False)
    conv = io_tensor(conv0)
    st = torch.from_numpy(st0).cuda()
    del conv0, st0
    rng = np.random.default_rng([seed, 8])
    dslots = torch.from_numpy(rng.choice(P, size=N, replace=False).astype(np.int32)).cuda()
    toks = [gi.make_decode_step_tokens(geo, N, seed, s) for s in range(steps)]
    dq, dz, da, db = (torch.stack([io_tensor(t[i]) for t in toks]) for i in range(4))
    del toks
    o = torch.empty((N, geo.value_dim), dtype=torch.bfloat16, device="cuda")

    def dstep(s):
        gdn.decode_step_indexed(cfg, params, dq[s], dz[s], da[s], db[s], N, dslots, P, conv, st, o, stream=stream)

    for s in range(min(10, steps)):
        dstep(s)
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gdn.profiler_reset()
    gdn.profiler_enable(True)
    a.record(stream)
    for s in range(steps):
        dstep(s)
    b.record(stream)
    b.synchronize()
    gdn.profiler_enable(False)
    d_ms = max_over_ranks(a.elapsed_time(b) / steps)
    kn, kms = gdn.profiler_read(gdn.K.DECODE)
    k_ms = max_over_ranks(kms / max(1, kn))
    dbytes = decode_bytes(geo, N)
    out = {"decode_indexed": {
        "value": round(whole_job_rate(world, N, 1, d_ms), 1), "unit": "tokens/s", "ms_per_step": round(d_ms, 5),
        "steps": steps, "num_seqs": N, "num_slots": P,
        "roofline": {"bound": "hbm", "achieved": round(dbytes / (k_ms / 1000.0) / 1e9, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(dbytes / (k_ms / 1000.0) / 1e9 / pk["hbm"], 4), "traffic": None,
                     "kernel": "decode (indexed)", "kernel_ms": round(k_ms, 5), "algorithmic_bytes": dbytes,
                     "peak_source": pk["src"]}}}
    del dq, dz, da, db, o

    lens = [1024] * 4 + [1] * 60
    cu_h = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu_h[-1])
    qkv, z, av, bv = (io_tensor(x) for x in gi.make_tokens(geo, np.random.default_rng([seed, 9]), T))
    mslots = torch.from_numpy(rng.choice(P, size=len(lens), replace=False).astype(np.int32)).cuda()
    cu_d = torch.from_numpy(cu_h).cuda()
    ws = torch.empty(max(256, gdn.prefill_indexed_workspace_size(cfg, T, len(lens), 64)), dtype=torch.uint8,
                     device="cuda")
    mo = torch.empty((T, geo.value_dim), dtype=torch.bfloat16, device="cuda")

    def mixed():
        gdn.prefill_indexed(cfg, params, qkv, z, av, bv, cu_d, cu_h, mslots, P, 64, 0, conv, st, mo, ws,
                            stream=stream)

    for _ in range(3):
        mixed()
    barrier()
    a.record(stream)
    for _ in range(reps):
        mixed()
    b.record(stream)
    b.synchronize()
    m_ms = max_over_ranks(a.elapsed_time(b) / reps)
    mbytes = prefill_bytes(geo, lens, zero_state=False)
    gbs = mbytes / (m_ms / 1000.0) / 1e9
    out["mixed_batch"] = {
        "value": round(whole_job_rate(world, T, 1, m_ms), 1), "unit": "tokens/s", "ms_per_step": round(m_ms, 5),
        "tokens": T, "prefill_seqs": 4, "decode_rows": 60, "chunk": 64, "num_slots": P,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm"], "unit": "GB/s",
                     "frac": round(gbs / pk["hbm"], 4), "traffic": None, "algorithmic_bytes": mbytes,
                     "peak_source": pk["src"]}}
    out["workload"] = ("a pool of 256 state slots, 16 key / 48 value heads x 128, bf16 inputs, fp32 states "
                       "~N(0,0.02); decode: 64 sequences at seeded slots, 50 steps; mixed: 4 x 1024 prefill tokens "
                       "and 60 decode rows in one indexed prefill call, chunk 64 (time per call, all kernels)")
    del qkv, z, av, bv, mo, ws, conv, st
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["gdn", "reference"], default="gdn")
    ap.add_argument("--decode-steps", type=int, default=DECODE_STEPS)
    ap.add_argument("--recurrent", action="store_true", help="time the token-recurrent prefill kernel")
    ap.add_argument("--fused", action="store_true", help="time the single-kernel chunked prefill")
    ap.add_argument("--affine", action="store_true", help="time the affine three-kernel chunked prefill at chunk 64")
    ap.add_argument("--chunk", type=int, choices=[16, 32, 64, 128], default=0,
                    help="chunk size of the timed prefill (default: the workload's, 64; 16/32/128 run the affine path)")
    ap.add_argument("--no-workloads", action="store_true", help="skip the long-context and varlen workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--projection-reps", type=int, default=20, help="timed launches per projection shape")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    return run_gdn(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark of the packed joint-attention block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl reference]

One step is one pass of the whole path over one synthetic pack: pack metadata
(mf_pack_build), modulation vectors (mf_adaln_params) and the fused block
(mf_block_fwd: adaLN modulation, RoPE (Q in the attention's load prologue, K by
a pass), tcgen05 varlen attention with the gated residual epilogue). Inputs are resident in HBM when the timed region starts.

Metric: useful attention TFLOP/s of the whole step, where useful FLOPs are
4 * D * H * sum(n_s^2) over the real samples (the padding segment is computed but
not counted). Also reported: block tokens/s, the attention kernel alone against
the measured bf16 tensor peak (roofline), the end-to-end rate through host
buffers (e2e) and the CPU oracle on a bounded sample (cpu_baseline).

Multi-GPU: every rank runs its own replica pack (same shapes, its own seed); no
data moves between ranks. Timing is the max over ranks of the CUDA-event time.
Under torchrun the ranks come from the environment (RANK, WORLD_SIZE, ...);
``--gpus N`` without them starts N replica processes itself, rank r on GPU r.
``--impl reference`` times the CPU oracle (the only reference this method has)
on rank 0; other ranks exit without work.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from packgen import make_workload  # noqa: E402

DEFAULT_CONFIG = 5  # the largest single-GPU pack: 2048^2 image plus three 4:1 images
METRIC = "packed varlen attention useful TFLOP/s (% bf16 peak); block tokens/s at 1 B200"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REF_ROW_STRIDE = 32  # reference arm: rows sampled per step at most (a step near 0.7 s)
REF_BUDGET_S = 300.0  # reference arm: the whole run's oracle time, about
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.txt")
# the attention kernel's sources: the traffic summary applies while they are unchanged
ATTN_SRC = [os.path.join(ROOT, "resolution_packed_diffusion_b200", "csrc", f)
            for f in ("attn_fwd.cu", "mf_ptx.cuh", "mf_internal.h")]


# ----------------------------------------------------------------- helpers
def useful_flops(w) -> float:
    tot = 0
    for d in w.descs:
        if d.is_dummy:
            continue
        n = d.frames * d.grid_h * d.grid_w + d.n_text
        tot += n * n
    return 4.0 * w.D * w.H * tot


def real_tokens(w) -> int:
    return int(sum(d.frames * d.grid_h * d.grid_w + d.n_text for d in w.descs if not d.is_dummy))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def rank_seed(index: int, rank: int) -> int:
    """Seed of a rank's replica pack: rank 0 uses the workload's own seed."""
    return 1000 + index + 7919 * rank


def reduce_timing(ms: float, units: float, world: int):
    """(max time over ranks, summed units over ranks); plain values at world 1."""
    if world == 1:
        return ms, units
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def attn_traffic_bytes(T_full: int):
    """DRAM bytes per attention launch from the committed ncu summary, scaled
    to this pack, or None when the kernel source changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    fields = {}
    for line in open(TRAFFIC_FILE):
        if "=" in line and not line.startswith("#"):
            k, v = line.strip().split("=", 1)
            fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    for f in ATTN_SRC:
        h.update(open(f, "rb").read())
    sha = h.hexdigest()[:16]
    if fields.get("kernel_sha") != sha or "workload" not in fields:
        return None
    if fields.get("workload") != str(T_full):
        return None
    return float(fields["bytes_per_launch"])


class ClockSampler:
    """nvidia-smi sampled every 100 ms from the start of the warm-up to the end of
    the timed steps (the timed region alone is often shorter than a sample)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle
def oracle_sample_step(w, heads, row_stride):
    """One bounded oracle step on the workload: pack metadata, modulation
    vectors, and, for every ``row_stride``-th token row, adaLN plus RoPE,
    attention over the row's whole sample and the gated residual for ``heads``.
    Returns (seconds, useful FLOPs of the sampled rows)."""
    import oracle
    from packgen import bf16_bits_to_f32
    t0 = time.perf_counter()
    pack = oracle.pack_build(w.descs, w.rope_axes)
    mod = oracle.adaln_params(w.c, w.W, w.hid)
    rows = np.arange(0, w.T, row_stride)
    x = bf16_bits_to_f32(w.x_bits[rows])
    oracle.adaln_modulate(x, mod, pack["tok_sample"][rows], pack["tok_mod"][rows], w.eps)
    q = bf16_bits_to_f32(w.q_bits[:, heads])
    k = bf16_bits_to_f32(w.k_bits[:, heads])
    v = bf16_bits_to_f32(w.v_bits[:, heads])
    k_r = oracle.rope_apply(k, pack["pos_ids"], w.rope_axes, w.base)
    q_r = np.zeros(q.shape)
    q_r[rows] = oracle.rope_apply(q, pack["pos_ids"], w.rope_axes, w.base, rows=rows)
    o, _ = oracle.varlen_attention(q_r, k_r, v, pack["cu_seqlens"], rows=rows)
    cols = np.concatenate([np.arange(h * w.D, (h + 1) * w.D) for h in heads])
    oracle.gated_residual(x[:, cols], o, mod[..., cols], pack["tok_sample"][rows],
                          pack["tok_mod"][rows])
    dt = time.perf_counter() - t0
    cu = pack["cu_seqlens"]
    fl = 0.0
    for s, d in enumerate(w.descs):
        if d.is_dummy:
            continue
        n = int(cu[s + 1] - cu[s])
        n_rows = int(((rows >= cu[s]) & (rows < cu[s + 1])).sum())
        fl += 4.0 * w.D * len(heads) * n * n_rows
    return dt, fl


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        blas = [i for i in info if i.get("user_api") == "blas"]
        if blas:
            return int(blas[0]["num_threads"]), blas[0].get("internal_api", "blas")
    except Exception:
        pass
    return len(os.sched_getaffinity(0)), "unknown"


def cpu_baseline(w, budget_s=12.0):
    """The oracle as it stands, on a bounded sample of the same workload:
    adaLN on all rows and RoPE + attention + gated residual for as many heads as
    fit in about ``budget_s`` seconds; its throughput is the sample's useful
    FLOPs over the sample's time."""
    dt, fl = oracle_sample_step(w, [0], 1)
    n = int(max(1, min(w.H, budget_s / max(dt, 1e-3))))
    heads = list(range(n))
    if n > 1:
        dt, fl = oracle_sample_step(w, heads, 1)
    threads, api = cpu_threads()
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"{w.name}: pack metadata, modulation vectors, adaLN on every token "
                       f"row and, for {n} of {w.H} heads, RoPE + attention + gated residual; "
                       f"fp64 NumPy ({api}); {dt:.1f} s"),
            "seconds": dt}


def run_reference(args, rank):
    if rank != 0:
        return
    w = make_workload(args.config)
    # warm-up and timed steps, each a one-head sample of the workload; the
    # warm-up steps also size the sample (every stride-th row, the stride
    # doubled while the remaining steps would overrun the time budget)
    stride = REF_ROW_STRIDE
    for i in range(args.warmup):
        dt, _ = oracle_sample_step(w, [0], stride)
        left = args.warmup - 1 - i + args.steps
        while dt * left > REF_BUDGET_S and stride < w.T:  # the next step re-measures
            stride *= 2
            dt *= 0.5
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample_step(w, [0], stride)
        times.append(dt)
        flops += fl
    total = sum(times)
    value = flops / total / 1e12
    threads, api = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": (f"each step: {w.name}, pack metadata, modulation vectors, "
                                    f"then for one token row in {stride}, adaLN and, "
                                    f"for head 0 of {w.H}, RoPE + attention over the row's "
                                    f"sample + gated residual; fp64 NumPy ({api})")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, args):
    return {"workload": w.name, "config_index": w.index, "T": w.T, "S": w.S, "H": w.H, "D": w.D,
            "hid": w.hid, "real_tokens": real_tokens(w),
            "samples": [list(d.as_tuple()) for d in w.descs], "rope_axes": w.rope_axes,
            "parallelism": f"replicas x{args.gpus}",
            "attention_cta_pairs": getattr(args, "cta_pair", None),
            "l2": ("inputs larger than L2: x, q, k, v total "
                   f"{4 * w.T * w.hid * 2 / 1e6:.0f} MB vs 126 MB L2; no flush")}


# ------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    import resolution_packed_diffusion_b200 as mf

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.config, seed=rank_seed(args.config, rank))
    T, H, D, hid, S = w.T, w.H, w.D, w.hid, w.S

    def dbf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    x, q, k, v = dbf16(w.x_bits), dbf16(w.q_bits), dbf16(w.k_bits), dbf16(w.v_bits)
    c = torch.from_numpy(w.c).to(dev)
    Wm = torch.from_numpy(w.W).to(dev)
    cu_d = torch.empty(S + 1, dtype=torch.int32, device=dev)
    pos = torch.empty((T, 3), dtype=torch.int32, device=dev)
    ts = torch.empty(T, dtype=torch.int32, device=dev)
    tm = torch.empty(T, dtype=torch.uint8, device=dev)
    mod = torch.empty((S, 2, 3, hid), dtype=torch.float32, device=dev)
    x_mod = torch.empty_like(x)
    y = torch.empty_like(x)
    ws_bytes = mf.mf_workspace_size(T, H, D, 1)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(bx=x, bq=q, bk=k, bv=v, bc=c, bW=Wm, bxm=x_mod, by=y):
        cu_h, _ = mf.mf_pack_build(w.descs, w.rope_axes, w.budget, cu_d, pos, ts, tm, stream)
        mf.mf_adaln_params(bc, bW, S, bc.shape[1], hid, mod, stream)
        mf.mf_block_fwd(bx, bq, bk, bv, mod, cu_d, cu_h, pos, ts, tm, S, H, D, w.rope_axes, w.base,
                        w.eps, bxm, by, ws, ws_bytes, stream)

    # pack ids, adaLN params, adaLN modulate, RoPE (cos, sin) table, RoPE pass over k,
    # attention (Q turned in its load prologue)
    launches_per_step = 6

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error during warm-up")
    # attention-kernel events, one pair per timed step
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in ev_a + ev_b:
        e.record(stream)  # creates the CUDA events before the library records them
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        mf.mf_set_attn_timing_events(ev_a[i], ev_b[i])
        step()
    t1.record(stream)
    mf.mf_set_attn_timing_events(None, None)
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error during the timed steps")

    flops = useful_flops(w)
    ms_step_local = ms_total / args.steps
    ms_step, flops_all = reduce_timing(ms_step_local, flops, world)
    tokens_all = reduce_timing(0.0, float(real_tokens(w)), world)[1]
    value = flops_all / (ms_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers. Every step copies
    # its inputs from pinned host memory and its outputs (y and x_mod) back. Two
    # device buffer sets and three streams (host-to-device copies, compute,
    # device-to-host copies) let step i's outputs travel back while step i+1's
    # inputs come in: PCIe carries both directions at once.
    pin = {n: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
           for n, a in (("x", w.x_bits), ("q", w.q_bits), ("k", w.k_bits), ("v", w.v_bits))}
    c_h = torch.from_numpy(w.c).pin_memory()
    W_h = torch.from_numpy(w.W).pin_memory()
    sets = [dict(x=x, q=q, k=k, v=v, c=c, W=Wm, x_mod=x_mod, y=y)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    out_h = [{n: torch.empty((T, hid), dtype=torch.int16).pin_memory() for n in ("y", "x_mod")}
             for _ in range(2)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of set b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # step on set b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # outputs of set b copied back
    for b in range(2):
        for e in (ev_done[b], ev_out[b]):
            e.record(stream)

    def e2e_step(i):
        b = i & 1
        bs = sets[b]
        s_in.wait_event(ev_done[b])  # the step that last read set b is finished
        with torch.cuda.stream(s_in):
            for n, t in pin.items():
                bs[n].view(torch.int16).copy_(t, non_blocking=True)
            bs["c"].copy_(c_h, non_blocking=True)
            bs["W"].copy_(W_h, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # set b's previous outputs are back on the host
        step(bs["x"], bs["q"], bs["k"], bs["v"], bs["c"], bs["W"], bs["x_mod"], bs["y"])
        ev_done[b].record(stream)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            for n in ("y", "x_mod"):
                out_h[b][n].copy_(bs[n].view(torch.int16), non_blocking=True)
        ev_out[b].record(s_out)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms, _ = reduce_timing(e0.elapsed_time(e1) / e2e_steps, 0.0, world)
    h2d = sum(t.numel() * t.element_size() for t in pin.values()) + \
        c_h.numel() * 4 + W_h.numel() * 4
    d2h = sum(t.numel() * t.element_size() for t in out_h[0].values())
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error during the end-to-end steps")
    if not all(np.array_equal(out_h[b][n].numpy(), out_h[0][n].numpy())
               for b in range(2) for n in ("y", "x_mod")):
        raise RuntimeError("end-to-end outputs differ between the two buffer sets")

    # ---- packed-CFG workloads: the guidance combine over the block output,
    # timed alone with the L2 flushed before every launch (its rows would
    # otherwise stay in the 126 MB L2 between launches)
    cfg_line = None
    if w.cfg_pairs:
        n_rows = sum(w.descs[c].frames * w.descs[c].grid_h * w.descs[c].grid_w
                     for c, _u in w.cfg_pairs)
        g_out = torch.empty((n_rows, hid), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = []
        for i in range(23):  # all enqueued back to back: no host gap before a launch
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            mf.mf_cfg_combine(y, w.descs, w.cfg_pairs, hid, 4.5, g_out, stream)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        times = [a.elapsed_time(b) for a, b in evs[3:]]
        if mf.mf_get_error(stream) != mf.MF_OK:
            raise RuntimeError("device error in the CFG combine")
        cfg_ms = float(np.median(times))
        cfg_bytes = 3 * n_rows * hid * 2  # both branches read, the guided rows written
        cfg_line = {"kernel": "cfg_combine_kernel", "ms": cfg_ms, "bytes": cfg_bytes,
                    "gbs": cfg_bytes / (cfg_ms * 1e-3) / 1e9, "w": 4.5,
                    "timing": "median of 20 launches, L2 flushed before each"}

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    attn_avg = float(np.mean(attn_ms))
    achieved = flops / (attn_avg * 1e-3) / 1e12
    # The attention kernel is timed inside the loop of whole block steps. When
    # that loop runs for a second or more, or the clocks show the power cap, the
    # GPU has settled under its power limit and the denominator is the measured
    # sustained bf16 rate; a shorter loop at full clocks takes the burst rate.
    # Both fractions are reported.
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    timed_s = ms_step * args.steps * 1e-3
    capped = "sw_power_cap" in (clk or {}).get("reasons", [])
    use_sustained = sustained != burst and (timed_s >= 1.0 or capped)
    peak = sustained if use_sustained else burst
    peak_why = (f"{peak_src} bf16_tflops_sustained (timed loop {timed_s:.2f} s"
                f"{', sw_power_cap active' if capped else ''})" if use_sustained else
                f"{peak_src} bf16_tflops (burst; timed loop {timed_s:.2f} s, no power cap seen)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, args),
        "block_tokens_per_s": tokens_all / (ms_step * 1e-3),
        "pct_bf16_peak": 100.0 * value / (burst * world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": attn_traffic_bytes(T),
                     "kernel": "varlen_attn_kernel<128, gated, 2D RoPE in the Q prologue>",
                     "peak_source": peak_why,
                     "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
                     "attn_ms": attn_avg},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": flops_all / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms},
        "clocks": clk,
    }
    if cfg_line is not None:
        cfg_line["frac"] = cfg_line["gbs"] / float(peaks["hbm_gbs"])
        line["cfg_combine"] = cfg_line
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def run_linear(args, rank, world, local_rank):
    """`--op linear`: the modality-specific linear layer as the block's fused
    Q, K, V projection (hid -> 3 hid) over the workload's pack."""
    import torch
    import resolution_packed_diffusion_b200 as mf

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.config, with_arrays=False, seed=rank_seed(args.config, rank))
    cu_h, T = mf.mf_pack_build(w.descs, w.rope_axes, w.budget)
    K, N = w.hid, 3 * w.hid
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(args.config, rank))
    x = torch.randn((T, K), device=dev, generator=g).to(torch.bfloat16)
    W = (torch.randn((2, N, K), device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    cu_d = torch.empty(w.S + 1, dtype=torch.int32, device=dev)
    pos = torch.empty((T, 3), dtype=torch.int32, device=dev)
    ts = torch.empty(T, dtype=torch.int32, device=dev)
    tm = torch.empty(T, dtype=torch.uint8, device=dev)
    mf.mf_pack_build(w.descs, w.rope_axes, w.budget, cu_d, pos, ts, tm)
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        mf.mf_modality_linear(x, W, tm, w.descs, K, N, out, 0, stream)
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        mf.mf_modality_linear(x, W, tm, w.descs, K, N, out, 0, stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error in the linear layer")
    flops = 2.0 * T * K * N
    ms_step, flops_all = reduce_timing(t0.elapsed_time(t1) / args.steps, flops, world)
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    print(json.dumps({
        "metric": "modality-specific linear (fused QKV projection) TFLOP/s", "op": "linear",
        "value": flops_all / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "config_index": args.config, "T": T, "K": K, "N": N,
                   "linear_cta_pairs": getattr(args, "linear_pair", None),
                   "l2": "x, W and out total %d MB vs 126 MB L2; no flush"
                         % ((T * K + 2 * N * K + T * N) * 2 >> 20)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None, "kernel": "modality_linear_kernel",
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": args.steps, "clocks": clk}), flush=True)


def run_mmdit(args, rank, world, local_rank):
    """`--op mmdit`: one whole NR-MMDiT block (adaLN, per-modality projections,
    RoPE + packed attention, gated residuals, GELU MLP of width 4 hid) over the
    workload's pack, random-init weights. `--op mmdit_bwd`: the block's backward
    (mf_mmdit_block_bwd: the forward recomputed, then every input, weight and
    modulation gradient) for a random loss gradient; its FLOPs count the
    recomputed forward and the backward (the linear layers' input and weight
    products, the attention backward's five products)."""
    bwd = args.op == "mmdit_bwd"
    import torch
    import resolution_packed_diffusion_b200 as mf

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.config, seed=rank_seed(args.config, rank))
    T, H, D, hid, S = w.T, w.H, w.D, w.hid, w.S
    F = 4 * hid
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(args.config, rank))

    def weight(n, k):
        return (torch.randn((2, n, k), device=dev, generator=g) / k ** 0.5).to(torch.bfloat16)

    Wq, Wk, Wv, Wo = (weight(hid, hid) for _ in range(4))
    Wup, Wdown = weight(F, hid), weight(hid, F)
    x = torch.from_numpy(np.ascontiguousarray(w.x_bits).view(np.int16)).to(dev).view(torch.bfloat16)
    c = torch.from_numpy(w.c).to(dev)
    Wm1 = torch.from_numpy(w.W).to(dev)
    Wm2 = (torch.randn(Wm1.shape, device=dev, generator=g) * 0.02).contiguous()
    mod_attn = torch.empty((S, 2, 3, hid), dtype=torch.float32, device=dev)
    mod_mlp = torch.empty_like(mod_attn)
    cu_d = torch.empty(S + 1, dtype=torch.int32, device=dev)
    pos = torch.empty((T, 3), dtype=torch.int32, device=dev)
    ts = torch.empty(T, dtype=torch.int32, device=dev)
    tm = torch.empty(T, dtype=torch.uint8, device=dev)
    y = torch.empty_like(x)
    if bwd:
        dy = torch.randn(x.shape, device=dev, generator=g).to(torch.bfloat16)
        grads = {n: torch.empty_like(W) for n, W in
                 (("q", Wq), ("k", Wk), ("v", Wv), ("o", Wo), ("up", Wup), ("down", Wdown))}
        dmod_attn, dmod_mlp = torch.empty_like(mod_attn), torch.empty_like(mod_mlp)
        ws_bytes = mf.mf_mmdit_bwd_workspace_size(T, S, H, D, F)
    else:
        ws_bytes = mf.mf_mmdit_workspace_size(T, H, D, F)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cu_h, _ = mf.mf_pack_build(w.descs, w.rope_axes, w.budget, cu_d, pos, ts, tm, stream)
        mf.mf_adaln_params(c, Wm1, S, c.shape[1], hid, mod_attn, stream)
        mf.mf_adaln_params(c, Wm2, S, c.shape[1], hid, mod_mlp, stream)
        if bwd:
            mf.mf_mmdit_block_bwd(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, w.descs,
                                  cu_d, cu_h, pos, ts, tm, S, H, D, F, w.rope_axes, w.base, w.eps,
                                  y, grads["q"], grads["k"], grads["v"], grads["o"], grads["up"],
                                  grads["down"], dmod_attn, dmod_mlp, ws, ws_bytes, stream)
        else:
            mf.mf_mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, w.descs, cu_d,
                                  cu_h, pos, ts, tm, S, H, D, F, w.rope_axes, w.base, w.eps, y,
                                  ws, ws_bytes, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error in the MMDiT block")
    gemm_flops = 2.0 * T * hid * hid * 4 + 2.0 * T * hid * F * 2
    flops = gemm_flops + useful_flops(w)
    if bwd:  # recomputed forward + input and weight products + the attention's five products
        flops = 3.0 * gemm_flops + 3.5 * useful_flops(w)
    ms_step, flops_all = reduce_timing(t0.elapsed_time(t1) / args.steps, flops, world)
    tokens_all = reduce_timing(0.0, float(real_tokens(w)), world)[1]
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    # kernels per step: pack ids and two modulation maps, then the block: 13 for
    # the forward (the attention's RoPE table and k pass included); for the
    # backward 12 (recomputed forward) + 12 (weight transposes) + 8 (MLP branch)
    # + 12 (attention branch) + 16 per modality with tokens (four input
    # transposes, six gradient transposes, six products), 6 zero fills otherwise
    mods_present = sum(1 for m in (0, 1) if any(
        (d.frames * d.grid_h * d.grid_w if m == 0 else d.n_text) > 0 for d in w.descs))
    launches = 3 + (44 + 16 * mods_present + 6 * (2 - mods_present) if bwd else 13)
    print(json.dumps({
        "metric": ("NR-MMDiT block backward TFLOP/s (recomputed forward + backward, GEMMs + "
                   "useful attention)" if bwd else
                   "NR-MMDiT block forward TFLOP/s (GEMMs + useful attention)"),
        "op": args.op,
        "value": flops_all / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic inputs, random-init weights",
        "config": {"workload": w.name, "config_index": args.config, "T": T, "H": H, "D": D,
                   "hid": hid, "mlp": F, "linear_cta_pairs": getattr(args, "linear_pair", None)},
        "block_tokens_per_s": tokens_all / (ms_step * 1e-3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": launches * args.steps, "clocks": clk}), flush=True)


def run_attn_bwd(args, rank, world, local_rank):
    """`--op attn_bwd`: the backward of the packed attention (mf_varlen_attn_bwd:
    row tables, the tcgen05 pass, dQ rounding) over the workload's pack, with O
    and the log-sum-exp from one forward before the timed region. Useful FLOPs:
    10 * D * H * sum(n_s^2) over the real samples (the five n x n x D products,
    S recomputed included)."""
    import torch
    import resolution_packed_diffusion_b200 as mf
    from packgen import draw_grad_bits

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.config, seed=rank_seed(args.config, rank))
    T, H, D, S = w.T, w.H, w.D, w.S

    def dbf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    q, k, v = dbf16(w.q_bits), dbf16(w.k_bits), dbf16(w.v_bits)
    d_o = dbf16(draw_grad_bits(rank_seed(args.config, rank), (T, H, D)))
    cu_h, _ = mf.mf_pack_build(w.descs, w.rope_axes, w.budget)
    cu_d = torch.from_numpy(np.ascontiguousarray(cu_h, dtype=np.int32)).to(dev)
    scale = 1.0 / D ** 0.5
    stream = torch.cuda.current_stream(dev)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    mf.mf_varlen_attn_fwd(q, k, v, cu_d, cu_h, S, H, D, scale, None, 2, 10000.0, o, lse, None, 0,
                          stream)
    dq, dk, dv = (torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    ws_bytes = mf.mf_attn_bwd_workspace_size(T, S, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step():
        mf.mf_varlen_attn_bwd(q, k, v, o, d_o, lse, cu_d, cu_h, S, H, D, scale, dq, dk, dv, ws,
                              ws_bytes, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error in the attention backward")
    flops = 2.5 * useful_flops(w)
    ms_step, flops_all = reduce_timing(t0.elapsed_time(t1) / args.steps, flops, world)
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    in_mb = (6 * T * H * D * 2 + T * H * D * 4) >> 20
    print(json.dumps({
        "metric": "packed varlen attention backward useful TFLOP/s", "op": "attn_bwd",
        "value": flops_all / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "config_index": args.config, "T": T, "H": H, "D": D,
                   "l2": "q, k, v, O, dO, dq/dk/dv and the fp32 dQ accumulator total %d MB vs "
                         "126 MB L2; no flush" % in_mb},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "attn_bwd_kernel (timed with its two small companion launches)",
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": 3 * args.steps, "clocks": clk}), flush=True)


def run_block_bwd(args, rank, world, local_rank):
    """`--op block_bwd`: the backward of the path block over the workload's pack,
    from upstream gradients dy (of y) and dx_mod (of x_mod): gate backward
    (dO, dgate), attention backward (dq, dk, dv of the rotated q, k from O and
    the log-sum-exp), RoPE backward, adaLN backward (dx = dy + the LayerNorm
    path, dshift, dscale) and the modulation map's backward (dc, dW). The
    forward state (rotated q and k, O, LSE) is
    computed once before the timed region. Useful FLOPs: the attention
    backward's 10 * D * H * sum(n_s^2) over the real samples."""
    import torch
    import resolution_packed_diffusion_b200 as mf
    from packgen import draw_grad_bits

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.config, seed=rank_seed(args.config, rank))
    T, H, D, S, hid = w.T, w.H, w.D, w.S, w.hid

    def dbf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    x = dbf16(w.x_bits.reshape(T, hid))
    q, k, v = dbf16(w.q_bits), dbf16(w.k_bits), dbf16(w.v_bits)
    seed = rank_seed(args.config, rank)
    dy = dbf16(draw_grad_bits(seed, (T, hid)))
    dxm = dbf16(draw_grad_bits(seed + 1, (T, hid)))
    cu_d = torch.empty(S + 1, dtype=torch.int32, device=dev)
    pos = torch.empty((T, 3), dtype=torch.int32, device=dev)
    ts = torch.empty(T, dtype=torch.int32, device=dev)
    tm = torch.empty(T, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    cu_h, _ = mf.mf_pack_build(w.descs, w.rope_axes, w.budget, cu_d, pos, ts, tm, stream)
    c = torch.from_numpy(w.c).to(dev)
    Wm = torch.from_numpy(w.W).to(dev)
    mod = torch.empty((S, 2, 3, hid), dtype=torch.float32, device=dev)
    mf.mf_adaln_params(c, Wm, S, c.shape[1], hid, mod, stream)
    scale = 1.0 / D ** 0.5
    q_r, k_r = torch.empty_like(q), torch.empty_like(k)
    mf.mf_rope_apply(q, k, pos, T, H, D, w.rope_axes, w.base, q_r, k_r, stream)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    mf.mf_varlen_attn_fwd(q_r, k_r, v, cu_d, cu_h, S, H, D, scale, None, w.rope_axes, w.base, o,
                          lse, None, 0, stream)
    d_o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    dq_r, dk_r, dv = (torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    dq, dk = torch.empty_like(dq_r), torch.empty_like(dk_r)
    dx = torch.empty_like(x)
    dmod = torch.empty((S, 2, 3, hid), dtype=torch.float32, device=dev)
    abw = mf.mf_attn_bwd_workspace_size(T, S, H, D)
    aws = torch.empty(abw, dtype=torch.uint8, device=dev)
    lbw = mf.mf_adaln_bwd_workspace_size(T)
    lws = torch.empty(max(lbw, 16), dtype=torch.uint8, device=dev)
    dc = torch.empty_like(c)
    dWm = torch.empty_like(Wm)

    def step():
        mf.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, hid, d_o, dmod, stream)
        mf.mf_varlen_attn_bwd(q_r, k_r, v, o, d_o, lse, cu_d, cu_h, S, H, D, scale, dq_r, dk_r, dv,
                              aws, abw, stream)
        mf.mf_rope_bwd(dq_r, dk_r, pos, T, H, D, w.rope_axes, w.base, dq, dk, stream)
        mf.mf_adaln_modulate_bwd(dxm, x, mod, ts, tm, dy, T, S, hid, w.eps, dx, dmod, lws, lbw,
                                 stream)
        mf.mf_adaln_params_bwd(dmod, c, Wm, S, c.shape[1], hid, dc, dWm, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error in the block backward")
    flops = 2.5 * useful_flops(w)
    ms_step, flops_all = reduce_timing(t0.elapsed_time(t1) / args.steps, flops, world)
    tokens_all = reduce_timing(0.0, float(real_tokens(w)), world)[1]
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    print(json.dumps({
        "metric": "path block backward useful TFLOP/s (attention backward FLOPs)",
        "op": "block_bwd",
        "value": flops_all / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "config_index": args.config, "T": T, "H": H, "D": D,
                   "hid": hid, "l2": "inputs and outputs far above the 126 MB L2; no flush"},
        "block_bwd_tokens_per_s": tokens_all / (ms_step * 1e-3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "whole backward step (attn_bwd_kernel dominant)",
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": 11 * args.steps, "clocks": clk}), flush=True)


def run_vae(args, rank, world, local_rank):
    """`--op vae_block`: one Mage-VAE conv block (SiLU(GroupNorm) -> 3x3 conv ->
    SiLU(GroupNorm) -> 3x3 conv + the input) at a decoder-stage size, seeded
    synthetic activations and random-init weights. FLOPs: the two convolutions,
    2 x 2 x 9 x C^2 per pixel."""
    import torch
    import resolution_packed_diffusion_b200 as mf
    from packgen import VAE_CONFIGS, make_vae_block

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    v = make_vae_block(args.vae_config, seed=rank_seed(len(VAE_CONFIGS), rank) + 17)
    N, H, W, C, G = v.N, v.H, v.W, v.C, v.G

    def dbf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    x, W1, W2 = dbf16(v.x_bits), dbf16(v.W1_bits), dbf16(v.W2_bits)
    f = {k: torch.from_numpy(getattr(v, k)).to(dev)
         for k in ("gamma1", "beta1", "gamma2", "beta2", "c1", "c2")}
    y = torch.empty_like(x)
    ws_bytes = mf.mf_vae_block_workspace_size(N, H, W, C, G)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mf.mf_vae_res_block(x, f["gamma1"], f["beta1"], W1, f["c1"], f["gamma2"], f["beta2"], W2,
                            f["c2"], N, H, W, C, G, v.eps, y, ws, ws_bytes, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop() if clocks else None
    if mf.mf_get_error(stream) != mf.MF_OK:
        raise RuntimeError("device error in the VAE block")
    flops = 4.0 * 9.0 * C * C * N * H * W
    ms_step, flops_all = reduce_timing(t0.elapsed_time(t1) / args.steps, flops, world)
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    act_mb = N * H * W * C * 2 / 1e6
    print(json.dumps({
        "metric": "Mage-VAE conv block TFLOP/s (two 3x3 convolutions)", "op": "vae_block",
        "value": flops_all / (ms_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic activations, random-init weights",
        "config": {"workload": f"VAE block {args.vae_config}", "N": N, "H": H, "W": W, "C": C,
                   "G": G, "conv_cta_pairs": getattr(args, "conv_pair", None),
                   "l2": "activations %.0f MB each, weights %.1f MB; no flush"
                   % (act_mb, 2 * C * 9 * C * 2 / 1e6)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "whole block (conv3x3_kernel dominant)",
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "gpu_launches": 8 * args.steps, "clocks": clk}), flush=True)


ARMS = {"block": "run_gpu", "linear": "run_linear", "mmdit": "run_mmdit", "mmdit_bwd": "run_mmdit",
        "attn_bwd": "run_attn_bwd", "block_bwd": "run_block_bwd", "vae_block": "run_vae"}


def run_rank(args, rank, world, local_rank, backend="nccl", arm=None):
    """One rank of the GPU arm: joins the process group when world > 1, runs
    the arm (``arm`` or the one ``--op`` names), leaves the group."""
    if arm is None and (getattr(args, "cta_pair", None) is not None
                        or getattr(args, "linear_pair", None) is not None
                        or getattr(args, "conv_pair", None) is not None):
        import torch
        import resolution_packed_diffusion_b200 as mf
        torch.cuda.set_device(local_rank)
        if getattr(args, "cta_pair", None) is not None:
            mf.mf_set_attn_cta_pair(args.cta_pair)
        if getattr(args, "linear_pair", None) is not None:
            mf.mf_set_linear_cta_pair(args.linear_pair)
        if getattr(args, "conv_pair", None) is not None:
            mf.mf_set_conv_cta_pair(args.conv_pair)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        (arm or globals()[ARMS[args.op]])(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_main(rank, world, port, args, backend, arm):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), LOCAL_WORLD_SIZE=str(world))
    run_rank(args, rank, world, rank, backend, arm)


def launch_replicas(args, n: int, backend: str = "nccl", arm=None):
    """``--gpus N`` outside torchrun: start N replica ranks in fresh (spawned)
    processes, rank r on GPU r, rendezvous on 127.0.0.1, and wait for all of
    them; a rank that fails makes the launch raise."""
    import torch.multiprocessing as mp
    mp.spawn(_replica_main, args=(n, _free_port(), args, backend, arm), nprocs=n, join=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="mf", choices=["mf", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cta-pair", type=int, default=None, choices=[0, 1],
                    help="attention on CTA pairs (1) or one CTA per SM (0); default: the "
                         "library's default")
    ap.add_argument("--linear-pair", type=int, default=None, choices=[0, 1],
                    help="linear layers on CTA pairs (1) or one CTA per SM (0); default: the "
                         "library's default")
    ap.add_argument("--conv-pair", type=int, default=None, choices=[0, 1],
                    help="VAE convolutions on CTA pairs (1) or one CTA per SM (0); default: "
                         "the library's default")
    ap.add_argument("--op", default="block", choices=sorted(ARMS),
                    help="block: the packed joint-attention block (the default line); "
                         "linear: the modality-specific linear layer as a QKV projection; "
                         "mmdit: one whole NR-MMDiT block around the path; "
                         "mmdit_bwd: that block's backward; "
                         "attn_bwd: the backward of the packed attention; "
                         "block_bwd: the backward of the whole path block; "
                         "vae_block: one Mage-VAE conv block")
    ap.add_argument("--vae-config", default="stage_1_8", choices=["tiny", "stage_1_8", "stage_1_4"],
                    help="shape of the --op vae_block workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")

    launched = "WORLD_SIZE" in os.environ
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if launched:
        args.gpus = world  # the launcher's rank count is what runs
    if args.impl == "reference":
        run_reference(args, rank)  # rank 0 alone; no GPU and no process group
        return
    if not launched and args.gpus > 1:
        launch_replicas(args, args.gpus)
        return
    run_rank(args, rank, world, local_rank)


if __name__ == "__main__":
    main()

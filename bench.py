"""Benchmark of the W4A4 / MXFP4 linear layer (MACaQ hot path) on B200.

Workload: the Llama-3-8B-shaped MLP up/gate projection, K = 4096, N = 14336, Hadamard block 32,
MXFP4 group 32, at M = 2048 tokens (the tensor-core-bound point of the M sweep). One step = one
pass of the whole online hot path on one batch: act_quant (scale + Hadamard + MXFP4 of X) followed
by the block-scaled GEMM against the prepared weights (prepared once, offline, outside the timed
region). The M sweep {1, 16, 128, 2048} is measured in the same run and reported under "sweep".

Metric: W4A4 layer TFLOPS (2 M N K per step / step time), with the GEMM's tensor-core roofline and
the act-quant kernel's HBM roofline. Inputs rotate through enough copies that every step reads
from HBM, not L2 (the copies together exceed twice the 126 MB L2).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs an independent replica (the layer has no cross-GPU step); the
value is the sum over ranks, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

K_DIM, N_DIM = 4096, 14336
M_MAIN = 2048
M_SWEEP = (1, 16, 128, 2048)
HAD_BLOCK = 32
L2_BYTES = 126 * 2 ** 20
LOAD_S = float(os.environ.get("MACAQ_BENCH_LOAD_S", "1.5"))  # warm replays before each timed replay (s)
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--M", type=int, default=M_MAIN)
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--profile", action="store_true", help="eager passes only, for ncu captures")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a4_mxfp4_quantized_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, M: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[f"{kernel}@M{M}"]
        return e["dram_bytes_per_launch"] if e.get("source_hash") == source_hash() else None
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


METRIC = "W4A4 layer TFLOPS (act_quant + block-scaled GEMM)"


def layer_config(M: int, world: int) -> dict:
    """The workload both arms report on."""
    return {"workload": f"llama3_8b_up_gate K={K_DIM} N={N_DIM} M={M} b={HAD_BLOCK}", "M": M, "N": N_DIM,
            "K": K_DIM, "had_block": HAD_BLOCK, "parallelism": f"replicas x{world}",
            "l2": f"inputs rotate over {copies_for(M)} copies (> 2x L2)"}


# ------------------------------------------------------------------------------------ ranks
def max_over_ranks(ms: float, dist_on: bool, device) -> float:
    """The slowest rank's time: every rank runs its own replica, the job ends with the last one."""
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    if dist_on:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank does flops_per_step per step, the step takes ms_per_step."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------------------------ our arm
def make_layer(M, dev, copies, plain=False):
    """The layer's device buffers. plain=True is the plain-MXFP4 comparator: no per-channel scale
    and no Hadamard (block 1), same kernels and shapes."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(M)
    W = c.W.to(dev)
    s = None if plain else c.s.to(dev)
    b = 1 if plain else HAD_BLOCK
    Xs = [c.X.to(dev)]
    Wqs, Wsfs = [], []
    Wq, Wsf, inv_s = mq.prep_weights(W, s, b)
    Wqs.append(Wq)
    Wsfs.append(Wsf)
    for _ in range(copies - 1):
        Wqs.append(Wq.clone())
        Wsfs.append(Wsf.clone())
        Xs.append(Xs[0].clone())
    del W
    Xq = [torch.empty(M, K_DIM // 2, dtype=torch.uint8, device=dev) for _ in range(copies)]
    Xsf = [torch.empty(mq.sf_bytes(M, K_DIM), dtype=torch.uint8, device=dev) for _ in range(copies)]
    Y = [torch.empty(M, N_DIM, dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    return dict(X=Xs, inv_s=inv_s, Wq=Wqs, Wsf=Wsfs, Xq=Xq, Xsf=Xsf, Y=Y, host_X=c.X, b=b)


def gemm_kernel_name(M):
    """The GEMM kernel the library picks for this layer (dense, K % 256 == 0, workspace given)."""
    if M <= 128:
        return "gemm_mxf4_skinny_kernel"
    return "gemm_mxf4_pair_kernel" if N_DIM % 256 == 0 else "gemm_mxf4_kernel"


def copies_for(M):
    per_copy = N_DIM * K_DIM * 0.53125 + M * K_DIM * (2 + 0.53125) + M * N_DIM * 2
    return max(2, int(np.ceil(2 * L2_BYTES / per_copy)))


def run_layer(mq, L, i, parts=("aq", "gemm")):
    if "fused" in parts:  # the layer in one call from bf16 X (quantizer inside the GEMM for M <= 16)
        mq.linear(L["X"][i], None, L["Wq"][i], L["Wsf"][i], mode=mq.A_BF16_FUSED, inv_s=L["inv_s"],
                  had_block=L["b"], Y=L["Y"][i])
    if "aq" in parts:
        mq.act_quant(L["X"][i], L["inv_s"], L["b"], Xq=L["Xq"][i], Xsf=L["Xsf"][i])
    if "gemm" in parts:
        mq.linear(L["Xq"][i], L["Xsf"][i], L["Wq"][i], L["Wsf"][i], Y=L["Y"][i])


def capture(mq, L, steps, ncopy, parts):
    """One CUDA graph holding `steps` passes (rotating over the input copies): replaying it times
    the kernels alone, without the per-call host overhead of the Python binding."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            run_layer(mq, L, i % ncopy, parts)
    return g


def replay_ms(g, stream):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def time_layer(M, steps, warmup, dev, dist_on, plain=False, fused=False):
    """Device time of `steps` layer passes (graph replay, rotating copies) and of each kernel alone.
    fused=True also times the one-call fused layer (returned as L["fused_ms"], per pass)."""
    import w4a4_mxfp4_quantized_b200 as mq

    ncopy = copies_for(M)
    L = make_layer(M, dev, ncopy, plain)
    for i in range(max(warmup, 1)):
        run_layer(mq, L, i % ncopy, ("aq", "gemm", "fused") if fused else ("aq", "gemm"))
    torch.cuda.synchronize(dev)
    g_pair = capture(mq, L, steps, ncopy, ("aq", "gemm"))
    g_aq = capture(mq, L, steps, ncopy, ("aq",))
    g_gemm = capture(mq, L, steps, ncopy, ("gemm",))
    stream = torch.cuda.current_stream(dev)
    for g in (g_pair, g_aq, g_gemm):  # warm replays
        g.replay()
    # keep the GPU under this load for a while before the timed replay, so the clock sampler
    # (200 ms period) records the clocks this workload runs at
    t_end = time.time() + LOAD_S
    while time.time() < t_end:
        g_pair.replay()
        torch.cuda.synchronize(dev)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    total_ms = replay_ms(g_pair, stream)
    if dist_on:
        torch.distributed.barrier()
    aq_ms = replay_ms(g_aq, stream) / steps
    gemm_ms = replay_ms(g_gemm, stream) / steps
    if fused:
        g_fused = capture(mq, L, steps, ncopy, ("fused",))
        g_fused.replay()
        L["fused_ms"] = replay_ms(g_fused, stream) / steps
        del g_fused
    status = mq.device_status()
    assert status == 0, f"device status {status}"
    del g_pair, g_aq, g_gemm
    return total_ms, aq_ms, gemm_ms, L


def time_graph(fn, steps, stream):
    """Device time per call of fn(i), i = 0..steps-1, captured in one graph and replayed."""
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            fn(i)
    g.replay()
    ms = replay_ms(g, stream) / steps
    del g
    return ms


def moe_section(dev, hbm, fp4_peak, steps=20):
    """The grouped path (MoE 30B-A3B gate/up: 128 experts, top-8 of T tokens, Zipf routing) at
    T = 64, 1024, 8192: grouped act_quant and grouped GEMM, each timed alone by graph replay.
    The weights (213 MB prepared) exceed L2 by themselves; X rotates over two copies."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    stream = torch.cuda.current_stream(dev)
    c0 = inputs.moe_30b_a3b(64, "gate_up")
    E, N, K = c0.W.shape
    Wd = c0.W.to(dev)
    Wq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
    Wsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device=dev)
    inv = torch.empty(E, K, dtype=torch.float32, device=dev)
    sd = c0.s.to(dev)
    for e in range(E):
        mq.prep_weights(Wd[e], sd[e], HAD_BLOCK, Wq=Wq[e], Wsf=Wsf[e], inv_s=inv[e])
    del Wd
    out = []
    for T in (64, 1024, 8192):
        c = inputs.moe_30b_a3b(T, "gate_up", draw_w=False)
        off = c.offsets.to(dev)
        rows = int(c.offsets[-1])
        counts = (c.offsets[1:] - c.offsets[:-1]).numpy()
        Xs = [c.X.to(dev), c.X.to(dev).clone()]
        Xq = [torch.empty(rows, K // 2, dtype=torch.uint8, device=dev) for _ in range(2)]
        Xsf = [torch.empty(mq.grouped_sf_bytes(rows, E, K), dtype=torch.uint8, device=dev) for _ in range(2)]
        Y = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
        aq = time_graph(lambda i: mq.act_quant(Xs[i % 2], inv, HAD_BLOCK, group_offsets=off, Xq=Xq[i % 2],
                                               Xsf=Xsf[i % 2]), steps, stream)
        gm = time_graph(lambda i: mq.grouped_linear(Xq[i % 2], Xsf[i % 2], off, Wq, Wsf, Y=Y), steps, stream)
        assert mq.device_status() == 0
        flops = 2.0 * N * K * rows
        g_bytes = int((counts > 0).sum()) * N * K * 0.53125 + rows * (0.53125 * K + 2 * N)
        a_bytes = rows * K * (2 + 0.5 + 1 / 32)
        out.append({"T": T, "rows": rows, "experts_used": int((counts > 0).sum()),
                    "grouped_gemm_us": gm * 1e3, "grouped_gemm_tflops": flops / (gm * 1e-3) / 1e12,
                    "grouped_gemm_gbs": g_bytes / (gm * 1e-3) / 1e9,
                    "grouped_gemm_frac_fp4_peak": flops / (gm * 1e-3) / 1e12 / fp4_peak,
                    "grouped_gemm_frac_hbm": g_bytes / (gm * 1e-3) / 1e9 / hbm,
                    "grouped_act_quant_us": aq * 1e3, "grouped_act_quant_gbs": a_bytes / (aq * 1e-3) / 1e9,
                    "grouped_act_quant_frac_hbm": a_bytes / (aq * 1e-3) / 1e9 / hbm})
        del Xs, Xq, Xsf, Y
    return {"workload": f"moe_30b_a3b gate/up E={E} top-8 K={K} N={N} b={HAD_BLOCK}", "points": out}


def weight_prep_section(dev, hbm, steps=10):
    """Offline weight preparation of the Llama-3-8B up/gate weights (bf16 in, codes + SF out)."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(1)
    W, s = c.W.to(dev), c.s.to(dev)
    Wq = torch.empty(N_DIM, K_DIM // 2, dtype=torch.uint8, device=dev)
    Wsf = torch.empty(mq.sf_bytes(N_DIM, K_DIM), dtype=torch.uint8, device=dev)
    inv = torch.empty(K_DIM, dtype=torch.float32, device=dev)
    ms = time_graph(lambda i: mq.prep_weights(W, s, HAD_BLOCK, Wq=Wq, Wsf=Wsf, inv_s=inv), steps,
                    torch.cuda.current_stream(dev))
    b = N_DIM * K_DIM * (2 + 0.5 + 1 / 32)
    return {"workload": f"llama3_8b_up_gate W [{N_DIM}, {K_DIM}] b={HAD_BLOCK}", "us": ms * 1e3,
            "gbs": b / (ms * 1e-3) / 1e9, "frac_hbm": b / (ms * 1e-3) / 1e9 / hbm}


def profile_mode(M, steps, warmup, dev):
    """Eager layer passes with no timing: the command the ncu captures run."""
    import w4a4_mxfp4_quantized_b200 as mq

    L = make_layer(M, dev, 2)
    for i in range(warmup + steps):
        run_layer(mq, L, i % 2)
    torch.cuda.synchronize(dev)
    assert mq.device_status() == 0


def time_e2e(M, steps, warmup, dev, L):
    """The same layer through the public API from pinned host X to host Y, copies included."""
    import w4a4_mxfp4_quantized_b200 as mq

    hX = L["host_X"].pin_memory()
    hY = torch.empty(M, N_DIM, dtype=torch.bfloat16).pin_memory()
    dX, dY = L["X"][0], L["Y"][0]
    stream = torch.cuda.current_stream(dev)

    def step():
        dX.copy_(hX, non_blocking=True)
        mq.act_quant(dX, L["inv_s"], HAD_BLOCK, Xq=L["Xq"][0], Xsf=L["Xsf"][0])
        mq.linear(L["Xq"][0], L["Xsf"][0], L["Wq"][0], L["Wsf"][0], Y=dY)
        hY.copy_(dY, non_blocking=True)

    for _ in range(warmup):
        step()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / steps, M * K_DIM * 2, M * N_DIM * 2


def cpu_baseline(M, budget_s=12.0):
    """The oracle as it stands, single-threaded, on a bounded row sample of the same layer."""
    import oracle
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(M)
    Wq, Wsf, inv_s = oracle.prep_weights(c.W, c.s, HAD_BLOCK)  # offline, not timed
    rows, elapsed, done = 1, 0.0, 0
    while elapsed < budget_s and done < M:
        n = min(rows, M - done)
        Xs = c.X[done:done + n]
        t0 = time.perf_counter()
        Xq, Xsf = oracle.act_quant(Xs, inv_s, HAD_BLOCK)
        oracle.linear(Xq, Xsf, Wq, Wsf)
        elapsed += time.perf_counter() - t0
        done += n
        rows *= 2
    flops = 2.0 * done * N_DIM * K_DIM
    return {"value": flops / elapsed / 1e12, "unit": "TFLOPS", "cores": 1, "kind": "oracle",
            "sample": f"{done} of {M} rows of the layer (act_quant + float64 GEMM over all N), "
                      f"{elapsed:.1f} s single-threaded C"}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    hbm, bf16, bf16_sus, peak_src = peaks()
    fp4_peak = bf16 * FP4_OVER_BF16

    if args.impl == "reference":
        if rank != 0:
            return
        steps = max(1, args.steps)
        cb = None
        vals = []
        for _ in range(steps):
            cb = cpu_baseline(args.M, budget_s=max(2.0, 60.0 / steps))
            vals.append(cb["value"])
        v = statistics.mean(vals)
        out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOPS",
               "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
               "ms_per_step": 2.0 * args.M * N_DIM * K_DIM / (v * 1e12) * 1e3, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": layer_config(args.M, args.gpus),
               "cpu_baseline": dict(cb, value=v),
               "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(out))
        return

    import w4a4_mxfp4_quantized_b200 as mq  # noqa: F401  (fails loudly without the built library)

    if dist_on:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    M = args.M
    if args.profile:
        profile_mode(M, args.steps, args.warmup, dev)
        return
    flops = 2.0 * M * N_DIM * K_DIM
    with ClockSampler(local) as clk:
        total_ms, aq_ms, gemm_ms, L = time_layer(M, args.steps, args.warmup, dev, dist_on)
    clocks = clk.summary()
    ms_step = max_over_ranks(total_ms, dist_on, dev) / args.steps
    value = job_tflops(world, flops, ms_step)

    del L
    p_total, p_aq, p_gemm, _ = time_layer(M, args.steps, args.warmup, dev, dist_on, plain=True)
    overhead = {"plain_mxfp4_ms_per_step": p_total / args.steps, "plain_act_quant_ms": p_aq, "plain_gemm_ms": p_gemm,
                "B_vs_plain_mxfp4_pipeline": (total_ms / args.steps) / (p_total / args.steps) - 1.0,
                "A_vs_gemm_on_prequantized_A": (total_ms / args.steps) / p_gemm - 1.0,
                "pages_figure_for_context": "2.3% end-to-end, Qwen3-32B in vLLM, hardware not stated"}
    _, _, _, L = time_layer(M, 3, 1, dev, dist_on)
    e2e_ms, h2d, d2h = time_e2e(M, max(3, args.steps // 2), 2, dev, L)
    e2e_ms = max_over_ranks(e2e_ms, dist_on, dev)
    e2e_value = job_tflops(world, flops, e2e_ms)

    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    gemm_kernel = gemm_kernel_name(M)
    aq_bytes = M * K_DIM * (2 + 0.5 + 1 / 32)
    sweep = []
    if not args.no_sweep:
        for m in M_SWEEP:
            tot, aq, gm, Lm = time_layer(m, max(10, args.steps), args.warmup, dev, dist_on, fused=True)
            fz = Lm["fused_ms"]
            del Lm
            fl = 2.0 * m * N_DIM * K_DIM
            g_bytes = N_DIM * K_DIM * 0.53125 + m * K_DIM * 0.53125 + m * N_DIM * 2
            a_bytes = m * K_DIM * (2 + 0.5 + 1 / 32)
            sweep.append({"M": m, "layer_tflops": fl / (tot / max(10, args.steps) * 1e-3) / 1e12,
                          "gemm_us": gm * 1e3, "gemm_tflops": fl / (gm * 1e-3) / 1e12,
                          "gemm_gbs": g_bytes / (gm * 1e-3) / 1e9,
                          "gemm_frac_fp4_peak": fl / (gm * 1e-3) / 1e12 / fp4_peak,
                          "gemm_frac_hbm": g_bytes / (gm * 1e-3) / 1e9 / hbm,
                          "act_quant_us": aq * 1e3, "act_quant_gbs": a_bytes / (aq * 1e-3) / 1e9,
                          "act_quant_frac_hbm": a_bytes / (aq * 1e-3) / 1e9 / hbm,
                          "fused_layer_us": fz * 1e3,
                          "fused_layer_tflops": fl / (fz * 1e-3) / 1e12,
                          "fused_form": "quantizer warps inside the skinny GEMM" if m <= 16
                          else "quantizer pass + GEMM in one call"})
    moe = moe_section(dev, hbm, fp4_peak) if not args.no_sweep else None
    prep = weight_prep_section(dev, hbm) if not args.no_sweep else None
    if rank != 0:
        if dist_on:
            torch.distributed.destroy_process_group()
        return
    out = {
        "metric": METRIC,
        "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp4 (e2m1 x e2m1, e8m0 scales, fp32 accumulate)", "data": "synthetic",
        "config": layer_config(M, world),
        "roofline": {"kernel": gemm_kernel, "bound": "tensor", "achieved": gemm_tflops,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                     "peak_source": f"{peak_src} bf16 burst x {FP4_OVER_BF16} (nominal FP4/BF16)",
                     "traffic": profiled_traffic(gemm_kernel, M)},
        "act_quant_roofline": {"kernel": "quant_kernel", "bound": "hbm", "achieved": aq_bytes / (aq_ms * 1e-3) / 1e9,
                               "peak": hbm, "unit": "GB/s", "frac": aq_bytes / (aq_ms * 1e-3) / 1e9 / hbm,
                               "peak_source": peak_src, "traffic": profiled_traffic("quant_kernel", M)},
        "kernel_ms": {"act_quant": aq_ms, "gemm": gemm_ms},
        "gpu_launches": 2 * args.steps,
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "clocks": dict(clocks, window="warm replays (1.5 s of this workload) and the timed replay"),
        "sweep": sweep,
        "transform_overhead": overhead,
        "moe": moe,
        "weight_prep": prep,
    }
    out["cpu_baseline"] = cpu_baseline(M) if world == 1 else None
    print(json.dumps(out))
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

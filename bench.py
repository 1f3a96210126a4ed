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
    p.add_argument("--profile-form", default="layer", choices=["layer", "fused", "w4a16", "moe"])
    p.add_argument("--details", default=None, help="also write every section's numbers to this JSON file")
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
    if "fused" in parts:  # the layer in one call from bf16 X (quantizer inside the GEMM kernel for M <= 4 and M > 128)
        mq.linear(L["X"][i], None, L["Wq"][i], L["Wsf"][i], mode=mq.A_BF16_ONE_LAUNCH, inv_s=L["inv_s"],
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


def time_graphs_interleaved(fns: dict, steps, stream, rounds=3):
    """Device time per call of each fn(i) (one graph of `steps` calls each), the graphs replayed in
    turn for `rounds` rounds; each keeps its fastest round. Under the power cap the SM clock drifts
    over seconds, so pipelines that are compared with each other are timed side by side."""
    graphs = {}
    for name, fn in fns.items():
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(i)
        g.replay()
        graphs[name] = g
    best = {name: float("inf") for name in fns}
    for _ in range(rounds):
        for name, g in graphs.items():
            best[name] = min(best[name], replay_ms(g, stream) / steps)
    del graphs
    return best


def moe_section(dev, hbm, fp4_peak, steps=20):
    """The grouped path (MoE 30B-A3B: 128 experts, top-8 of T tokens, Zipf routing) at T = 64, 1024,
    8192 for both projections: gate/up (2048 -> 1536) and down (768 -> 2048). Grouped act_quant and
    grouped GEMM are timed alone by graph replay. The prepared weights (213 MB gate/up, 107 MB down)
    are read once per call; X rotates over two copies."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    stream = torch.cuda.current_stream(dev)
    out = []
    for proj in ("gate_up", "down"):
        c0 = inputs.moe_30b_a3b(64, proj)
        E, N, K = c0.W.shape
        Wd = c0.W.to(dev)
        Wq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
        Wsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device=dev)
        inv = torch.empty(E, K, dtype=torch.float32, device=dev)
        sd = c0.s.to(dev)
        for e in range(E):
            mq.prep_weights(Wd[e], sd[e], HAD_BLOCK, Wq=Wq[e], Wsf=Wsf[e], inv_s=inv[e])
        del Wd
        for T in (64, 1024, 8192):
            c = inputs.moe_30b_a3b(T, proj, draw_w=False)
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
            glue = {}
            if proj == "gate_up":   # dispatch: quantize token rows through the routing's row index
                Xt = [c.X_tok.to(dev), c.X_tok.to(dev).clone()]
                idx = c.routing.token.to(torch.int32).to(dev)
                glue["gather_act_quant_us"] = 1e3 * time_graph(
                    lambda i: mq.act_quant_gather(Xt[i % 2], idx, inv, HAD_BLOCK, group_offsets=off, Xq=Xq[i % 2],
                                                  Xsf=Xsf[i % 2]), steps, stream)
                del Xt
            else:                   # combine: the down projection's rows back to token order, weighted
                pos, wts = c.routing.pos.to(dev), c.routing.weights.to(dev)
                out_t = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
                cm = time_graph(lambda i: mq.moe_combine(Y, pos, wts, out=out_t), steps, stream)
                c_bytes = rows * N * 2 + T * N * 2 + T * 8 * 8
                glue.update({"combine_us": cm * 1e3, "combine_gbs": c_bytes / (cm * 1e-3) / 1e9,
                             "combine_frac_hbm": c_bytes / (cm * 1e-3) / 1e9 / hbm})
            assert mq.device_status() == 0
            flops = 2.0 * N * K * rows
            used = int((counts > 0).sum())
            g_bytes = used * N * K * 0.53125 + rows * (0.53125 * K + 2 * N)
            a_bytes = rows * K * (2 + 0.5 + 1 / 32)
            out.append({"proj": proj, "T": T, "rows": rows, "experts_used": used, "K": K, "N": N,
                        "grouped_gemm_us": gm * 1e3, "grouped_gemm_tflops": flops / (gm * 1e-3) / 1e12,
                        "grouped_gemm_gbs": g_bytes / (gm * 1e-3) / 1e9,
                        "grouped_gemm_frac_fp4_peak": flops / (gm * 1e-3) / 1e12 / fp4_peak,
                        "grouped_gemm_frac_hbm": g_bytes / (gm * 1e-3) / 1e9 / hbm,
                        "grouped_act_quant_us": aq * 1e3, "grouped_act_quant_gbs": a_bytes / (aq * 1e-3) / 1e9,
                        "grouped_act_quant_frac_hbm": a_bytes / (aq * 1e-3) / 1e9 / hbm, **glue})
            del Xs, Xq, Xsf, Y
        del Wq, Wsf, inv
    return {"workload": f"moe_30b_a3b E=128 top-8, gate/up 2048->1536 and down 768->2048, b={HAD_BLOCK}",
            "points": out}


def _rotations(per_copy_bytes):
    """Input copies so that consecutive steps read HBM, not L2 (the copies exceed twice L2)."""
    return max(1, int(np.ceil(2 * L2_BYTES / per_copy_bytes)))


def prefill_section(dev, hbm, fp4_peak, steps=10):
    """Large prefill sweep, all eight shapes M in {4096, 16384} x K in {8192, 16384} x N in {8192,
    28672}: per shape the plain-MXFP4 pipeline (b = 1, no s: act_quant + GEMM), the transform
    pipeline (1/s, H_32: act_quant + GEMM), the one-launch call (bf16 X in, the 2-SM GEMM quantizes X itself), and the GEMM and the
    act_quant alone. Overheads: (B) transform pipeline over the plain pipeline, (A) transform
    pipeline over the GEMM on pre-quantized A. Inputs are drawn on the GPU with the same recipe."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    stream = torch.cuda.current_stream(dev)
    out = []
    for M in inputs.PREFILL_M:
        for K in inputs.PREFILL_K:
            for N in inputs.PREFILL_N:
                c = inputs.large_prefill(M, K, N, device=str(dev))
                per_copy = N * K * 0.53125 + M * K * (2 + 0.53125) + M * N * 2
                ncopy = _rotations(per_copy)
                Wq, Wsf, inv = mq.prep_weights(c.W, c.s, HAD_BLOCK)
                pWq, pWsf, _ = mq.prep_weights(c.W, None, 1)
                del c.W
                L = {"X": [c.X] + [c.X.clone() for _ in range(ncopy - 1)],
                     "Wq": [Wq] + [Wq.clone() for _ in range(ncopy - 1)],
                     "Wsf": [Wsf] + [Wsf.clone() for _ in range(ncopy - 1)],
                     "pWq": [pWq] + [pWq.clone() for _ in range(ncopy - 1)],
                     "pWsf": [pWsf] + [pWsf.clone() for _ in range(ncopy - 1)],
                     "Xq": [torch.empty(M, K // 2, dtype=torch.uint8, device=dev) for _ in range(ncopy)],
                     "Xsf": [torch.empty(mq.sf_bytes(M, K), dtype=torch.uint8, device=dev) for _ in range(ncopy)],
                     "Y": [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(ncopy)]}
                ws = torch.zeros(mq.fused_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
                j = lambda i: i % ncopy

                def plain(i):
                    mq.act_quant(L["X"][j(i)], None, 1, Xq=L["Xq"][j(i)], Xsf=L["Xsf"][j(i)])
                    mq.linear(L["Xq"][j(i)], L["Xsf"][j(i)], L["pWq"][j(i)], L["pWsf"][j(i)], Y=L["Y"][j(i)])

                def transform(i):
                    mq.act_quant(L["X"][j(i)], inv, HAD_BLOCK, Xq=L["Xq"][j(i)], Xsf=L["Xsf"][j(i)])
                    mq.linear(L["Xq"][j(i)], L["Xsf"][j(i)], L["Wq"][j(i)], L["Wsf"][j(i)], Y=L["Y"][j(i)])

                def fused(i):   # one launch: the 2-SM GEMM quantizes X itself
                    mq.linear(L["X"][j(i)], None, L["Wq"][j(i)], L["Wsf"][j(i)], mode=mq.A_BF16_ONE_LAUNCH, inv_s=inv,
                              had_block=HAD_BLOCK, Y=L["Y"][j(i)], workspace=ws)

                def gemm(i):
                    mq.linear(L["Xq"][j(i)], L["Xsf"][j(i)], L["Wq"][j(i)], L["Wsf"][j(i)], Y=L["Y"][j(i)])

                def aq(i):
                    mq.act_quant(L["X"][j(i)], inv, HAD_BLOCK, Xq=L["Xq"][j(i)], Xsf=L["Xsf"][j(i)])

                def aq_plain(i):
                    mq.act_quant(L["X"][j(i)], None, 1, Xq=L["Xq"][j(i)], Xsf=L["Xsf"][j(i)])

                t = time_graphs_interleaved({"plain": plain, "transform": transform, "fused": fused, "gemm": gemm,
                                             "act_quant": aq, "act_quant_plain": aq_plain}, steps, stream)
                assert mq.device_status() == 0
                flops = 2.0 * M * N * K
                a_bytes = M * K * (2 + 0.5 + 1 / 32)
                out.append({"M": M, "K": K, "N": N, "copies": ncopy,
                            **{f"{k}_ms": v for k, v in t.items()},
                            "gemm_tflops": flops / (t["gemm"] * 1e-3) / 1e12,
                            "gemm_frac_fp4_peak": flops / (t["gemm"] * 1e-3) / 1e12 / fp4_peak,
                            "transform_tflops": flops / (t["transform"] * 1e-3) / 1e12,
                            "fused_tflops": flops / (t["fused"] * 1e-3) / 1e12,
                            "act_quant_gbs": a_bytes / (t["act_quant"] * 1e-3) / 1e9,
                            "act_quant_frac_hbm": a_bytes / (t["act_quant"] * 1e-3) / 1e9 / hbm,
                            "overhead_B_transform": t["transform"] / t["plain"] - 1.0,
                            "overhead_B_fused": t["fused"] / t["plain"] - 1.0,
                            "overhead_A_transform": t["transform"] / t["gemm"] - 1.0,
                            "overhead_A_fused": t["fused"] / t["gemm"] - 1.0,
                            # the transform's own cost: the only kernel that differs between the two
                            # pipelines is act_quant (the GEMMs differ only in their operand bits, which
                            # under the power cap moves the clock and with it the whole-pipeline ratio)
                            "overhead_B_act_quant_only": (t["act_quant"] - t["act_quant_plain"]) / t["plain"]})
                del L, ws, Wq, Wsf, pWq, pWsf, c
                torch.cuda.empty_cache()
    return {"workload": "large prefill, M x K x N in {4096,16384} x {8192,16384} x {8192,28672}, b=32",
            "points": out}


def qwen3_section(dev, hbm, fp4_peak, steps=10):
    """The Qwen3-32B decoder-layer linears in sequence at M in {1, 8, 64, 4096}: one step = the four
    act_quants (qkv, o, gate/up and down inputs) and the seven GEMMs (q, k, v, o, gate, up, down);
    also the same layer with the fused QKV (N = 10240) and GateUp (N = 51200) linears (four GEMMs).
    The 487.6 M weights (259 MB prepared) exceed L2, so every step reads them from HBM."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    stream = torch.cuda.current_stream(dev)
    xs0, ws = inputs.qwen3_32b_layer(1, device=str(dev))
    prepped, keys = {}, {}
    for name, K, N, key in inputs.QWEN3_32B_LINEARS:
        prepped[name] = mq.prep_weights(ws[name], xs0[key].s, HAD_BLOCK)
        keys[name] = key
    inv = {}
    for name, _, _, key in inputs.QWEN3_32B_LINEARS:
        inv.setdefault(key, prepped[name][2])
    fused_w = {"qkv": mq.prep_weights(torch.cat([ws["q_proj"], ws["k_proj"], ws["v_proj"]]), xs0["qkv"].s, HAD_BLOCK),
               "gateup": mq.prep_weights(torch.cat([ws["gate_proj"], ws["up_proj"]]), xs0["gateup"].s, HAD_BLOCK)}
    # gate/up interleaved in blocks of 64 rows for the fused SwiGLU epilogue
    swiglu_w = mq.prep_weights(mq.interleave_gate_up(ws["gate_proj"], ws["up_proj"]), xs0["gateup"].s, HAD_BLOCK)
    del ws
    w_params = sum(K * N for _, K, N, _ in inputs.QWEN3_32B_LINEARS)
    out = []
    for M in inputs.QWEN3_32B_M:
        xs, _ = inputs.qwen3_32b_layer(M, draw_w=False, device=str(dev))
        A = {key: mq.act_quant(xs[key].X, inv[key], HAD_BLOCK) for key in xs}
        Y = {name: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for name, _, N, _ in inputs.QWEN3_32B_LINEARS}
        Yf = {"qkv": torch.empty(M, 10240, dtype=torch.bfloat16, device=dev),
              "gateup": torch.empty(M, 51200, dtype=torch.bfloat16, device=dev)}

        def layer(i):
            for key in xs:
                mq.act_quant(xs[key].X, inv[key], HAD_BLOCK, Xq=A[key][0], Xsf=A[key][1])
            for name in prepped:
                mq.linear(A[keys[name]][0], A[keys[name]][1], prepped[name][0], prepped[name][1], Y=Y[name])

        def layer_fused_weights(i):
            for key in xs:
                mq.act_quant(xs[key].X, inv[key], HAD_BLOCK, Xq=A[key][0], Xsf=A[key][1])
            for key in ("qkv", "gateup"):
                mq.linear(A[key][0], A[key][1], fused_w[key][0], fused_w[key][1], Y=Yf[key])
            for name in ("o_proj", "down_proj"):
                mq.linear(A[keys[name]][0], A[keys[name]][1], prepped[name][0], prepped[name][1], Y=Y[name])

        I = 25600
        H = (torch.empty(M, I // 2, dtype=torch.uint8, device=dev), torch.empty(mq.sf_bytes(M, I), dtype=torch.uint8, device=dev))
        GU = torch.empty(M, 2 * I, dtype=torch.float32, device=dev)
        ws_sw = torch.zeros(max(int(mq.lib().macaq_linear_swiglu_workspace_bytes(M, 2 * I, 5120)),
                                mq.workspace_bytes(M, 2 * I, 5120), 1), dtype=torch.uint8, device=dev)

        def swiglu_fused(i):
            mq.linear_swiglu(A["gateup"][0], A["gateup"][1], swiglu_w[0], swiglu_w[1], inv["down"], HAD_BLOCK,
                             Hq=H[0], Hsf=H[1], workspace=ws_sw)

        def swiglu_two_step(i):
            mq.linear(A["gateup"][0], A["gateup"][1], swiglu_w[0], swiglu_w[1], out_dtype=mq.OUT_F32, Y=GU, workspace=ws_sw)
            mq.swiglu_act_quant(GU, inv["down"], HAD_BLOCK, Hq=H[0], Hsf=H[1])

        def layer_swiglu(i):   # q, k, v, o as in layer(); gate/up with the fused epilogue feeding down
            for key in ("qkv", "o"):
                mq.act_quant(xs[key].X, inv[key], HAD_BLOCK, Xq=A[key][0], Xsf=A[key][1])
            mq.act_quant(xs["gateup"].X, inv["gateup"], HAD_BLOCK, Xq=A["gateup"][0], Xsf=A["gateup"][1])
            for name in ("q_proj", "k_proj", "v_proj", "o_proj"):
                mq.linear(A[keys[name]][0], A[keys[name]][1], prepped[name][0], prepped[name][1], Y=Y[name])
            swiglu_fused(i)
            mq.linear(H[0], H[1], prepped["down_proj"][0], prepped["down_proj"][1], Y=Y["down_proj"])

        t = time_graph(layer, steps, stream)
        tf = time_graph(layer_fused_weights, steps, stream)
        tsw = time_graphs_interleaved({"fused": swiglu_fused, "two_step": swiglu_two_step, "layer": layer_swiglu},
                                      steps, stream)
        per = {}
        for name in prepped:
            per[name] = time_graph(lambda i, n=name: mq.linear(A[keys[n]][0], A[keys[n]][1], prepped[n][0], prepped[n][1],
                                                                Y=Y[n]), steps, stream) * 1e3
        assert mq.device_status() == 0
        flops = 2.0 * M * w_params
        bytes_ = w_params * 0.53125 + sum(M * xs[k].X.shape[1] * (2 + 2 * 0.53125) for k in xs) + \
            sum(2 * M * N for _, _, N, _ in inputs.QWEN3_32B_LINEARS)
        out.append({"M": M, "layer_us": t * 1e3, "layer_tflops": flops / (t * 1e-3) / 1e12,
                    "layer_frac_fp4_peak": flops / (t * 1e-3) / 1e12 / fp4_peak,
                    "layer_gbs": bytes_ / (t * 1e-3) / 1e9, "layer_frac_hbm": bytes_ / (t * 1e-3) / 1e9 / hbm,
                    "layer_fused_qkv_gateup_us": tf * 1e3, "gemm_us": per,
                    "swiglu_fused_us": tsw["fused"] * 1e3, "swiglu_two_step_us": tsw["two_step"] * 1e3,
                    "layer_swiglu_chain_us": tsw["layer"] * 1e3})
        del xs, A, Y, Yf, H, GU, ws_sw
    return {"workload": "qwen3_32b decoder-layer linears (q,k,v,o,gate,up,down), b=32", "points": out}


def copy_ceiling(dev, nbytes, steps=20):
    """A device-to-device copy that moves nbytes (half read, half written), timed like the kernels:
    the rate a plain stream of that size reaches on this GPU, for context beside the HBM peak."""
    n = int(nbytes // 4)
    ncopy = _rotations(nbytes)
    src = [torch.empty(n // 2, dtype=torch.int32, device=dev) for _ in range(ncopy)]
    dst = [torch.empty(n // 2, dtype=torch.int32, device=dev) for _ in range(ncopy)]
    ms = time_graph(lambda i: dst[i % ncopy].copy_(src[i % ncopy]), steps, torch.cuda.current_stream(dev))
    return {"bytes": int(nbytes), "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9}


def flip_section(dev, sweeps=1):
    """Flip-Refinement of the Llama-3-8B up/gate weights [14336, 4096] with a Hessian from 512
    transformed calibration rows (the Hessian product is plumbing: torch, fp32). One timed call."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(2048)
    W, s = c.W.to(dev), c.s.to(dev)
    Wq, Wsf, inv = mq.prep_weights(W, s, HAD_BLOCK)
    Xt = (c.X[:512].to(dev).float() * inv)
    Xt = Xt.view(512, -1, HAD_BLOCK) @ torch.from_numpy(_sylvester(HAD_BLOCK)).to(dev)
    Xt = Xt.view(512, -1)
    H = (Xt.T @ Xt / 512).contiguous()
    q = Wq.clone()
    mq.flip_refine(W, s, H, q, Wsf, HAD_BLOCK, sweeps)          # warm-up (and the module load)
    torch.cuda.synchronize()
    q.copy_(Wq)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(dev)
    a.record(stream)
    flips = mq.flip_refine(W, s, H, q, Wsf, HAD_BLOCK, sweeps)
    b.record(stream)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    return {"workload": f"llama3_8b_up_gate W [{N_DIM}, {K_DIM}], H from 512 rows, {sweeps} sweep(s)",
            "ms": a.elapsed_time(b), "moves_per_row": float(flips.float().mean()),
            "codes_changed_frac": float((q != Wq).float().mean())}


def _sylvester(b):
    h = np.ones((1, 1), np.float32)
    while h.shape[0] < b:
        h = np.block([[h, h], [h, -h]])
    return h


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


def had_block_section(dev, hbm, fp4_peak, M=2048, steps=20):
    """The Llama-3-8B up/gate layer at M = 2048 with each Hadamard block size b in {16, 32, 64, 128}
    (weights prepared per b): act_quant alone and act_quant + GEMM, timed side by side. Inputs rotate
    over copies larger than twice L2."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(M, draw_w=True)
    W, s = c.W.to(dev), c.s.to(dev)
    ncopy = copies_for(M)
    X = [c.X.to(dev)] + [None] * (ncopy - 1)
    for i in range(1, ncopy):
        X[i] = X[0].clone()
    Xq = [torch.empty(M, K_DIM // 2, dtype=torch.uint8, device=dev) for _ in range(ncopy)]
    Xsf = [torch.empty(mq.sf_bytes(M, K_DIM), dtype=torch.uint8, device=dev) for _ in range(ncopy)]
    Y = [torch.empty(M, N_DIM, dtype=torch.bfloat16, device=dev) for _ in range(ncopy)]
    flops = 2.0 * M * N_DIM * K_DIM
    aq_bytes = M * K_DIM * 2.53125
    out = []
    for b in (16, 32, 64, 128):
        Wq, Wsf, inv = mq.prep_weights(W, s, b)
        Wqs = [Wq] + [Wq.clone() for _ in range(ncopy - 1)]
        Wsfs = [Wsf] + [Wsf.clone() for _ in range(ncopy - 1)]

        def aq(i, b=b, inv=inv):
            j = i % ncopy
            mq.act_quant(X[j], inv, b, Xq=Xq[j], Xsf=Xsf[j])

        def layer(i, b=b, inv=inv, Wqs=Wqs, Wsfs=Wsfs):
            j = i % ncopy
            mq.act_quant(X[j], inv, b, Xq=Xq[j], Xsf=Xsf[j])
            mq.linear(Xq[j], Xsf[j], Wqs[j], Wsfs[j], Y=Y[j])

        t = time_graphs_interleaved({"aq": aq, "layer": layer}, steps, torch.cuda.current_stream(dev))
        out.append({"had_block": b, "act_quant_us": t["aq"] * 1e3,
                    "act_quant_frac_hbm": aq_bytes / (t["aq"] * 1e-3) / 1e9 / hbm,
                    "layer_us": t["layer"] * 1e3, "layer_tflops": flops / (t["layer"] * 1e-3) / 1e12})
        del Wqs, Wsfs
    assert mq.device_status() == 0
    return {"workload": f"llama3_8b_up_gate M={M} K={K_DIM} N={N_DIM}, b in 16..128", "points": out}


def profile_moe(steps, warmup, dev, T=8192):
    """Eager passes of the MoE 30B-A3B gate/up projection at T tokens (grouped act_quant then the
    grouped GEMM, which runs on 2-SM pairs at T = 8192), for ncu captures."""
    import w4a4_mxfp4_quantized_b200 as mq
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.moe_30b_a3b(T, "gate_up")
    E, N, K = c.W.shape
    Wq = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
    Wsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device=dev)
    inv = torch.empty(E, K, dtype=torch.float32, device=dev)
    W, s = c.W.to(dev), c.s.to(dev)
    for e in range(E):
        mq.prep_weights(W[e], s[e], HAD_BLOCK, Wq=Wq[e], Wsf=Wsf[e], inv_s=inv[e])
    del W
    off = c.offsets.to(dev)
    X = c.X.to(dev)
    for _ in range(warmup + steps):
        Xq, Xsf = mq.act_quant(X, inv, HAD_BLOCK, group_offsets=off)
        mq.grouped_linear(Xq, Xsf, off, Wq, Wsf)
    torch.cuda.synchronize(dev)
    assert mq.device_status() == 0


def profile_mode(M, steps, warmup, dev, form="layer"):
    """Eager layer passes with no timing: the commands the ncu captures run. form: "layer" (act_quant
    then the GEMM), "fused" (the one-call layer from bf16 X), "w4a16" (the weight-only layer), "moe"
    (the MoE gate/up projection at T = 8192)."""
    import w4a4_mxfp4_quantized_b200 as mq

    if form == "moe":
        profile_moe(steps, warmup, dev)
        return
    L = make_layer(M, dev, 2)
    for i in range(warmup + steps):
        if form == "fused":
            run_layer(mq, L, i % 2, ("fused",))
        elif form == "w4a16":
            mq.linear_w4a16(L["X"][i % 2], L["inv_s"], L["Wq"][i % 2], L["Wsf"][i % 2], had_block=HAD_BLOCK,
                            Y=L["Y"][i % 2])
        else:
            run_layer(mq, L, i % 2)
    torch.cuda.synchronize(dev)
    assert mq.device_status() == 0


def time_e2e(M, steps, warmup, dev, L, fused=False):
    """The same layer through the public API from pinned host X to host Y, copies included (the
    one-call fused form when fused, else act_quant then linear)."""
    import w4a4_mxfp4_quantized_b200 as mq

    hX = L["host_X"].pin_memory()
    hY = torch.empty(M, N_DIM, dtype=torch.bfloat16).pin_memory()
    dX, dY = L["X"][0], L["Y"][0]
    stream = torch.cuda.current_stream(dev)

    def step():
        dX.copy_(hX, non_blocking=True)
        if fused:
            mq.linear(dX, None, L["Wq"][0], L["Wsf"][0], mode=mq.A_BF16_ONE_LAUNCH, inv_s=L["inv_s"], had_block=HAD_BLOCK,
                      Y=dY)
        else:
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


CPU_ROWS = 8  # rows of the layer per oracle worker and sample (fixed, so the per-row rate is reproducible)


def cpu_setup(M):
    """Inputs of the layer for the oracle: X bits, and W' prepared by the oracle (offline, untimed)."""
    import oracle
    from w4a4_mxfp4_quantized_b200 import inputs

    c = inputs.llama3_8b_up(M)
    Wq, Wsf, inv_s = oracle.prep_weights(c.W, c.s, HAD_BLOCK)
    bits = c.X.contiguous().view(torch.int16).numpy().view(np.uint16)
    return c, bits, Wq, Wsf, inv_s


def cpu_baseline(M, samples=2):
    """The oracle as it stands, on the host cores: every worker process (one per core) runs
    act_quant + the float64 GEMM over all N on its own CPU_ROWS rows of the layer; the value is the
    rows all workers finished / the wall time of the sample (best of `samples`). Also the same work on
    one core, and the oracle's act_quant and weight prep timed in full on one core (GB/s of
    2.53125 B per element)."""
    import oracle
    from oracle import timing

    c, bits, Wq, Wsf, inv_s = cpu_setup(M)
    t1 = timing.single_thread_sample(bits[:CPU_ROWS], Wq, Wsf, inv_s, HAD_BLOCK)
    with timing.LayerPool(Wq, Wsf, inv_s, HAD_BLOCK) as pool:
        best = None
        for i in range(samples):
            wall, rows = pool.sample(bits, CPU_ROWS, start=i * pool.workers * CPU_ROWS)
            best = wall if best is None else min(best, wall)
        workers = pool.workers
    t0 = time.perf_counter()
    oracle.act_quant(bits, inv_s, HAD_BLOCK)
    t_aq = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.prep_weights(c.W, c.s, HAD_BLOCK)
    t_prep = time.perf_counter() - t0
    per_row = 2.0 * N_DIM * K_DIM
    return {"value": workers * CPU_ROWS * per_row / best / 1e12, "unit": "TFLOPS", "cores": workers, "kind": "oracle",
            "sample": f"{workers} processes x {CPU_ROWS} rows of the layer (act_quant + float64 GEMM over all N), "
                      f"best of {samples}: {best:.2f} s",
            "single_core_tflops": CPU_ROWS * per_row / t1 / 1e12,
            "act_quant_gbs_1core": M * K_DIM * 2.53125 / t_aq / 1e9,
            "weight_prep_gbs_1core": N_DIM * K_DIM * 2.53125 / t_prep / 1e9}


def reference_arm(args):
    """--impl reference: the oracle timed on the host cores on the same workload, metric and unit.
    One step = one all-core sample (every core's worker on CPU_ROWS rows of the layer)."""
    from oracle import timing

    _, bits, Wq, Wsf, inv_s = cpu_setup(args.M)
    walls, rows = [], 0
    with timing.LayerPool(Wq, Wsf, inv_s, HAD_BLOCK) as pool:
        for i in range(args.warmup + args.steps):
            wall, rows = pool.sample(bits, CPU_ROWS, start=i * pool.workers * CPU_ROWS)
            if i >= args.warmup:
                walls.append(wall)
        workers = pool.workers
    ms = 1e3 * sum(walls) / len(walls)
    v = rows * 2.0 * N_DIM * K_DIM / (ms * 1e-3) / 1e12
    sample = f"each step: {workers} processes x {CPU_ROWS} rows of the layer (act_quant + float64 GEMM over all N)"
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": layer_config(args.M, args.gpus),
            "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": workers, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _r(x, n=3):
    return None if x is None else float(f"{x:.{n}g}")


def summary(sweep, overhead, prefill, qwen3, moe, prep, ceiling, flip=None, hb=None):
    """Short strings of the sections (the full numbers go to --details), so that the whole line stays
    about 3 KB. Legend: g = GEMM alone, aq = act_quant alone, f = one-call layer, wo = weight-only
    layer (us); fp4 / hbm = fraction of the FP4 / HBM peak; B = transform pipeline vs plain MXFP4,
    1L = the one-launch form vs plain MXFP4; fusedW = Qwen3 layer with fused QKV and GateUp weights;
    sw = gate/up GEMM with the SwiGLU epilogue vs the two-step form (us)."""
    out = {"legend": "us; g gemm, aq act_quant, f one-call layer, wo weight-only, B vs plain mxfp4, 1L one launch"}
    if sweep:
        out["sweep"] = " | ".join(
            f"M{p['M']} g{p['gemm_us']:.1f} {p['gemm_frac_hbm']:.2f}hbm {p['gemm_frac_fp4_peak']:.2f}fp4 "
            f"aq{p['act_quant_us']:.1f} f{p['fused_layer_us']:.1f}"
            + (f" wo{p['w4a16_layer_us']:.1f}" if p.get("w4a16_layer_us") else "") for p in sweep)
    out["overhead"] = {k: _r(overhead[k]) for k in ("B_vs_plain_mxfp4_pipeline", "A_vs_gemm_on_prequantized_A")}
    if prefill:
        out["prefill"] = " | ".join(
            f"{p['M'] // 1024}k{p['K'] // 1024}k{p['N'] // 1024}k {p['gemm_frac_fp4_peak']:.2f}fp4 "
            f"B{100 * p['overhead_B_transform']:+.1f}% 1L{100 * p['overhead_B_fused']:+.0f}% "
            f"aq{p['act_quant_frac_hbm']:.2f}hbm" for p in prefill["points"])
    if qwen3:
        out["qwen3"] = " | ".join(
            f"M{p['M']} {p['layer_us']:.0f}us fusedW{p['layer_fused_qkv_gateup_us']:.0f} "
            f"sw{p['swiglu_fused_us']:.0f}/{p['swiglu_two_step_us']:.0f}" for p in qwen3["points"])
    if moe:
        def glue(p):
            if "combine_us" in p:
                return f" comb{p['combine_frac_hbm']:.2f}hbm"
            return ""
        out["moe"] = " | ".join(
            f"{'gu' if p['proj'] == 'gate_up' else 'dn'}T{p['T']} g{p['grouped_gemm_us']:.0f} "
            f"{p['grouped_gemm_frac_hbm']:.2f}hbm {p['grouped_gemm_frac_fp4_peak']:.2f}fp4{glue(p)}"
            for p in moe["points"])
    if hb:
        out["had_block"] = " | ".join(f"b{p['had_block']} aq{p['act_quant_us']:.1f} layer{p['layer_us']:.1f}"
                                      for p in hb["points"])
    if flip:
        out["flip_refine"] = f"{flip['ms']:.0f}ms {flip['moves_per_row']:.0f}moves/row"
    if prep:
        out["weight_prep"] = f"{prep['us']:.1f}us {prep['frac_hbm']:.2f}hbm"
    if ceiling:
        out["copy_ceiling"] = "; ".join(f"{c['bytes'] / 1e6:.0f}MB {c['gbs']:.0f}GB/s" for c in ceiling)
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    hbm, bf16, bf16_sus, peak_src = peaks()
    fp4_peak = bf16 * FP4_OVER_BF16

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)))
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
        profile_mode(M, args.steps, args.warmup, dev, args.profile_form)
        return
    flops = 2.0 * M * N_DIM * K_DIM
    with ClockSampler(local) as clk:
        total_ms, aq_ms, gemm_ms, L = time_layer(M, args.steps, args.warmup, dev, dist_on, fused=True)
    clocks = clk.summary()
    two_kernel_ms = total_ms / args.steps
    fused_ms = L["fused_ms"]
    # the step is the faster of the library's two forms of the layer: act_quant then the GEMM (two
    # launches), or the one call from bf16 X (one launch for large M: the GEMM quantizes X itself)
    fused_step = fused_ms < two_kernel_ms
    ms_step = max_over_ranks(fused_ms if fused_step else two_kernel_ms, dist_on, dev)
    value = job_tflops(world, flops, ms_step)

    del L
    p_total, p_aq, p_gemm, Lp = time_layer(M, args.steps, args.warmup, dev, dist_on, plain=True, fused=True)
    p_fused = Lp["fused_ms"]
    del Lp
    p_step = p_fused if fused_step else p_total / args.steps
    overhead = {"plain_mxfp4_ms_per_step": p_step, "plain_act_quant_ms": p_aq, "plain_gemm_ms": p_gemm,
                "B_vs_plain_mxfp4_pipeline": ms_step / p_step - 1.0,
                "A_vs_gemm_on_prequantized_A": ms_step / p_gemm - 1.0,
                "two_kernel_B": two_kernel_ms / (p_total / args.steps) - 1.0,
                "pages_figure_for_context": "2.3% end-to-end, Qwen3-32B in vLLM, hardware not stated"}
    _, _, _, L = time_layer(M, 3, 1, dev, dist_on)
    e2e_ms, h2d, d2h = time_e2e(M, max(3, args.steps // 2), 2, dev, L, fused_step)
    del L
    e2e_ms = max_over_ranks(e2e_ms, dist_on, dev)
    e2e_value = job_tflops(world, flops, e2e_ms)

    # the dominant kernel: the GEMM, or in the one-launch form the GEMM that also quantizes X
    gemm_tflops = flops / ((fused_ms if fused_step else gemm_ms) * 1e-3) / 1e12
    gemm_kernel = gemm_kernel_name(M) + (" (one launch, quantizing X itself)" if fused_step else "")
    aq_bytes = M * K_DIM * (2 + 0.5 + 1 / 32)
    sweep, prefill, qwen3, moe, prep, ceiling, flip, hb = [], None, None, None, None, [], None, None
    if not args.no_sweep:
        for m in M_SWEEP:
            tot, aq, gm, Lm = time_layer(m, max(10, args.steps), args.warmup, dev, dist_on, fused=True)
            fz = Lm["fused_ms"]
            wo = None
            if m <= 64:   # the weight-only layer on the same weights (bf16 activations)
                ncp = len(Lm["X"])
                Yw = torch.empty(m, N_DIM, dtype=torch.bfloat16, device=dev)
                wo = time_graph(lambda i: mq.linear_w4a16(Lm["X"][i % ncp], Lm["inv_s"], Lm["Wq"][i % ncp],
                                                          Lm["Wsf"][i % ncp], had_block=HAD_BLOCK, Y=Yw),
                                max(10, args.steps), torch.cuda.current_stream(dev))
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
                          "fused_form": "quantizer warps inside the skinny GEMM" if m <= 4
                          else ("quantizer pass + skinny GEMM" if m <= 128 else "2-SM GEMM quantizing X itself (one launch)"),
                          "w4a16_layer_us": None if wo is None else wo * 1e3,
                          "w4a16_frac_hbm": None if wo is None else
                          (N_DIM * K_DIM * 0.53125 + m * K_DIM * 2 + m * N_DIM * 2) / (wo * 1e-3) / 1e9 / hbm})
        prefill = prefill_section(dev, hbm, fp4_peak)
        qwen3 = qwen3_section(dev, hbm, fp4_peak)
        moe = moe_section(dev, hbm, fp4_peak)
        prep = weight_prep_section(dev, hbm)
        hb = had_block_section(dev, hbm, fp4_peak)
        flip = flip_section(dev)
        ceiling = [copy_ceiling(dev, aq_bytes), copy_ceiling(dev, 16384 * 16384 * 2.53125)]
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
        "kernel_ms": {"act_quant": aq_ms, "gemm": gemm_ms, "two_kernel_step": two_kernel_ms, "one_call_step": fused_ms},
        "form": "one call (bf16 X in, in-GEMM quantization)" if fused_step else "act_quant + GEMM",
        "gpu_launches": (1 if fused_step else 2) * args.steps,
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "clocks": dict(clocks, window="warm replays (1.5 s of this workload) and the timed replay"),
    }
    out["cpu_baseline"] = cpu_baseline(M) if world == 1 else None
    out["summary"] = summary(sweep, overhead, prefill, qwen3, moe, prep, ceiling, flip, hb)
    out["summary"]["gemm_alone"] = f"{gemm_ms * 1e3:.1f}us {flops / (gemm_ms * 1e-3) / 1e12 / fp4_peak:.3f}fp4"
    if args.details:
        with open(args.details, "w") as f:
            json.dump({**out, "sweep": sweep, "transform_overhead": overhead, "prefill": prefill, "qwen3": qwen3,
                       "moe": moe, "weight_prep": prep, "copy_ceiling": ceiling, "flip_refine": flip,
                       "had_block": hb}, f, indent=1)
    print(json.dumps(out))
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

"""GPU parity at the full sizes of every workload, on densely sampled GEMM rows.

Qwen3-32B decoder layer (seven linears at M = 1, 8, 64, 4096, plus the fused QKV and GateUp
linears), the MoE 30B-A3B grouped GEMMs (gate/up 2048 -> 1536 and down 768 -> 2048 at T = 64,
1024, 8192 tokens routed top-8 over 128 experts), and all eight shapes of the large-prefill dense
sweep. Each side quantizes with its own code: activation codes and scales must match the oracle bit
for bit over the whole tensor, weight codes and scales over the whole matrix, and the fp32 GEMM
output within 1e-5 of sum|terms| on every column of the checked rows: all rows up to 512, else 256
random rows plus the first and last row of every 128-row tile (every tile the persistent kernels
hand out, whichever round it falls in). The bf16 output must be the round-to-nearest-even cast of
the fp32 output over the whole matrix.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import grouped_sf_rows, unswizzle

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def checked_rows(M, seed, tile_starts=None):
    """All rows when M <= 512; else 256 random rows plus both edge rows of every 128-row tile
    (tile_starts: the first row of each tile with its end, for grouped layouts)."""
    if M <= 512:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    if tile_starts is None:
        starts = np.arange(0, M, 128)
        ends = np.minimum(starts + 128, M)
    else:
        starts, ends = tile_starts
    edges = np.concatenate([starts, ends - 1])
    return np.unique(np.concatenate([edges, rng.choice(M, 256, replace=False)]))


def grouped_tiles(off):
    """First row and end row of every 128-row tile of every non-empty expert."""
    starts, ends = [], []
    for e in range(len(off) - 1):
        for r0 in range(int(off[e]), int(off[e + 1]), 128):
            starts.append(r0)
            ends.append(min(r0 + 128, int(off[e + 1])))
    return np.array(starts, np.int64), np.array(ends, np.int64)


def close(y32, rows, Y, T):
    y = y32.double().cpu().numpy()[rows]
    err = np.abs(y - Y)
    bad = np.argwhere(err > RTOL * T + 1e-30)
    assert bad.size == 0, f"{len(bad)} outputs off, worst rel {np.max(err / (T + 1e-30)):.3g} at {bad[:3].tolist()}"


@functools.lru_cache(maxsize=None)
def qwen3_weights():
    """The seven Qwen3-32B weights (drawn once) and the oracle's prepared form of each, keyed by the
    input they share a scale with; s comes from the input of the same key (M-independent draw)."""
    xs, ws = inputs.qwen3_32b_layer(1)
    prepped = {}
    for name, K, N, key in inputs.QWEN3_32B_LINEARS:
        prepped[name] = oracle.prep_weights(ws[name], xs[key].s, 32)
    return ws, prepped


def check_gpu_weights(W, s, b, oWq, oWsf, oinv):
    N, K = W.shape
    gWq, gWsf, ginv = mq.prep_weights(W.cuda(), s.cuda(), b)
    np.testing.assert_array_equal(gWq.cpu().numpy(), oWq)
    np.testing.assert_array_equal(unswizzle(gWsf.cpu().numpy(), N, K), oWsf)
    np.testing.assert_array_equal(ginv.cpu().numpy().view(np.uint32), oinv.view(np.uint32))
    return gWq, gWsf, ginv


def check_act(X, ginv, oinv, b):
    M, K = X.shape
    oXq, oXsf = oracle.act_quant(X, oinv, b)
    gXq, gXsf = mq.act_quant(X.cuda(), ginv, b)
    np.testing.assert_array_equal(gXq.cpu().numpy(), oXq)
    np.testing.assert_array_equal(unswizzle(gXsf.cpu().numpy(), M, K), oXsf)
    return (gXq, gXsf), (oXq, oXsf)


def check_gemm(g_act, o_act, gW, oW, seed):
    (gXq, gXsf), (oXq, oXsf) = g_act, o_act
    (gWq, gWsf), (oWq, oWsf) = gW, oW
    M = gXq.shape[0]
    y32 = mq.linear(gXq, gXsf, gWq, gWsf, out_dtype=mq.OUT_F32)
    y16 = mq.linear(gXq, gXsf, gWq, gWsf, out_dtype=mq.OUT_BF16)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    rows = checked_rows(M, seed)
    Y, T = oracle.linear_matmul(oXq, oXsf, oWq, oWsf, rows=rows)
    close(y32, rows, Y, T)


@pytest.mark.parametrize("M", inputs.QWEN3_32B_M)
def test_qwen3_32b_layer(M):
    """The seven linears in sequence (q, k, v share one input and s; gate, up share one), then the
    fused QKV (N = 10240) and GateUp (N = 51200) linears over the same inputs."""
    xs, _ = inputs.qwen3_32b_layer(M, draw_w=False)
    ws, prepped = qwen3_weights()
    acts = {}
    gw = {}
    for j, (name, K, N, key) in enumerate(inputs.QWEN3_32B_LINEARS):
        c = xs[key]
        oWq, oWsf, oinv = prepped[name]
        gWq, gWsf, ginv = check_gpu_weights(ws[name], c.s, 32, oWq, oWsf, oinv)
        gw[name] = (gWq, gWsf)
        if key not in acts:
            acts[key] = check_act(c.X, ginv, oinv, 32)
        check_gemm(*acts[key], (gWq, gWsf), (oWq, oWsf), seed=M * 10 + j)
    for fused, parts, key in (("qkv", ("q_proj", "k_proj", "v_proj"), "qkv"), ("gateup", ("gate_proj", "up_proj"), "gateup")):
        # a fused linear is its parts' weight rows stacked: prepare the stacked matrix on the GPU and
        # compare with the oracle's per-part preparations stacked the same way
        W = torch.cat([ws[p] for p in parts])
        oWq = np.concatenate([prepped[p][0] for p in parts])
        oWsf = np.concatenate([prepped[p][1] for p in parts])
        gWq, gWsf, _ = check_gpu_weights(W, xs[key].s, 32, oWq, oWsf, prepped[parts[0]][2])
        assert W.shape[0] == {"qkv": 10240, "gateup": 51200}[fused]
        check_gemm(*acts[key], (gWq, gWsf), (oWq, oWsf), seed=M * 10 + len(fused))


@pytest.mark.parametrize("M", inputs.PREFILL_M)
@pytest.mark.parametrize("K", inputs.PREFILL_K)
@pytest.mark.parametrize("N", inputs.PREFILL_N)
def test_large_prefill(M, K, N):
    c = inputs.large_prefill(M, K, N)
    oWq, oWsf, oinv = oracle.prep_weights(c.W, c.s, 32)
    gWq, gWsf, ginv = check_gpu_weights(c.W, c.s, 32, oWq, oWsf, oinv)
    del c.W
    g_act, o_act = check_act(c.X, ginv, oinv, 32)
    check_gemm(g_act, o_act, (gWq, gWsf), (oWq, oWsf), seed=M + K + N)


@pytest.mark.parametrize("T", inputs.MOE_T)
@pytest.mark.parametrize("proj", ["gate_up", "down"])
def test_moe_30b_a3b(T, proj):
    """Grouped act-quant (per-expert s) and grouped GEMM: gate/up X_perm [8T, 2048] -> [8T, 1536],
    down [8T, 768] -> [8T, 2048], Zipf routing with empty experts at small T."""
    c = inputs.moe_30b_a3b(T, proj)
    E, N, K = c.W.shape
    off = c.offsets.numpy()
    oWq = np.empty((E, N, K // 2), np.uint8)
    oWsf = np.empty((E, N, K // 32), np.uint8)
    oinv = np.empty((E, K), np.float32)
    gWq = torch.empty(E, N, K // 2, dtype=torch.uint8, device="cuda")
    gWsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    ginv = torch.empty(E, K, dtype=torch.float32, device="cuda")
    Wd, sd = c.W.cuda(), c.s.cuda()
    for e in range(E):
        oWq[e], oWsf[e], oinv[e] = oracle.prep_weights(c.W[e], c.s[e], 32)
        mq.prep_weights(Wd[e], sd[e], 32, Wq=gWq[e], Wsf=gWsf[e], inv_s=ginv[e])
    del Wd
    np.testing.assert_array_equal(gWq.cpu().numpy(), oWq)
    gsf = gWsf.cpu().numpy()
    for e in range(E):
        np.testing.assert_array_equal(unswizzle(gsf[e], N, K), oWsf[e])
    oXq, oXsf = oracle.act_quant(c.X, oinv, 32, offsets=off)
    off_d = c.offsets.cuda()
    mq.check_group_offsets(c.offsets, int(off[-1]))
    gXq, gXsf = mq.act_quant(c.X.cuda(), ginv, 32, group_offsets=off_d)
    np.testing.assert_array_equal(gXq.cpu().numpy(), oXq)
    np.testing.assert_array_equal(unswizzle(gXsf.cpu().numpy(), off[-1], K, grouped_sf_rows(off)), oXsf)
    y32 = mq.grouped_linear(gXq, gXsf, off_d, gWq, gWsf, out_dtype=mq.OUT_F32)
    y16 = mq.grouped_linear(gXq, gXsf, off_d, gWq, gWsf, out_dtype=mq.OUT_BF16)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    rows = checked_rows(int(off[-1]), T + len(proj), tile_starts=grouped_tiles(off))
    Y, Tt = oracle.grouped_linear_matmul(oXq, oXsf, off, oWq, oWsf, rows=rows)
    close(y32, rows, Y, Tt)

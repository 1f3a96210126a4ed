"""GPU parity at the full sizes of the remaining workloads, on sampled outputs.

Qwen3-32B decoder layer (seven linears, four distinct inputs, heavy-tailed channels), the MoE
30B-A3B gate/up at T = 8192 (65536 routed rows over 128 experts), and the large-prefill dense sweep at
its smallest and largest shapes. Each side quantizes with its own code: the activation codes and
scales must match the oracle bit for bit over the whole tensor, the weight codes over the whole
matrix, and the GEMM on sampled rows (first, last and random ones) within 1e-5 of sum|terms|.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import unswizzle

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def sampled_rows(M, seed, n=6):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, n)]))


def close(y32, rows, Y, T):
    y = y32.double().cpu().numpy()[rows]
    err = np.abs(y - Y)
    assert np.all(err <= RTOL * T + 1e-30), f"worst rel {np.max(err / (T + 1e-30)):.3g}"


def check_layer(X, W, s, b, seed):
    """One dense layer through both sides; returns nothing, asserts every comparison."""
    M, K = X.shape
    N = W.shape[0]
    oWq, oWsf, oinv = oracle.prep_weights(W, s, b)
    gWq, gWsf, ginv = mq.prep_weights(W.cuda(), s.cuda(), b)
    np.testing.assert_array_equal(gWq.cpu().numpy(), oWq)
    np.testing.assert_array_equal(unswizzle(gWsf.cpu().numpy(), N, K), oWsf)
    oXq, oXsf = oracle.act_quant(X, oinv, b)
    gXq, gXsf = mq.act_quant(X.cuda(), ginv, b)
    np.testing.assert_array_equal(gXq.cpu().numpy(), oXq)
    np.testing.assert_array_equal(unswizzle(gXsf.cpu().numpy(), M, K), oXsf)
    y32 = mq.linear(gXq, gXsf, gWq, gWsf, out_dtype=mq.OUT_F32)
    y16 = mq.linear(gXq, gXsf, gWq, gWsf, out_dtype=mq.OUT_BF16)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
    rows = sampled_rows(M, seed)
    Y, T = oracle.linear(oXq, oXsf, oWq, oWsf, rows=rows)
    close(y32, rows, Y, T)


@pytest.mark.parametrize("M", [1, 64, 4096])
def test_qwen3_32b_layer(M):
    xs, ws = inputs.qwen3_32b_layer(M)
    for j, (name, K, N, key) in enumerate(inputs.QWEN3_32B_LINEARS):
        c = xs[key]
        check_layer(c.X, ws[name], c.s, 32, seed=M * 10 + j)


@pytest.mark.parametrize("M,K,N", [(4096, 8192, 8192), (16384, 16384, 28672)])
def test_large_prefill(M, K, N):
    c = inputs.large_prefill(M, K, N)
    check_layer(c.X, c.W, c.s, 32, seed=M + K + N)


def test_moe_gate_up_t8192():
    c = inputs.moe_30b_a3b(8192, "gate_up")
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
    np.testing.assert_array_equal(gWq.cpu().numpy(), oWq)
    oXq, oXsf = oracle.act_quant(c.X, oinv, 32, offsets=off)
    off_d = c.offsets.cuda()
    gXq, gXsf = mq.act_quant(c.X.cuda(), ginv, 32, group_offsets=off_d)
    np.testing.assert_array_equal(gXq.cpu().numpy(), oXq)
    y32 = mq.grouped_linear(gXq, gXsf, off_d, gWq, gWsf, out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    rows = sampled_rows(int(off[-1]), 8192, n=24)
    Y, T = oracle.grouped_linear(oXq, oXsf, off, oWq, oWsf, rows=rows)
    close(y32, rows, Y, T)

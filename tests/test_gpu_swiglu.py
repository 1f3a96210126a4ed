"""GPU parity of the down projection's input quantization fused after the gate/up GEMM (SwiGLU).

1. The standalone kernel (macaq_swiglu_act_quant) on seeded fp32 gate/up values: codes and scales bit
   for bit equal to the oracle's swiglu_act_quant (same fixed fp32 exp, same transform and MXFP4).
2. The fused GEMM epilogue (2-SM pair kernel, M > 128) against the GPU's two-step form (the same GEMM
   with fp32 output, then the standalone kernel): bit for bit, since both see the same accumulators.
3. End to end against the oracle on operands whose fp32 GEMM sums are exact (products are multiples
   of 2^-11 below 2^11 in magnitude), so the oracle's float64 GEMM rounded to fp32 is the accumulator
   value and every code must match, for the fused, skinny and general GEMM forms.
4. The Qwen3-32B gate/up -> down chain on realistic inputs: the accumulators differ from the oracle's
   float64 sums within the GEMM tolerance, so the check is on what that allows: scales within one
   step and different in under 0.5 % of groups (a group maximum at a power-of-two boundary), every
   element within two steps of the coarser grid, and fewer than 1 % of code bytes different. (GPU outputs are decoded by
   the test itself; the oracle only ever sees the seeded inputs.)
"""
import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs
from sfutil import Guarded, sf_index, swizzle, unswizzle

pytestmark = pytest.mark.gpu


def split_gu(GU):
    """[M, 2I] with 64-column gate/up blocks -> (G, U) [M, I]."""
    M, N = GU.shape
    v = GU.reshape(M, N // 128, 2, 64)
    return np.ascontiguousarray(v[:, :, 0].reshape(M, N // 2)), np.ascontiguousarray(v[:, :, 1].reshape(M, N // 2))


def check_h(hq, hsf, M, I, oq, osf):
    np.testing.assert_array_equal(hq.cpu().numpy(), oq)
    sf = hsf.cpu().numpy()
    np.testing.assert_array_equal(unswizzle(sf, M, I), osf)
    pad = np.arange(M, (M + 127) // 128 * 128)
    if pad.size:
        assert np.all(sf[sf_index(pad, I)] == 0), "padding rows of the SF must be zero"


@pytest.mark.parametrize("b", [1, 16, 32, 64])
@pytest.mark.parametrize("M,I", [(1, 128), (37, 768), (300, 256)])
def test_standalone_kernel_matches_oracle(M, I, b):
    rng = np.random.default_rng(M * 7 + I + b)
    GU = rng.normal(0, 3, (M, 2 * I)).astype(np.float32)
    # zeros, tiny values, and gates past the exp clamp at both ends (finite products: NaN and Inf are
    # outside the contract)
    GU[:, :8] = np.float32([0.0, -0.0, 1e-30, -1e-30, 150.0, -150.0, 1.0e4, -1.0e4])[None, :8]
    inv = np.exp(rng.uniform(-2.0, 0.7, I)).astype(np.float32)
    for with_s in (True, False):
        G, U = split_gu(GU)
        oq, osf = oracle.swiglu_act_quant(G, U, inv if with_s else None, b)
        hq = Guarded(M * I // 2, shape=(M, I // 2))
        hsf = Guarded(mq.sf_bytes(M, I))
        mq.swiglu_act_quant(torch.from_numpy(GU).cuda(), torch.from_numpy(inv).cuda() if with_s else None, b,
                            Hq=hq.t, Hsf=hsf.t)
        torch.cuda.synchronize()
        assert hq.intact() and hsf.intact()
        check_h(hq.t, hsf.t, M, I, oq, osf)


def random_ops(seed, M, N, K, a_scales=(112, 140), w_scales=(112, 140)):
    rng = np.random.default_rng(seed)
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Asf = rng.integers(a_scales[0], a_scales[1], (M, K // 32), dtype=np.uint8)
    Wsf = rng.integers(w_scales[0], w_scales[1], (N, K // 32), dtype=np.uint8)
    return Aq, Asf, Wq, Wsf


def to_gpu(Aq, Asf, Wq, Wsf):
    K = Aq.shape[1] * 2
    return (torch.from_numpy(Aq).cuda(), torch.from_numpy(swizzle(Asf, K)).cuda(), torch.from_numpy(Wq).cuda(),
            torch.from_numpy(swizzle(Wsf, K)).cuda())


@pytest.mark.parametrize("b", [1, 32, 64])
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (300, 768, 1024), (2048, 2816, 4096)])
def test_fused_epilogue_equals_two_step(M, N, K, b):
    Aq, Asf, Wq, Wsf = random_ops(M + N + K + b, M, N, K, (118, 126), (118, 126))
    dA, dAsf, dW, dWsf = to_gpu(Aq, Asf, Wq, Wsf)
    I = N // 2
    inv = torch.exp(torch.linspace(-2.0, 0.7, I)).to(torch.float32).cuda()
    hq, hsf = mq.linear_swiglu(dA, dAsf, dW, dWsf, inv, b)
    gu = mq.linear(dA, dAsf, dW, dWsf, out_dtype=mq.OUT_F32)
    rq, rsf = mq.swiglu_act_quant(gu, inv, b)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    assert torch.equal(hq, rq)
    assert torch.equal(hsf[:mq.sf_bytes(M, I)], rsf[:mq.sf_bytes(M, I)])


@pytest.mark.parametrize("M,N,K", [(300, 512, 4096), (16, 768, 4096), (16, 512, 1152), (130, 768, 2048)])
def test_exact_accumulation_end_to_end(M, N, K):
    """A scales fixed at 2^-3 and W scales in {2^-6, 2^-5}: every partial sum is a multiple of 2^-11
    below 2^11, exact in fp32 whatever the order, so the GPU accumulators equal the oracle's float64
    sums. M > 128 runs the fused epilogue; M = 16 the skinny GEMM (K % 256 == 0) or the general one
    (K = 1152), each followed by the standalone kernel."""
    Aq, Asf, Wq, Wsf = random_ops(3 * M + N + K, M, N, K, (124, 125), (121, 123))
    dA, dAsf, dW, dWsf = to_gpu(Aq, Asf, Wq, Wsf)
    Y, _ = oracle.linear_matmul(Aq, Asf, Wq, Wsf)
    assert np.array_equal(Y.astype(np.float32).astype(np.float64), Y), "the sums are not exact in fp32"
    GU = Y.astype(np.float32)
    I = N // 2
    inv = np.exp(np.linspace(-2.0, 0.7, I)).astype(np.float32)
    G, U = split_gu(GU)
    for b in (1, 32, 64):
        oq, osf = oracle.swiglu_act_quant(G, U, inv, b)
        hq, hsf = mq.linear_swiglu(dA, dAsf, dW, dWsf, torch.from_numpy(inv).cuda(), b)
        torch.cuda.synchronize()
        assert mq.device_status() == 0
        check_h(hq, hsf, M, I, oq, osf)


E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def decode(q, sf):
    """Values of MXFP4 rows (codes [rows, K/2], row-major scales [rows, K/32]) in float64: the
    documented layout, read back on the test side."""
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1)
    return E2M1[codes] * np.repeat(np.exp2(sf.astype(np.float64) - 127), 32, axis=1)


@pytest.mark.parametrize("M", [64, 4096])
def test_qwen3_32b_gate_up_down_chain(M):
    """X -> act_quant -> fused gate/up + SwiGLU + down act_quant -> down linear, on the Qwen3-32B
    shapes (5120 -> 2 x 25600 -> 5120), against the oracle's pipeline on checked rows."""
    xs, ws = inputs.qwen3_32b_layer(M)
    c, cd = xs["gateup"], xs["down"]
    Wgu = mq.interleave_gate_up(ws["gate_proj"], ws["up_proj"])
    oWq, oWsf, oinv = oracle.prep_weights(Wgu, c.s, 32)
    _, _, dinv = oracle.prep_weights(ws["down_proj"][:128], cd.s, 32)
    gWq, gWsf, ginv = mq.prep_weights(Wgu.cuda(), c.s.cuda(), 32)
    gdq, gdsf, gdinv = mq.prep_weights(ws["down_proj"].cuda(), cd.s.cuda(), 32)
    gXq, gXsf = mq.act_quant(c.X.cuda(), ginv, 32)
    hq, hsf = mq.linear_swiglu(gXq, gXsf, gWq, gWsf, gdinv, 32)
    y = mq.linear(hq, hsf, gdq, gdsf, out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    rows = np.arange(M) if M <= 64 else np.unique(np.concatenate(
        [np.arange(0, M, 128), np.arange(127, M, 128), np.random.default_rng(M).choice(M, 64, replace=False)]))
    oXq, oXsf = oracle.act_quant(c.X, oinv, 32)
    GUo, _ = oracle.linear_matmul(oXq, oXsf, oWq, oWsf, rows=rows)
    G, U = split_gu(GUo.astype(np.float32))
    oq, osf = oracle.swiglu_act_quant(G, U, dinv, 32)
    I = Wgu.shape[0] // 2
    gq = hq.cpu().numpy()[rows]
    gsf = unswizzle(hsf.cpu().numpy(), M, I)[rows]
    # a scale can differ only where the group's maximum sits at a power-of-two boundary, by one step
    assert np.all(np.abs(gsf.astype(np.int32) - osf.astype(np.int32)) <= 1)
    assert np.mean(gsf != osf) < 0.005
    o_val = oracle.dequant(oq, osf)
    g_val = decode(gq, gsf)
    top = np.repeat(np.maximum(gsf, osf).astype(np.float64), 32, axis=1)
    # each side rounds within one step of its grid (saturation included): two steps of the coarser one
    assert np.all(np.abs(g_val - o_val) <= np.exp2(top - 125) + 1e-30)
    assert np.mean(gq != oq) < 0.01
    assert bool(torch.isfinite(y).all())

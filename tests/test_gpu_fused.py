"""GPU parity of the fused layer (mode A_BF16_FUSED: bf16 X in, the call quantizes it).

The quantization is bit-exact and the GEMM plan is the same as for the quantized mode, so the fused
result must equal act_quant followed by the quantized linear bit for bit; it is also checked against
the oracle's pipeline (oracle act_quant, float64 GEMM) within 1e-5 of sum|terms| per element. M <= 4
with K % 256 == 0 runs the quantizer inside the skinny GEMM kernel; larger M runs the two-pass form.
Mode A_BF16_ONE_LAUNCH gives the same result; for M > 128 the 2-SM GEMM quantizes X itself in one
launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import inputs

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def layer(seed, M, N, K, b, with_s):
    c = inputs.dense_case(seed, M, K, N, n_outliers=3, outlier_factor=30.0, w_std=0.02)
    s = c.s if with_s else None
    Wq, Wsf, inv = mq.prep_weights(c.W.cuda(), None if s is None else s.cuda(), b)
    return c, Wq, Wsf, inv


def unfused(X, inv, b, Wq, Wsf, out_dtype):
    Xq, Xsf = mq.act_quant(X, inv, b)
    return mq.linear(Xq, Xsf, Wq, Wsf, out_dtype=out_dtype)


def fused(X, inv, b, Wq, Wsf, out_dtype, mode=mq.A_BF16_FUSED):
    return mq.linear(X, None, Wq, Wsf, mode=mode, inv_s=inv, had_block=b, out_dtype=out_dtype)


def counters_zero():
    """The workspace's counter region stays zero between calls, whatever scratch a call used."""
    ws = mq._workspace(torch.device("cuda"), 0)
    return int(ws[:mq.WORKSPACE_COUNTER_BYTES].count_nonzero()) == 0


def check_against_oracle(c, b, with_s, Wq_gpu, Wsf_gpu, y32, rows=None):
    """The oracle quantizes X itself; W' comes from the oracle's own weight prep."""
    s = c.s if with_s else None
    inv_s = None if s is None else (np.float32(1.0) / s.numpy()).astype(np.float32)
    Xq, Xsf = oracle.act_quant(c.X, inv_s, b)
    Wq, Wsf, _ = oracle.prep_weights(c.W, s, b)
    Y, T = oracle.linear(Xq, Xsf, Wq, Wsf, rows=rows)
    y = y32.double().cpu().numpy()
    if rows is not None:
        y = y[rows]
    err = np.abs(y - Y)
    assert np.all(err <= RTOL * T + 1e-30), f"worst rel {np.max(err / (T + 1e-30)):.3g}"


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("with_s", [True, False])
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (3, 512, 1024), (4, 1024, 4096)])
def test_in_kernel_fusion_equals_two_pass(M, N, K, b, with_s):
    c, Wq, Wsf, inv = layer(4000 + M + N + K + b, M, N, K, b, with_s)
    X = c.X.cuda()
    for out in (mq.OUT_F32, mq.OUT_BF16):
        ref = unfused(X, inv, b, Wq, Wsf, out)
        for _ in range(2):  # twice on one workspace: the counters must reset themselves
            got = fused(X, inv, b, Wq, Wsf, out)
            torch.cuda.synchronize()
            assert mq.device_status() == 0
            assert torch.equal(got.view(torch.int16 if out == mq.OUT_BF16 else torch.int32),
                               ref.view(torch.int16 if out == mq.OUT_BF16 else torch.int32))
    check_against_oracle(c, b, with_s, Wq, Wsf, got if out == mq.OUT_F32 else fused(X, inv, b, Wq, Wsf, mq.OUT_F32))


@pytest.mark.parametrize("M,N,K", [(16, 1024, 4096), (17, 512, 1024), (128, 256, 512), (300, 512, 1280), (7, 384, 384)])
def test_two_pass_fusion(M, N, K):
    """Shapes outside the in-kernel form (M > 4, or K % 256 != 0): quantizer pass + GEMM."""
    b = 32
    c, Wq, Wsf, inv = layer(5000 + M + N + K, M, N, K, b, True)
    X = c.X.cuda()
    ref = unfused(X, inv, b, Wq, Wsf, mq.OUT_F32)
    got = fused(X, inv, b, Wq, Wsf, mq.OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int32), ref.view(torch.int32))
    assert counters_zero()
    check_against_oracle(c, b, True, Wq, Wsf, got)


@pytest.mark.parametrize("M", [1, 16])
def test_llama3_8b_up_decode_fused(M):
    c = inputs.llama3_8b_up(M)
    Wq, Wsf, inv = mq.prep_weights(c.W.cuda(), c.s.cuda(), 32)
    X = c.X.cuda()
    ref = unfused(X, inv, 32, Wq, Wsf, mq.OUT_BF16)
    got = fused(X, inv, 32, Wq, Wsf, mq.OUT_BF16)
    y32 = fused(X, inv, 32, Wq, Wsf, mq.OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), got.view(torch.int16))
    check_against_oracle(c, 32, True, Wq, Wsf, y32, rows=np.unique([0, M - 1]))


@pytest.mark.parametrize("T,mode", [(64, mq.A_BF16_FUSED), (8192, mq.A_BF16_FUSED), (8192, mq.A_BF16_ONE_LAUNCH)])
def test_grouped_fused_equals_two_pass(T, mode):
    """The grouped fused call equals the grouped quantizer followed by the grouped GEMM bit for bit;
    at T = 8192 (512 rows per expert on average) the GEMM runs on 2-SM pairs. The one-launch mode
    behaves as the fused mode for grouped calls."""
    m = inputs.moe_30b_a3b(T, "gate_up")
    E = m.offsets.numel() - 1
    K = m.X.shape[1]
    W = m.W.cuda()
    N = W.shape[1]
    Wq = torch.empty(E, N, K // 2, dtype=torch.uint8, device="cuda")
    Wsf = torch.empty(E, mq.sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    inv = torch.empty(E, K, dtype=torch.float32, device="cuda")
    for e in range(E):
        mq.prep_weights(W[e], m.s[e].cuda(), 32, Wq=Wq[e], Wsf=Wsf[e], inv_s=inv[e])
    X, off = m.X.cuda(), m.offsets.cuda()
    Xq, Xsf = mq.act_quant(X, inv, 32, group_offsets=off)
    ref = mq.grouped_linear(Xq, Xsf, off, Wq, Wsf, out_dtype=mq.OUT_F32)
    got = mq.grouped_linear(X, None, off, Wq, Wsf, mode=mode, inv_s=inv, had_block=32, out_dtype=mq.OUT_F32)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    rows = np.arange(int(m.offsets[-1]))
    assert torch.equal(got[rows].view(torch.int32), ref[rows].view(torch.int32))
    assert counters_zero()
    if T != 64:
        return
    # a split-tile skinny call on the same workspace right after the grouped fused call
    c, Wq1, Wsf1, inv1 = layer(31, 64, 1024, 5120, 32, True)
    X1 = c.X.cuda()
    assert torch.equal(fused(X1, inv1, 32, Wq1, Wsf1, mq.OUT_F32).view(torch.int32),
                       unfused(X1, inv1, 32, Wq1, Wsf1, mq.OUT_F32).view(torch.int32))
    check_against_oracle(c, 32, True, Wq1, Wsf1, unfused(X1, inv1, 32, Wq1, Wsf1, mq.OUT_F32), rows=np.array([0, 63]))


def test_fused_needs_a_workspace():
    c, Wq, Wsf, inv = layer(77, 4, 256, 256, 32, True)
    X = c.X.cuda()
    Y = torch.empty(4, 256, dtype=torch.bfloat16, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = mq.lib().macaq_linear(mq.A_BF16_FUSED, X.data_ptr(), None, inv.data_ptr(), 4, 256, 256, 32,
                                   Wq.data_ptr(), Wsf.data_ptr(), Y.data_ptr(), mq.OUT_BF16, None, 0, st)
    assert mq.status_str(status) == "MACAQ_ERR_WORKSPACE"
    assert mq.fused_workspace_bytes(4, 256, 256) > mq.WORKSPACE_COUNTER_BYTES


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (300, 768, 1024), (2048, 14336 // 4, 4096), (4160, 1024, 8192),
                                   (2048, 14336, 512), (1300, 14336, 1024)])
def test_in_gemm_quantization_large_m(M, N, K, b):
    """Mode A_BF16_ONE_LAUNCH, M > 128 with N and K multiples of 256: one launch, the 2-SM GEMM quantizes X itself (its
    epilogue warps, between tiles) and reads A back by TMA. The result equals act_quant followed by
    the quantized layer bit for bit, twice in a row on one workspace, and the counter region is zero
    afterwards. N = 14336 gives 56 column tiles, so the host cuts the raster into bands of three
    256-row tiles: 2048 rows make three bands (the last one of two), 1300 rows two bands with a
    partial last row tile; 4160 rows at N = 1024 make a second, partial band of the default height."""
    c, Wq, Wsf, inv = layer(6000 + M + N + K + b, M, N, K, b, True)
    X = c.X.cuda()
    ref = unfused(X, inv, b, Wq, Wsf, mq.OUT_F32)
    ref16 = unfused(X, inv, b, Wq, Wsf, mq.OUT_BF16)
    for _ in range(2):
        got = fused(X, inv, b, Wq, Wsf, mq.OUT_F32, mq.A_BF16_ONE_LAUNCH)
        got16 = fused(X, inv, b, Wq, Wsf, mq.OUT_BF16, mq.A_BF16_ONE_LAUNCH)
        torch.cuda.synchronize()
        assert mq.device_status() == 0
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32))
        assert torch.equal(got16.view(torch.int16), ref16.view(torch.int16))
        assert counters_zero()
    if b == 32:
        rows = np.unique(np.concatenate([[0, M - 1], np.arange(127, M, 128)]))[:24]
        check_against_oracle(c, b, True, Wq, Wsf, got, rows=rows)


def test_in_gemm_quantization_wait_runs_out_and_resets():
    """A 1 ns wait limit makes the producers' ready-count waits (and the pipeline waits) run out: the
    kernel reports MACAQ_ERR_TIMEOUT, the last CTA still zeroes the counters, and the next call is
    exact again."""
    M, N, K = 512, 512, 1024
    c, Wq, Wsf, inv = layer(78, M, N, K, 32, True)
    X = c.X.cuda()
    ref = unfused(X, inv, 32, Wq, Wsf, mq.OUT_F32)
    torch.cuda.synchronize()
    mq.device_status(reset=True)
    try:
        mq.set_wait_limit_ns(1)
        fused(X, inv, 32, Wq, Wsf, mq.OUT_F32, mq.A_BF16_ONE_LAUNCH)
        torch.cuda.synchronize()
    finally:
        mq.set_wait_limit_ns(0)
    assert mq.device_status(reset=True) == 6
    assert counters_zero()
    got = fused(X, inv, 32, Wq, Wsf, mq.OUT_F32, mq.A_BF16_ONE_LAUNCH)
    torch.cuda.synchronize()
    assert mq.device_status() == 0
    assert torch.equal(got.view(torch.int32), ref.view(torch.int32))
